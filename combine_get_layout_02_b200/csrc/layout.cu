// Dispatch layout on the GPU: per-expert / per-rank counts, prefix sums and the
// stable receive row of every (token, slot) copy.
//
// The DeepEP pages describe dispatch only as routing each token to its gated
// experts, with the host waiting on GPU-made receive counts (brainleap "Day2
// DeepEP", caption "CPU 将隐式地等待 GPU 接收到的计数信号").  The order inside
// an expert is ascending token order: the result equals one sequential walk
// over t = 0..N-1, j = 0..k-1 that hands out the next free row of each expert.
//
// Block b owns tokens [256 b, 256 b + 256); in the per-token phases thread i
// owns token 256 b + i, so warp w owns 32 consecutive tokens, one per lane.
//
//   histogram : the block's ids are loaded coalesced (8 independent loads per
//               thread) into shared memory and counted per expert; each token
//               builds its rank set (a 64-bit register mask, or shared-memory
//               words for R > 64), which gives tokens_per_rank and the
//               is_token_in_rank row; the block's expert and rank counts go to
//               its row of the workspace.
//   bases     : every block reads the workspace table column-wise (16
//               independent loads per thread) to get, per expert, the total
//               and the copies in earlier blocks; an exclusive scan over
//               experts gives expert_offset, hence the block's first row per
//               expert.  Block 0 writes the global counts, offsets and max.
//   ranks     : each warp marks, per expert, which of its lanes route there (a
//               32-bit lane mask); a copy's row is the block base plus the
//               popcounts of that expert's masks in lower warps plus the lower
//               lanes of its own warp's mask.  A token that names one expert
//               twice makes the block fall back to an in-order walk over
//               32-pair chunks with __match_any_sync.
//
// Launch shapes.  When every block fits on the GPU at once (all prefill and
// decode shapes here), one cooperative kernel does all three phases and the
// blocks exchange histograms through the workspace: each block publishes its
// row, then release-stores a 64-bit tag unique to the call into its flag word,
// and waits, with a bounded spin (CGL_ETIMEOUT after ~1 s), until every flag
// shows that tag.  Otherwise two kernels run: histogram, then bases + ranks,
// the second launched with programmatic dependent launch.
#include <atomic>
#include <chrono>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokensPerBlock = kThreads;            // one token per thread in the per-token phases
constexpr int kTokensPerWarp = kTokensPerBlock / kWarps;
constexpr int kUnroll = 8;                           // independent id loads per thread
constexpr int kColUnroll = 16;                       // independent histogram loads per thread
constexpr int kMaxFusedBlocks = kThreads;            // the fused kernel polls one flag per thread
constexpr size_t kSmemDefault = 47 * 1024;           // dynamic bytes that need no opt-in (48 KiB minus
                                                     // room for the kernels' static shared memory)
constexpr long long kWaitCycles = 1LL << 31;         // bound on the inter-block wait (~1 s)

__device__ __forceinline__ int tokens_in_block(int64_t n, int64_t t0) {
    const int64_t rem = n - t0;
    return rem <= 0 ? 0 : (rem < kTokensPerBlock ? (int)rem : kTokensPerBlock);
}

// Workspace: [flags: blocks x u64][pad to 256 B][expert counts: blocks x E][pad][rank counts: blocks x R]
struct WsLayout {
    int64_t blocks;
    size_t e_off, r_off, bytes;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

WsLayout ws_layout(int64_t n, int E, int R) {
    WsLayout w;
    w.blocks = n > 0 ? (n + kTokensPerBlock - 1) / kTokensPerBlock : 1;
    w.e_off = align256((size_t)w.blocks * sizeof(uint64_t));
    w.r_off = w.e_off + align256((size_t)w.blocks * (size_t)E * sizeof(int32_t));
    w.bytes = w.r_off + (size_t)w.blocks * (size_t)R * sizeof(int32_t);
    return w;
}

__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__host__ __device__ __forceinline__ int rank_mask_words(int R) { return R > 64 ? (R + 31) >> 5 : 0; }

// Shared-memory regions; a null region is not used by that kernel.
struct Smem {
    int32_t *idx;      // [kTokensPerBlock][ks] ids, odd row stride ks = k | 1 (no bank conflicts)
    int32_t *he;       // [E] this block's copies per expert
    int32_t *hr;       // [R] this block's tokens per rank
    uint32_t *rmask;   // [kTokensPerBlock][rw] rank masks when R > 64
    int32_t *total;    // [E] copies per expert, all blocks
    int32_t *base;     // [E] first receive row of this block's copies
    int32_t *off;      // [E] exclusive prefix of total
    uint32_t *lanes;   // [kWarps][E] lanes of each warp routing to e (per-warp counts on the fallback walk)
};

// Words of dynamic shared memory.  kind 0: fused kernel, 1: histogram kernel, 2: assign kernel.
__host__ __device__ __forceinline__ size_t smem_words(int kind, int k, int E, int R) {
    const size_t ids = (size_t)kTokensPerBlock * (size_t)(k | 1);
    const size_t hist = (size_t)E + (size_t)R + (size_t)kTokensPerBlock * rank_mask_words(R);
    const size_t rank = 3 * (size_t)E + (size_t)kWarps * E;
    return ids + (kind != 2 ? hist : 0) + (kind != 1 ? rank : 0);
}

__device__ Smem carve(int kind, int32_t *p, int k, int E, int R) {
    Smem s = {};
    s.idx = p;
    p += kTokensPerBlock * (k | 1);
    if (kind != 2) {
        s.he = p; p += E;
        s.hr = p; p += R;
        s.rmask = reinterpret_cast<uint32_t *>(p);
        p += kTokensPerBlock * rank_mask_words(R);
    }
    if (kind != 1) {
        s.total = p; p += E;
        s.base = p; p += E;
        s.off = p; p += E;
        s.lanes = reinterpret_cast<uint32_t *>(p);
    }
    return s;
}

__device__ void zero_shared(const Smem &s, int E, int R) {
    const int tid = threadIdx.x;
    if (s.he)
        for (int i = tid; i < E; i += kThreads) s.he[i] = 0;
    if (s.hr)
        for (int i = tid; i < R; i += kThreads) s.hr[i] = 0;
    if (s.rmask)
        for (int i = tid; i < kTokensPerBlock * rank_mask_words(R); i += kThreads) s.rmask[i] = 0;
    if (s.lanes)
        for (int i = tid; i < kWarps * E; i += kThreads) s.lanes[i] = 0;
}

// Load the block's ids into s.idx (coalesced, kUnroll loads in flight per
// thread); with kCount also histogram them into s.he.  Returns true if an id
// outside [-1, E) was seen.
template <bool kCount>
__device__ bool load_ids(const int32_t *__restrict__ idx, int64_t t0, int nt, int k, int E, const Smem &s) {
    const int tid = threadIdx.x;
    const int ks = k | 1;
    const int pairs = nt * k;
    const int32_t *src = idx + t0 * k;
    bool bad = false;
    for (int base = 0; base < pairs; base += kThreads * kUnroll) {
        int32_t ev[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int p = base + u * kThreads + tid;
            ev[u] = p < pairs ? __ldg(src + p) : -1;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int p = base + u * kThreads + tid;
            if (p >= pairs) continue;
            const int tl = p / k;
            const int32_t e = ev[u];
            s.idx[tl * ks + (p - tl * k)] = e;
            if (e == -1) continue;
            if (e < -1 || e >= E) { bad = true; continue; }
            if (kCount) atomicAdd(&s.he[e], 1);
        }
    }
    return bad;
}

// Per-token pass (thread = token).  kRanks: build the token's rank set, count
// it into s.hr and, for R <= 64, write its is_token_in_rank row (larger R is
// written by write_rank_rows).  kLanes: mark the token's experts in its warp's
// lane masks.  Returns true if the token names one expert twice.
template <bool kRanks, bool kLanes>
__device__ bool per_token(int64_t t0, int nt, int k, int E, int R, uint8_t *__restrict__ in_rank,
                          const Smem &s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid >= nt) return false;
    const int per = E / R;
    const int rw = rank_mask_words(R);
    const int32_t *my = s.idx + tid * (k | 1);
    uint64_t m64 = 0;
    bool dup = false;
    for (int j = 0; j < k; ++j) {
        const int32_t e = my[j];
        if (e < 0 || e >= E) continue;
        for (int jj = 0; jj < j; ++jj) dup |= (my[jj] == e);
        if (kLanes) atomicOr(&s.lanes[warp * E + e], 1u << lane);
        if (kRanks) {
            const int r = e / per;
            bool fresh;
            if (R <= 64) {
                const uint64_t bit = 1ull << r;
                fresh = !(m64 & bit);
                m64 |= bit;
            } else {
                uint32_t &wd = s.rmask[tid * rw + (r >> 5)];
                const uint32_t bit = 1u << (r & 31);
                fresh = !(wd & bit);
                wd |= bit;
            }
            if (fresh) atomicAdd(&s.hr[r], 1);
        }
    }
    if (kRanks && R <= 64) {
        uint8_t *row = in_rank + (t0 + tid) * R;
        if ((R & 15) == 0) {   // 16-byte aligned: (t0 + tid) * R is a multiple of 16
            for (int q = 0; q < R; q += 16) {
                const uint32_t bits = (uint32_t)(m64 >> q) & 0xFFFFu;
                uint32_t wv[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) wv[j] = (((bits >> (4 * j)) & 0xFu) * 0x00204081u) & 0x01010101u;
                *reinterpret_cast<uint4 *>(row + q) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        } else {
            for (int r = 0; r < R; ++r) row[r] = (uint8_t)((m64 >> r) & 1u);
        }
    }
    return dup;
}

// is_token_in_rank rows of the block from the shared-memory masks (R > 64).
// The block's rows are contiguous and 16-byte aligned.  Needs a barrier before.
__device__ void write_rank_rows(int64_t t0, int nt, int R, uint8_t *__restrict__ in_rank, const Smem &s) {
    const int tid = threadIdx.x;
    const int rw = rank_mask_words(R);
    uint8_t *row0 = in_rank + t0 * R;
    const int nbytes = nt * R;
    if ((R & 15) == 0) {
        for (int q = tid * 16; q < nbytes; q += kThreads * 16) {
            const int tl = q / R, r0 = q - tl * R;
            const uint32_t bits = (s.rmask[tl * rw + (r0 >> 5)] >> (r0 & 31)) & 0xFFFFu;
            uint32_t wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = (((bits >> (4 * j)) & 0xFu) * 0x00204081u) & 0x01010101u;
            *reinterpret_cast<uint4 *>(row0 + q) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    } else {
        for (int q = tid; q < nbytes; q += kThreads) {
            const int tl = q / R, r = q - tl * R;
            row0[q] = (uint8_t)((s.rmask[tl * rw + (r >> 5)] >> (r & 31)) & 1u);
        }
    }
}

// Sum of column c of a [rows][ncols] table, and of its rows [0, upto) into *pre.
// kCoherent: read through L2 only (the table was written by other blocks of the
// running grid); otherwise through the read-only path (written by an earlier kernel).
template <bool kCoherent>
__device__ __forceinline__ int32_t column_sum(const int32_t *t, int rows, int ncols, int c, int upto,
                                              int32_t *pre) {
    int32_t tot = 0, p = 0;
    for (int r0 = 0; r0 < rows; r0 += kColUnroll) {
        int32_t v[kColUnroll];
#pragma unroll
        for (int u = 0; u < kColUnroll; ++u) {
            const int32_t *a = t + (int64_t)(r0 + u) * ncols + c;
            v[u] = r0 + u < rows ? (kCoherent ? __ldcg(a) : __ldg(a)) : 0;
        }
#pragma unroll
        for (int u = 0; u < kColUnroll; ++u) {
            tot += v[u];
            p += r0 + u < upto ? v[u] : 0;
        }
    }
    *pre = p;
    return tot;
}

// Exclusive scan of v[0..n) in shared memory (n <= kMaxExperts) into out[];
// returns the total.  All threads of the block must call it.
__device__ int32_t block_exclusive_scan(const int32_t *v, int32_t *out, int n, int32_t *warp_sums) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kThreads - 1) / kThreads;   // <= 4
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int32_t local = 0;
    for (int i = i0; i < i1; ++i) local += v[i];
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t s = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xFFFFFFFFu, s, o);
            if (lane >= o) s += u;
        }
        if (lane < kWarps) warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    int32_t run = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - local;
    for (int i = i0; i < i1; ++i) {
        out[i] = run;
        run += v[i];
    }
    const int32_t total = warp_sums[kWarps - 1];
    __syncthreads();
    return total;
}

// Bases phase: s.total, s.off, s.base from the workspace table; block 0 writes
// the global counts; all blocks share filling recv_src = -1 for unused rows.
template <bool kCoherent>
__device__ void block_bases(const int32_t *ws_e, const int32_t *ws_r, int64_t n, int k, int E, int R,
                            int cap, int32_t *__restrict__ tokens_per_expert,
                            int32_t *__restrict__ tokens_per_rank, int32_t *__restrict__ expert_offset,
                            int32_t *__restrict__ max_count, int32_t *__restrict__ recv_src,
                            const Smem &s, int32_t *scan_tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = gridDim.x, b = blockIdx.x;
    for (int e = tid; e < E; e += kThreads) {
        int32_t pre;
        s.total[e] = column_sum<kCoherent>(ws_e, nb, E, e, b, &pre);
        s.base[e] = pre;
    }
    __syncthreads();
    const int32_t m_total = block_exclusive_scan(s.total, s.off, E, scan_tmp);
    for (int e = tid; e < E; e += kThreads) s.base[e] += cap > 0 ? e * cap : s.off[e];

    if (b == 0) {
        int32_t mx = 0;
        for (int e = tid; e < E; e += kThreads) {
            tokens_per_expert[e] = s.total[e];
            expert_offset[e] = s.off[e];
            mx = max(mx, s.total[e]);
        }
        if (tid == 0) expert_offset[E] = m_total;
        for (int r = tid; r < R; r += kThreads) {
            int32_t unused;
            tokens_per_rank[r] = column_sum<kCoherent>(ws_r, nb, R, r, 0, &unused);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if (lane == 0) scan_tmp[warp] = mx;
        __syncthreads();
        if (tid == 0) {
            int32_t m = 0;
            for (int w = 0; w < kWarps; ++w) m = max(m, scan_tmp[w]);
            *max_count = m;
        }
    }

    const int64_t step = (int64_t)nb * kThreads;
    if (cap > 0) {
        const int64_t rows = (int64_t)E * cap;
        for (int64_t i = (int64_t)b * kThreads + tid; i < rows; i += step) {
            const int e = (int)(i / cap);
            if (i - (int64_t)e * cap >= s.total[e]) recv_src[i] = -1;
        }
    } else {
        for (int64_t i = m_total + (int64_t)b * kThreads + tid; i < n * k; i += step) recv_src[i] = -1;
    }
    __syncthreads();
}

// Ranks phase.  `any_dup` is block-uniform.  When !any_dup, s.lanes must hold
// the complete lane masks (barrier before).
__device__ void block_ranks(int64_t t0, int nt, int k, int E, int cap, int64_t recv_rows, bool any_dup,
                            int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src,
                            uint32_t *status, const Smem &s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ks = k | 1;
    bool over = false, bad_row = false;
    if (!any_dup) {
        if (tid < nt) {
            const int32_t *my = s.idx + tid * ks;
            const uint32_t lower = (1u << lane) - 1u;
            for (int j = 0; j < k; ++j) {
                const int32_t e = my[j];
                int32_t d = -1;
                if (e >= 0 && e < E) {
                    int32_t pos = s.base[e] + __popc(s.lanes[warp * E + e] & lower);
                    for (int w = 0; w < warp; ++w) pos += __popc(s.lanes[w * E + e]);
                    if (cap > 0 && pos - e * cap >= cap) over = true;
                    else if (pos >= recv_rows) bad_row = true;
                    else d = pos;
                }
                const int64_t q = (t0 + tid) * k + j;
                dst_pos[q] = d;
                if (d >= 0) recv_src[d] = (int32_t)q;
            }
        }
    } else {
        // in-order walk: per-warp counts (in the lane-mask words), per-expert warp scan, rows
        int32_t *cnt = reinterpret_cast<int32_t *>(s.lanes);
        const int p_begin = warp * kTokensPerWarp * k;
        const int p_end = min(p_begin + kTokensPerWarp * k, nt * k);
        int32_t *wc = cnt + warp * E;
        for (int e = lane; e < E; e += 32) wc[e] = 0;
        __syncwarp();
        for (int p = p_begin + lane; p < p_end; p += 32) {
            const int tl = p / k;
            const int32_t e = s.idx[tl * ks + (p - tl * k)];
            if (e >= 0 && e < E) atomicAdd(&wc[e], 1);
        }
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) {
            int32_t run = s.base[e];
            for (int w = 0; w < kWarps; ++w) {
                const int32_t c = cnt[w * E + e];
                cnt[w * E + e] = run;
                run += c;
            }
        }
        __syncthreads();
        for (int p0 = p_begin; p0 < p_end; p0 += 32) {
            const int p = p0 + lane;
            const int tl = p / k;
            const int32_t e = p < p_end ? s.idx[tl * ks + (p - tl * k)] : -1;
            const bool valid = e >= 0 && e < E;
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? e : -1);
            const int32_t pos = valid ? wc[e] + __popc(peers & ((1u << lane) - 1u)) : -1;
            __syncwarp();
            if (valid && lane == 31 - __clz(peers)) wc[e] += __popc(peers);
            __syncwarp();
            if (p < p_end) {
                int32_t d = -1;
                if (valid) {
                    if (cap > 0 && pos - e * cap >= cap) over = true;
                    else if (pos >= recv_rows) bad_row = true;
                    else d = pos;
                }
                const int64_t q = t0 * k + p;
                dst_pos[q] = d;
                if (d >= 0) recv_src[d] = (int32_t)q;
            }
        }
    }
    if (over) report(status, kErrCapacity);
    if (bad_row) report(status, kErrRange);
}

// ------------------------------------------------------------------ kernels

__global__ void __launch_bounds__(kThreads)
layout_fused_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap,
                    uint64_t *flags, int32_t *ws_e, int32_t *ws_r, uint64_t tag,
                    int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                    uint8_t *__restrict__ in_rank, int32_t *__restrict__ expert_offset,
                    int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                    int32_t *__restrict__ recv_src, int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_fused[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve(0, smem_fused, k, E, R);
    const int tid = threadIdx.x;
    const int nb = gridDim.x, b = blockIdx.x;
    const int64_t t0 = (int64_t)b * kTokensPerBlock;
    const int nt = tokens_in_block(n, t0);

    griddep_launch_dependents();   // the copy kernels may get resident; they wait for this grid
    zero_shared(s, E, R);
    __syncthreads();
    const bool bad = load_ids<true>(idx, t0, nt, k, E, s);
    __syncthreads();
    const bool dup = per_token<true, true>(t0, nt, k, E, R, in_rank, s);
    __syncthreads();
    if (R > 64) write_rank_rows(t0, nt, R, in_rank, s);
    for (int i = tid; i < E; i += kThreads) ws_e[(int64_t)b * E + i] = s.he[i];
    for (int i = tid; i < R; i += kThreads) ws_r[(int64_t)b * R + i] = s.hr[i];
    const bool any_bad = __syncthreads_or(bad);   // also orders the workspace writes before the flag
    const bool any_dup = __syncthreads_or(dup);
    if (tid == 0) {
        __threadfence();
        st_release_u64(flags + b, tag);
        if (any_bad) report(status, kErrRange);
    }

    // every block's histogram row must be visible before the bases phase
    bool timed_out = false;
    if (tid < nb) {
        const long long start = clock64();
        while (ld_acquire_u64(flags + tid) != tag) {
            if (clock64() - start > kWaitCycles) { timed_out = true; break; }
            __nanosleep(100);
        }
        __threadfence();
    }
    if (__syncthreads_or(timed_out)) {
        if (tid == 0) report(status, 1u << CGL_ETIMEOUT);
        return;
    }
    block_bases<true>(ws_e, ws_r, n, k, E, R, cap, tokens_per_expert, tokens_per_rank, expert_offset,
                      max_count, recv_src, s, scan_tmp);
    block_ranks(t0, nt, k, E, cap, recv_rows, any_dup, dst_pos, recv_src, status, s);
}

__global__ void __launch_bounds__(kThreads)
layout_count_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R,
                    int32_t *__restrict__ ws_e, int32_t *__restrict__ ws_r,
                    uint8_t *__restrict__ in_rank, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_count[];
    const Smem s = carve(1, smem_count, k, E, R);
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * kTokensPerBlock;
    const int nt = tokens_in_block(n, t0);

    griddep_launch_dependents();   // the assign kernel may start; it waits for this grid
    zero_shared(s, E, R);
    __syncthreads();
    const bool bad = load_ids<true>(idx, t0, nt, k, E, s);
    __syncthreads();
    per_token<true, false>(t0, nt, k, E, R, in_rank, s);
    __syncthreads();
    if (R > 64) write_rank_rows(t0, nt, R, in_rank, s);
    for (int i = tid; i < E; i += kThreads) ws_e[(int64_t)blockIdx.x * E + i] = s.he[i];
    for (int i = tid; i < R; i += kThreads) ws_r[(int64_t)blockIdx.x * R + i] = s.hr[i];
    if (__syncthreads_or(bad) && tid == 0) report(status, kErrRange);
}

__global__ void __launch_bounds__(kThreads)
layout_assign_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap,
                     const int32_t *__restrict__ ws_e, const int32_t *__restrict__ ws_r,
                     int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                     int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                     int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src,
                     int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_assign[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve(2, smem_assign, k, E, R);
    const int64_t t0 = (int64_t)blockIdx.x * kTokensPerBlock;
    const int nt = tokens_in_block(n, t0);

    griddep_launch_dependents();   // the copy kernels may get resident; they wait for this grid
    zero_shared(s, E, R);
    __syncthreads();
    // topk_idx is not written by the histogram kernel, which started only after
    // everything before it in the stream had finished: it may be read before the wait
    load_ids<false>(idx, t0, nt, k, E, s);
    __syncthreads();
    const bool dup = per_token<false, true>(t0, nt, k, E, R, nullptr, s);
    const bool any_dup = __syncthreads_or(dup);
    griddep_wait();
    block_bases<false>(ws_e, ws_r, n, k, E, R, cap, tokens_per_expert, tokens_per_rank, expert_offset,
                       max_count, recv_src, s, scan_tmp);
    block_ranks(t0, nt, k, E, cap, recv_rows, any_dup, dst_pos, recv_src, status, s);
}

// ------------------------------------------------------------------ host side

std::mutex g_mu;
int g_fused_ctas_per_sm[64] = {0};   // fused-kernel occupancy at kSmemDefault, per device (-1: none)

// Largest grid of the fused kernel that is certain to be co-resident; 0 if none.
int fused_capacity() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_fused_ctas_per_sm[dev] == 0) {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, layout_fused_kernel, kThreads,
                                                          kSmemDefault) != cudaSuccess)
            return 0;
        g_fused_ctas_per_sm[dev] = v > 0 ? v : -1;
    }
    const int per_sm = g_fused_ctas_per_sm[dev];
    return per_sm > 0 ? per_sm * device_sm_count() : 0;
}

// A 64-bit tag unique to each call: a per-process salt (never 0) in the high
// half and a call counter in the low half, so no flag left by another call,
// and no freshly zeroed memory, can match it.
uint64_t next_tag() {
    static std::atomic<uint64_t> counter{0};
    static const uint64_t salt = [] {
        uint64_t v = (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
        v ^= v >> 29;
        v *= 0xBF58476D1CE4E5B9ull;
        v ^= v >> 32;
        return (v & 0xFFFFFFFFull) | 1ull;
    }();
    return (salt << 32) | ((counter.fetch_add(1) + 1) & 0xFFFFFFFFull);
}

}  // namespace

size_t layout_workspace_bytes(int64_t n, int E, int R) { return ws_layout(n, E, R).bytes; }

bool layout_needs_smem_optin(int E, int R, int k) {
    return smem_words(0, k, E, R) * sizeof(int32_t) > kSmemDefault;
}

bool layout_fused_fits(int64_t n, int k, int E, int R) {
    const WsLayout w = ws_layout(n, E, R);
    return smem_words(0, k, E, R) * sizeof(int32_t) <= kSmemDefault && w.blocks <= kMaxFusedBlocks &&
           w.blocks <= fused_capacity();
}

cgl_status launch_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                         int32_t *tokens_per_expert, int32_t *tokens_per_rank, uint8_t *in_rank,
                         int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                         int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream) {
    const WsLayout w = ws_layout(n, E, R);
    uint64_t *flags = static_cast<uint64_t *>(ws);
    int32_t *ws_e = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.e_off);
    int32_t *ws_r = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.r_off);
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;

    if (layout_fused_fits(n, k, E, R)) {
        const size_t smem0 = smem_words(0, k, E, R) * sizeof(int32_t);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)w.blocks);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t err = cudaLaunchKernelEx(
            &cfg, layout_fused_kernel, idx, n, k, E, R, cap, flags, ws_e, ws_r, next_tag(),
            tokens_per_expert, tokens_per_rank, in_rank, expert_offset, max_count, dst_pos, recv_src,
            recv_rows, status);
        return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
    }

    const size_t smem1 = smem_words(1, k, E, R) * sizeof(int32_t);
    const size_t smem2 = smem_words(2, k, E, R) * sizeof(int32_t);
    if (smem1 > kSmemDefault && !ensure_smem_attr((const void *)layout_count_kernel, smem1)) return CGL_ECUDA;
    if (smem2 > kSmemDefault && !ensure_smem_attr((const void *)layout_assign_kernel, smem2)) return CGL_ECUDA;
    layout_count_kernel<<<(unsigned)w.blocks, kThreads, smem1, stream>>>(idx, n, k, E, R, ws_e, ws_r,
                                                                          in_rank, status);
    if (cudaGetLastError() != cudaSuccess) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(layout_assign_kernel, dim3((unsigned)w.blocks), dim3(kThreads), smem2,
                                       stream, idx, n, k, E, R, cap, (const int32_t *)ws_e,
                                       (const int32_t *)ws_r, tokens_per_expert, tokens_per_rank,
                                       expert_offset, max_count, dst_pos, recv_src, recv_rows, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
