// Dispatch layout on the GPU: per-expert / per-rank counts, prefix sums and the
// stable receive row of every (token, slot) copy.
//
// The DeepEP pages describe dispatch only as routing each token to its gated
// experts, with the host waiting on GPU-made receive counts (brainleap "Day2
// DeepEP", caption "CPU 将隐式地等待 GPU 接收到的计数信号").  The order inside
// an expert is ascending token order: the result equals one sequential walk
// over t = 0..N-1, j = 0..k-1 that hands out the next free row of each expert.
//
// Two launches, no global atomics and no inter-block waiting:
//   count  : block b histograms the expert ids of its 256 tokens (shared-memory
//            atomics) and marks is_token_in_rank; the histograms go to the
//            workspace, one row per block.
//   assign : every block re-reads the (small) histogram table to get its own
//            starting row per expert (expert offset + copies in earlier
//            blocks), then ranks its pairs in order: each warp owns 32
//            consecutive tokens, counts its pairs per expert with
//            __match_any_sync, a per-expert scan over the 8 warps gives each
//            warp its base, and a second walk hands out rows.  Block 0 also
//            writes the global counts, offsets and max.
#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokensPerBlock = 256;
constexpr int kTokensPerWarp = kTokensPerBlock / kWarps;

__device__ __forceinline__ int tokens_in_block(int64_t n, int64_t t0) {
    const int64_t rem = n - t0;
    return rem <= 0 ? 0 : (rem < kTokensPerBlock ? (int)rem : kTokensPerBlock);
}

struct WsLayout {
    int64_t blocks;
    size_t rank_off;   // byte offset of the per-block rank histograms
    size_t bytes;
};

WsLayout ws_layout(int64_t n, int e, int r) {
    WsLayout w;
    w.blocks = n > 0 ? (n + kTokensPerBlock - 1) / kTokensPerBlock : 1;
    size_t eb = (size_t)w.blocks * (size_t)e * sizeof(int32_t);
    w.rank_off = (eb + 255) / 256 * 256;
    w.bytes = w.rank_off + (size_t)w.blocks * (size_t)r * sizeof(int32_t);
    return w;
}

__global__ void __launch_bounds__(kThreads)
layout_count_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R,
                    int32_t *__restrict__ ws_e, int32_t *__restrict__ ws_r,
                    uint8_t *__restrict__ in_rank, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_count[];
    int32_t *h_e = smem_count;   // [E]
    int32_t *h_r = h_e + E;      // [R]
    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * kTokensPerBlock;
    const int nt = tokens_in_block(n, t0);

    for (int i = tid; i < E; i += kThreads) h_e[i] = 0;
    for (int i = tid; i < R; i += kThreads) h_r[i] = 0;
    // zero this block's rows of is_token_in_rank (16-byte aligned: t0*R is a multiple of 256)
    {
        uint8_t *row0 = in_rank + t0 * R;
        const int64_t nbytes = (int64_t)nt * R;
        const int64_t nvec = nbytes / 16;
        for (int64_t i = tid; i < nvec; i += kThreads)
            reinterpret_cast<uint4 *>(row0)[i] = make_uint4(0, 0, 0, 0);
        for (int64_t i = nvec * 16 + tid; i < nbytes; i += kThreads) row0[i] = 0;
    }
    __syncthreads();

    bool bad = false;
    if (tid < nt) {
        const int64_t t = t0 + tid;
        const int32_t *my = idx + t * k;
        const int per = E / R;
        int ranks[kMaxTopk];
        for (int j = 0; j < k; ++j) {
            const int32_t e = __ldg(my + j);
            ranks[j] = -1;
            if (e == -1) continue;
            if (e < -1 || e >= E) { bad = true; continue; }
            atomicAdd(&h_e[e], 1);
            const int r = e / per;
            bool seen = false;
            for (int jj = 0; jj < j; ++jj) seen |= (ranks[jj] == r);
            ranks[j] = r;
            if (!seen) {
                atomicAdd(&h_r[r], 1);
                in_rank[t * R + r] = 1;
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < E; i += kThreads) ws_e[(int64_t)blockIdx.x * E + i] = h_e[i];
    for (int i = tid; i < R; i += kThreads) ws_r[(int64_t)blockIdx.x * R + i] = h_r[i];
    if (__syncthreads_or(bad) && tid == 0) report(status, kErrRange);
}

// Exclusive scan of v[0..n) in shared memory (n <= kMaxExperts), result in out[];
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

__global__ void __launch_bounds__(kThreads)
layout_assign_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap,
                     const int32_t *__restrict__ ws_e, const int32_t *__restrict__ ws_r,
                     int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                     int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                     int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src,
                     int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_assign[];
    int32_t *s_total = smem_assign;          // [E] copies per expert (all blocks)
    int32_t *s_off = s_total + E;            // [E] exclusive prefix of s_total
    int32_t *s_base = s_off + E;             // [E] first row of this block's copies
    int32_t *s_wc = s_base + E;              // [kWarps][E] per-warp counts, then bases
    int32_t *s_idx = s_wc + kWarps * E;      // [kTokensPerBlock * k]
    __shared__ int32_t s_scan[32];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = gridDim.x, b = blockIdx.x;
    const int64_t t0 = (int64_t)b * kTokensPerBlock;
    const int nt = tokens_in_block(n, t0);

    for (int i = tid; i < nt * k; i += kThreads) s_idx[i] = __ldg(idx + t0 * k + i);
    for (int e = tid; e < E; e += kThreads) {
        int32_t pre = 0, tot = 0;
        for (int bb = 0; bb < nb; ++bb) {
            const int32_t v = __ldg(ws_e + (int64_t)bb * E + e);
            tot += v;
            pre += bb < b ? v : 0;
        }
        s_total[e] = tot;
        s_base[e] = pre;
    }
    __syncthreads();
    const int32_t m_total = block_exclusive_scan(s_total, s_off, E, s_scan);
    for (int e = tid; e < E; e += kThreads) s_base[e] += cap > 0 ? e * cap : s_off[e];

    if (b == 0) {
        int32_t mx = 0;
        for (int e = tid; e < E; e += kThreads) {
            tokens_per_expert[e] = s_total[e];
            expert_offset[e] = s_off[e];
            mx = max(mx, s_total[e]);
        }
        if (tid == 0) expert_offset[E] = m_total;
        for (int r = tid; r < R; r += kThreads) {
            int32_t s = 0;
            for (int bb = 0; bb < nb; ++bb) s += __ldg(ws_r + (int64_t)bb * R + r);
            tokens_per_rank[r] = s;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if (lane == 0) s_scan[warp] = mx;
        __syncthreads();
        if (tid == 0) {
            int32_t m = 0;
            for (int w = 0; w < kWarps; ++w) m = max(m, s_scan[w]);
            *max_count = m;
        }
    }

    // receive rows that get no copy: recv_src = -1 (spread over all blocks)
    {
        const int64_t step = (int64_t)nb * kThreads;
        if (cap > 0) {
            const int64_t rows = (int64_t)E * cap;
            for (int64_t i = (int64_t)b * kThreads + tid; i < rows; i += step) {
                const int e = (int)(i / cap);
                if (i - (int64_t)e * cap >= s_total[e]) recv_src[i] = -1;
            }
        } else {
            for (int64_t i = m_total + (int64_t)b * kThreads + tid; i < n * k; i += step) recv_src[i] = -1;
        }
    }

    // pass A: per-warp counts over the warp's pairs, in order
    const int p_begin = warp * kTokensPerWarp * k;
    const int p_end = min(p_begin + kTokensPerWarp * k, nt * k);
    int32_t *wc = s_wc + warp * E;
    for (int e = lane; e < E; e += 32) wc[e] = 0;
    __syncwarp();
    for (int p0 = p_begin; p0 < p_end; p0 += 32) {
        const int p = p0 + lane;
        const int32_t e = p < p_end ? s_idx[p] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? e : -1);
        if (valid && lane == __ffs(peers) - 1) wc[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per expert: turn the warp counts into each warp's first row
    for (int e = tid; e < E; e += kThreads) {
        int32_t run = s_base[e];
        for (int w = 0; w < kWarps; ++w) {
            const int32_t c = s_wc[w * E + e];
            s_wc[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();

    // pass B: hand out rows in order
    bool over = false, bad_row = false;
    for (int p0 = p_begin; p0 < p_end; p0 += 32) {
        const int p = p0 + lane;
        const int32_t e = p < p_end ? s_idx[p] : -1;
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
    if (over) report(status, kErrCapacity);
    if (bad_row) report(status, kErrRange);
}

}  // namespace

size_t layout_workspace_bytes(int64_t n, int E, int R) { return ws_layout(n, E, R).bytes; }

size_t layout_assign_smem_bytes(int E, int k) {
    return (size_t)(3 * E + kWarps * E + kTokensPerBlock * k) * sizeof(int32_t);
}

cgl_status launch_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                         int32_t *tokens_per_expert, int32_t *tokens_per_rank, uint8_t *in_rank,
                         int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                         int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream) {
    const WsLayout w = ws_layout(n, E, R);
    int32_t *ws_e = static_cast<int32_t *>(ws);
    int32_t *ws_r = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.rank_off);
    const size_t smem1 = (size_t)(E + R) * sizeof(int32_t);
    const size_t smem2 = (size_t)(3 * E + kWarps * E + kTokensPerBlock * k) * sizeof(int32_t);
    if (smem2 > 48 * 1024) {
        if (!ensure_smem_attr((const void *)layout_assign_kernel, smem2)) return CGL_ECUDA;
    }
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;
    layout_count_kernel<<<(unsigned)w.blocks, kThreads, smem1, stream>>>(idx, n, k, E, R, ws_e, ws_r,
                                                                          in_rank, status);
    layout_assign_kernel<<<(unsigned)w.blocks, kThreads, smem2, stream>>>(
        idx, n, k, E, R, cap, ws_e, ws_r, tokens_per_expert, tokens_per_rank, expert_offset,
        max_count, dst_pos, recv_src, recv_rows, status);
    return cudaGetLastError() == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
