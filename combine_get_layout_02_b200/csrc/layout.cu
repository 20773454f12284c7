// Dispatch layout on the GPU: per-expert / per-rank counts, prefix sums and the
// stable receive row of every (token, slot) copy.
//
// The DeepEP pages describe dispatch only as routing each token to its gated
// experts, with the host waiting on GPU-made receive counts (brainleap "Day2
// DeepEP", section "All-to-All通信", the figure caption on the host waiting for
// the receive counts).  The order inside
// an expert is ascending token order: the result equals one sequential walk
// over t = 0..N-1, j = 0..k-1 that hands out the next free row of each expert.
//
// Work split.  Block b owns T consecutive tokens, T = min(64 CH, 256 CH / k),
// so at most 256 CH (token, slot) pairs, CH = 1, 2 or 4 chunks of 32 pairs per
// warp; pair p of the block (row-major (t, j) order) belongs to warp
// p / (32 CH), which walks its chunks in order.  The whole layout is latency
// bound: every phase is a few instructions per pair on one SM, so the pairs
// are spread over more blocks (smaller CH) until the grid reaches 64 blocks;
// past that the all-blocks read of the count table (blocks^2 (E + R) words
// through L2) costs more than the per-pair work it saves.
//
//   ranks in warp : per chunk, __match_any_sync groups the lanes that name
//                   one expert; a lane's rank is the warp's running count of
//                   that expert plus the lower lanes of its group, and the
//                   group's lowest lane advances the count (warp-private
//                   shared-memory counters, one per expert).  A token that
//                   names one expert twice needs no special case.  (On
//                   sm_100a match.any costs ~390 cycles of latency and ~56
//                   SM cycles of issue per warp: the main per-pair cost.)
//   block counts  : a per-expert pass over the 8 warps turns the warp counts
//                   into warp offsets and the block's count per expert.
//   rank sets     : per token, the set of ranks it reaches (slots of one
//                   token are adjacent lanes: a segmented shuffle-OR when k
//                   divides 32, shared-memory atomics otherwise); distinct
//                   tokens per rank come from ballots (idle warps split
//                   the ranks); the bitmasks are
//                   expanded to the block's is_token_in_rank bytes with
//                   coalesced 16-byte stores.
//   bases         : every block reads the workspace table of per-block counts
//                   column-wise (16-byte loads, rows split over thread groups)
//                   for the copies of each expert in earlier blocks and in
//                   total; an exclusive scan over experts gives expert_offset.
//                   Block 0 writes the global counts, offsets and max.
//   rows          : row = expert base + earlier blocks + warp offset + rank.
//
// Launch shapes.  Batches of 2 to 8 one-chunk blocks (up to 256 tokens at
// k = 8, e.g. 128 decode tokens as 4 CTAs) run as one thread-block cluster
// that exchanges counts through distributed shared memory (below).  With one
// block the block's own counts are the totals and nothing is exchanged.
// When every block fits on the GPU at once, one cooperative kernel does
// everything and the blocks exchange their counts through the workspace: each
// block writes its row, then release-stores this launch's 64-bit tag into its
// flag word, and waits, with a bounded spin (CGL_ETIMEOUT after ~1 s), until
// every flag shows that tag; one warp polls with relaxed loads and a single
// fence follows (an acquire load per poll would invalidate L1 every time).
// One exchange round only: on this part each dependent round trip through L2
// costs about a microsecond, more than the column sums it would save.  The
// tag's low half is a generation counter kept in the workspace, its high half
// a per-call value from the host with the top bit set (so no count word and no
// zeroed word ever equals a tag).  Every launch advances the generation by
// exactly one compare-and-swap from the value its blocks read, on success (block
// 0, after its wait) and on a timeout (every block that gave up), so no two
// launches on one workspace share a tag: not graph replays (same host value,
// new generation), and not a launch after one that timed out, whose published
// flags would otherwise match the next launch's tag before that launch's blocks
// had written their counts.  Otherwise two kernels run (counts, then bases +
// rows), the second with programmatic dependent launch; it recomputes the
// cheap in-warp ranks.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxPairs = 1024;                   // (token, slot) pairs per block
constexpr int kChunks = kMaxPairs / kThreads;     // 32-pair chunks per warp (4)
constexpr int kMaxTokensPerBlock = 256;
constexpr int kColUnroll = 16;                    // independent workspace loads per thread
constexpr int kPartWords = 2048;                  // column partial sums (per group and expert)
constexpr size_t kSmemDefault = 47 * 1024;        // dynamic bytes that need no opt-in (48 KiB
                                                  // minus room for static shared memory)
constexpr long long kWaitCycles = 1LL << 31;      // bound on the inter-block wait (~1 s)

// Tokens per block when each warp takes CH chunks of 32 pairs (CH = 1, 2, 4).
__host__ __device__ __forceinline__ int tokens_per_block(int k, int CH = kChunks) {
    const int t = (kThreads * CH) / k;
    const int cap = kMaxTokensPerBlock / kChunks * CH;
    return t < cap ? (t > 0 ? t : 1) : cap;
}

// Chunks per warp of the one-launch layout for n tokens: a single block when
// all pairs fit in one, else the smallest of 1, 2, 4 that keeps the grid at
// most kSpreadBlocks blocks (fewer pairs per SM, same number of exchange rows).
constexpr int kSpreadBlocks = 64;
__host__ __device__ __forceinline__ int layout_chunks(int64_t n, int k) {
    if (n <= tokens_per_block(k, kChunks)) return kChunks;
    for (int ch = 1; ch < kChunks; ch *= 2) {
        const int t = tokens_per_block(k, ch);
        if ((n + t - 1) / t <= kSpreadBlocks) return ch;
    }
    return kChunks;
}
__host__ __device__ __forceinline__ int mask_words(int R) { return (R + 31) >> 5; }

// Workspace: [generation: u64][flags: blocks x u64][pad to 256 B][expert counts: blocks x E][pad]
//            [rank counts: blocks x R]
struct WsLayout {
    int64_t blocks;
    size_t e_off, r_off, bytes;
};

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

WsLayout ws_layout_blocks(int64_t blocks, int E, int R) {
    WsLayout w;
    w.blocks = blocks;
    w.e_off = align256((size_t)(w.blocks + 1) * sizeof(uint64_t));
    w.r_off = w.e_off + align256((size_t)w.blocks * (size_t)E * sizeof(int32_t));
    w.bytes = w.r_off + (size_t)w.blocks * (size_t)R * sizeof(int32_t);
    return w;
}

WsLayout ws_layout(int64_t n, int k, int E, int R) {
    const int T = tokens_per_block(k, layout_chunks(n, k));
    return ws_layout_blocks(n > 0 ? (n + T - 1) / T : 1, E, R);
}

__device__ __forceinline__ void st_release_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// The tag of a launch: the host's per-call salt (top bit set) in the high
// half, generation g0 + 1 in the low half.  Count words (non-negative int32)
// never have the top bit of a high half set.
__device__ __forceinline__ uint64_t launch_tag(uint32_t salt, uint64_t g0) {
    return ((uint64_t)salt << 32) | ((g0 + 1) & 0xFFFFFFFFull);
}


// Barrier of the 256 layout threads (warps 0-7, hardware barrier 1).  In the
// 256-thread layout kernels that is the whole block; the fused layout +
// dispatch kernel runs other warps beside them, which never take part.
__device__ __forceinline__ void lsync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool lsync_or(bool v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, 1, 256, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((int)v) : "memory");
    return r != 0;
}

// Shared-memory add without a return value (red.shared): the pointer must point
// into shared memory; spelling out the state space keeps the compiler from a
// generic atomic, which is several times slower here.
__device__ __forceinline__ void red_shared_add(int32_t *p, int v) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(p)), "r"(v) : "memory");
}

// q = e / d for 0 <= e < 1024 and 1 <= d <= 1024 as (e * m) >> 20 with
// m = ceil(2^20 / d): exact on that range because e * (m * d - 2^20) < 2^20.
__device__ __forceinline__ uint32_t div_magic(int d) { return ((1u << 20) + (uint32_t)d - 1u) / (uint32_t)d; }
__device__ __forceinline__ int div_small(int e, uint32_t m) { return (int)(((uint32_t)e * m) >> 20); }

// Shared memory (32-bit words).  kind 0: fused kernel, 1: counts kernel, 2: rows kernel.
struct Smem {
    int32_t *wc;       // [kWarps][E] warp counts per expert, then warp offsets
    int32_t *he;       // [E] block count per expert
    uint32_t *mask;    // [T][mask_words(R)] rank set per token            (kinds 0, 1)
    int32_t *hr;       // [R] block count of distinct tokens per rank     (kinds 0, 1)
    int32_t *total;    // [E] count per expert over all blocks             (kinds 0, 2)
    int32_t *base;     // [E] first row of this block's copies per expert  (kinds 0, 2)
    int32_t *off;      // [E] exclusive prefix of total                    (kinds 0, 2)
    int32_t *part;     // [kPartWords] column partial sums                 (kinds 0, 2)
};

__host__ __device__ __forceinline__ size_t smem_words(int kind, int k, int E, int R) {
    size_t w = (size_t)kWarps * E + E;
    if (kind != 2) w += (size_t)tokens_per_block(k) * mask_words(R) + R;
    if (kind != 1) w += 3 * (size_t)E + kPartWords;
    return w;
}

__device__ Smem carve(int kind, int32_t *p, int k, int E, int R) {
    Smem s = {};
    s.wc = p; p += kWarps * E;
    s.he = p; p += E;
    if (kind != 2) {
        s.mask = reinterpret_cast<uint32_t *>(p); p += tokens_per_block(k) * mask_words(R);
        s.hr = p; p += R;
    }
    if (kind != 1) {
        s.total = p; p += E;
        s.base = p; p += E;
        s.off = p; p += E;
        s.part = p;
    }
    return s;
}

// Block-level view of one block's pairs; CH = 32-pair chunks per warp (a block
// holds up to 8 * 32 * CH pairs).
template <int CH>
struct PairsT {
    int64_t t0;      // first token of the block
    int nt;          // tokens in the block
    int np;          // pairs in the block (nt * k)
    int32_t e[CH];   // key of each of this thread's pairs (-1: no copy)
    int32_t rk[CH];  // rank among the warp's earlier pairs with that key
};
using Pairs = PairsT<kChunks>;

template <int CH = kChunks>
__device__ __forceinline__ int pair_of(int i) { return (threadIdx.x >> 5) * (CH * 32) + i * 32 + (threadIdx.x & 31); }

// Load this thread's ids (coalesced: each warp reads 32 consecutive ids per
// chunk) of block `token_block` (T tokens per block).  Nothing waits for the
// loads here: check_pairs is the first use.
template <int CH = kChunks>
__device__ __forceinline__ void load_pairs_only(const int32_t *__restrict__ idx, int64_t n, int k,
                                                int64_t token_block, int T, PairsT<CH> &P) {
    P.t0 = token_block * T;
    const int64_t rem = n - P.t0;
    P.nt = rem <= 0 ? 0 : (rem < T ? (int)rem : T);
    P.np = P.nt * k;
    const int32_t *src = idx + P.t0 * k;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int p = pair_of<CH>(i);
        P.e[i] = p < P.np ? __ldg(src + p) : -1;
    }
}

// Returns true if an id outside [-1, E_ids) was loaded; such slots make no copy.
template <int CH = kChunks>
__device__ __forceinline__ bool check_pairs(int E_ids, PairsT<CH> &P) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        if (P.e[i] < -1 || P.e[i] >= E_ids) { bad = true; P.e[i] = -1; }
    }
    return bad;
}

template <int CH = kChunks>
__device__ __forceinline__ bool load_pairs(const int32_t *__restrict__ idx, int64_t n, int k, int E_ids,
                                           int64_t token_block, int T, PairsT<CH> &P) {
    load_pairs_only<CH>(idx, n, k, token_block, T, P);
    return check_pairs<CH>(E_ids, P);
}

// Turn the loaded ids into keys and rank the keys within the warp.  Expert
// mode: key = expert id.  Rank mode (kRankKeys): key = the expert's rank
// e / key_div for the first slot of the token on that rank, else -1 (one copy
// per token and rank).  Keys index s.wc[.][0, nkeys).  s.wc must be zero.
template <bool kRankKeys, int CH = kChunks>
__device__ __forceinline__ void key_and_rank(const int32_t *__restrict__ idx, int k, int E_ids, int key_div,
                                             int nkeys, const Smem &s, PairsT<CH> &P) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lower = (1u << lane) - 1u;
    if (kRankKeys) {
        const uint32_t m = div_magic(key_div);
        if ((32 % k) == 0) {
            // a token's slots are adjacent lanes of one chunk: the first slot on a
            // rank is the lowest lane of its (token, rank) group
            const int tshift = __ffs(k) - 1;
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int32_t e = P.e[i];
                const int r = e >= 0 ? div_small(e, m) : 0;
                const int key = e >= 0 ? (((lane >> tshift) << 11) | r) : (int)(0x80000000u | (uint32_t)lane);
                const unsigned grp = __match_any_sync(0xFFFFFFFFu, key);
                P.e[i] = (e >= 0 && (grp & lower) == 0) ? r : -1;
            }
        } else {
            const int32_t *src = idx + P.t0 * k;
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int32_t e = P.e[i];
                if (e < 0) continue;
                const int p = pair_of<CH>(i);
                const int tl = p / k, j = p - tl * k;
                const int r = div_small(e, m);
                bool first = true;
                for (int jj = 0; jj < j; ++jj) {
                    const int32_t e2 = __ldg(src + tl * k + jj);
                    if (e2 >= 0 && e2 < E_ids && div_small(e2, m) == r) first = false;
                }
                P.e[i] = first ? r : -1;
            }
        }
    }
    // the matches of all chunks first (independent, so their latencies overlap),
    // then the chain through the warp's counters
    unsigned grp[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) grp[i] = __match_any_sync(0xFFFFFFFFu, P.e[i]);
    int32_t *wc = s.wc + warp * nkeys;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int32_t e = P.e[i];
        const unsigned peers = grp[i];
        const int32_t before = e >= 0 ? wc[e] : 0;
        __syncwarp();
        if (e >= 0 && (peers & lower) == 0) wc[e] = before + __popc(peers);
        __syncwarp();
        P.rk[i] = before + __popc(peers & lower);
    }
}

template <bool kRankKeys, int CH = kChunks>
__device__ bool load_and_rank(const int32_t *__restrict__ idx, int64_t n, int k, int E_ids, int key_div,
                              int nkeys, int64_t token_block, int T, const Smem &s, PairsT<CH> &P) {
    const bool bad = load_pairs<CH>(idx, n, k, E_ids, token_block, T, P);
    key_and_rank<kRankKeys, CH>(idx, k, E_ids, key_div, nkeys, s, P);
    return bad;
}

// Warp counts -> warp offsets (in place) and block counts per expert.  Needs a barrier before.
template <int NT = kThreads>
__device__ void warp_offsets(int E, const Smem &s) {
    for (int e = threadIdx.x; e < E; e += NT) {
        int32_t run = 0;
#pragma unroll
        for (int w = 0; w < (NT / 32); ++w) {
            const int32_t c = s.wc[w * E + e];
            s.wc[w * E + e] = run;
            run += c;
        }
        s.he[e] = run;
    }
}

// Rank sets of the block's tokens into s.mask (zeroed before).
template <int CH = kChunks>
__device__ void rank_sets(int k, int E, int R, const Smem &s, const PairsT<CH> &P) {
    const int lane = threadIdx.x & 31;
    const uint32_t pm = div_magic(E / R);
    const int rw = mask_words(R);
    if ((32 % k) == 0 && R <= 64) {
        // the k slots of a token are k adjacent lanes of one chunk
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int32_t e = P.e[i];
            uint64_t m = e >= 0 ? (1ull << div_small(e, pm)) : 0ull;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1)
                if (o < k) m |= __shfl_xor_sync(0xFFFFFFFFu, m, o);
            const int p = pair_of<CH>(i);
            if (p < P.np && (lane % k) == 0) {
                const int tl = p / k;
                s.mask[tl * rw] = (uint32_t)m;
                if (rw > 1) s.mask[tl * rw + 1] = (uint32_t)(m >> 32);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int32_t e = P.e[i];
            if (e < 0) continue;
            const int r = div_small(e, pm);
            atomicOr(&s.mask[(pair_of<CH>(i) / k) * rw + (r >> 5)], 1u << (r & 31));
        }
    }
}

// Distinct tokens per rank of the block into s.hr (zeroed before).  Needs a
// barrier before.  R <= 64: one ballot per (32-token group, rank); when there
// are more warps than token groups, the spare warps split the ranks.
template <int CH = kChunks, int NT = kThreads>
__device__ void rank_counts(int k, int R, const Smem &s, const PairsT<CH> &P) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rw = mask_words(R);
    if (R <= 64) {
        constexpr int kW = NT / 32;
        const int ngroups = (P.nt + 31) >> 5;
        if (ngroups == 0) return;
        const int slices = ngroups >= kW ? 1 : kW / ngroups;
        const int slice = warp / (ngroups >= kW ? kW : ngroups);
        if (slice >= slices) return;
        const int r0 = R * slice / slices, r1 = R * (slice + 1) / slices;
        const int g0 = ngroups >= kW ? warp : warp % ngroups;
        const int gstep = ngroups >= kW ? kW : ngroups;
        for (int g = g0; g < ngroups; g += gstep) {
            const int tl = g * 32 + lane;
            uint64_t m = 0;
            if (tl < P.nt) {
                m = s.mask[tl * rw];
                if (rw > 1) m |= (uint64_t)s.mask[tl * rw + 1] << 32;
            }
            int32_t c0 = 0, c1 = 0;
#pragma unroll 4
            for (int r = r0; r < r1; ++r) {
                const int c = __popc(__ballot_sync(0xFFFFFFFFu, (m >> r) & 1ull));
                if (r == lane) c0 = c;
                if (r == lane + 32) c1 = c;
            }
            if (c0) atomicAdd(&s.hr[lane], c0);
            if (c1) atomicAdd(&s.hr[lane + 32], c1);
        }
    } else {
        for (int r = threadIdx.x; r < R; r += NT) {
            int32_t c = 0;
            for (int tl = 0; tl < P.nt; ++tl) c += (s.mask[tl * rw + (r >> 5)] >> (r & 31)) & 1u;
            s.hr[r] = c;
        }
    }
}

// is_token_in_rank rows of the block (contiguous; 16-byte aligned when R % 16 == 0).
template <int CH = kChunks, int NT = kThreads>
__device__ void write_rank_rows(int R, uint8_t *__restrict__ in_rank, const Smem &s, const PairsT<CH> &P) {
    const int rw = mask_words(R);
    uint8_t *row0 = in_rank + P.t0 * R;
    const int nbytes = P.nt * R;
    if ((R & 15) == 0) {
        for (int q = threadIdx.x * 16; q < nbytes; q += NT * 16) {
            const int tl = q / R, r0 = q - tl * R;
            const uint32_t bits = (s.mask[tl * rw + (r0 >> 5)] >> (r0 & 31)) & 0xFFFFu;
            uint32_t wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = (((bits >> (4 * j)) & 0xFu) * 0x00204081u) & 0x01010101u;
            *reinterpret_cast<uint4 *>(row0 + q) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    } else {
        for (int q = threadIdx.x; q < nbytes; q += NT) {
            const int tl = q / R, r = q - tl * R;
            row0[q] = (uint8_t)((s.mask[tl * rw + (r >> 5)] >> (r & 31)) & 1u);
        }
    }
}

template <bool kCoherent>
__device__ __forceinline__ int4 ld_col4(const int32_t *p) {
    const int4 *q = reinterpret_cast<const int4 *>(p);
    return kCoherent ? __ldcg(q) : __ldg(q);
}
template <bool kCoherent>
__device__ __forceinline__ int32_t ld_col1(const int32_t *p) {
    return kCoherent ? __ldcg(p) : __ldg(p);
}

// Column sums of a [nb][ncols] table: out_tot[c] over all rows, out_pre[c] over
// rows < upto (out_pre may be null).  16-byte loads when ncols % 4 == 0; when a
// row needs fewer loads than there are threads, G thread groups split the
// rows and their partial sums meet in `part`.  kCoherent: the table was
// written by other blocks of the running grid (read through L2 only).
template <bool kCoherent, int U = kColUnroll>
__device__ void column_sums(const int32_t *t, int nb, int ncols, int upto, int32_t *out_tot,
                            int32_t *out_pre, int32_t *part) {
    const int tid = threadIdx.x;
    const int width = (ncols & 3) == 0 ? 4 : 1;    // columns per load
    const int nq = ncols / width;                    // loads per row
    int G = nq >= kThreads ? 1 : kThreads / nq;
    if (2 * G * ncols > kPartWords) G = kPartWords / (2 * ncols);
    if (G < 1) G = 1;
    const int q0 = G > 1 ? tid % nq : tid;
    const int g = G > 1 ? tid / nq : 0;
    const int qstep = G > 1 ? nq : kThreads;
    if (g < G) {
        for (int q = q0; q < nq; q += qstep) {
            int32_t tot[4] = {0, 0, 0, 0}, pre[4] = {0, 0, 0, 0};
            for (int r0 = g; r0 < nb; r0 += G * U) {
                int4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int r = r0 + u * G;
                    const int32_t *a = t + (int64_t)r * ncols + q * width;
                    if (r >= nb) v[u] = make_int4(0, 0, 0, 0);
                    else if (width == 4) v[u] = ld_col4<kCoherent>(a);
                    else v[u] = make_int4(ld_col1<kCoherent>(a), 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int32_t below = r0 + u * G < upto ? 1 : 0;
                    tot[0] += v[u].x; tot[1] += v[u].y; tot[2] += v[u].z; tot[3] += v[u].w;
                    pre[0] += below * v[u].x; pre[1] += below * v[u].y;
                    pre[2] += below * v[u].z; pre[3] += below * v[u].w;
                }
            }
            for (int c = 0; c < width; ++c) {
                const int col = q * width + c;
                if (G > 1) {
                    part[g * ncols + col] = tot[c];
                    part[(G + g) * ncols + col] = pre[c];
                } else {
                    out_tot[col] = tot[c];
                    if (out_pre) out_pre[col] = pre[c];
                }
            }
        }
    }
    if (G > 1) {
        lsync();
        for (int col = tid; col < ncols; col += kThreads) {
            int32_t a = 0, b = 0;
            for (int gg = 0; gg < G; ++gg) {
                a += part[gg * ncols + col];
                b += part[(G + gg) * ncols + col];
            }
            out_tot[col] = a;
            if (out_pre) out_pre[col] = b;
        }
    }
    lsync();
}

// Exclusive scan of v[0..n) in shared memory (n <= kMaxExperts) into out[];
// returns the total.  All threads of the block must call it.
template <int NT = kThreads>
__device__ int32_t block_exclusive_scan(const int32_t *v, int32_t *out, int n, int32_t *warp_sums) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + NT - 1) / NT;   // <= 4
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
    lsync();
    if (warp == 0) {
        int32_t s = lane < (NT / 32) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xFFFFFFFFu, s, o);
            if (lane >= o) s += u;
        }
        if (lane < (NT / 32)) warp_sums[lane] = s;   // inclusive over warps
    }
    lsync();
    int32_t run = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - local;
    for (int i = i0; i < i1; ++i) {
        out[i] = run;
        run += v[i];
    }
    const int32_t total = warp_sums[(NT / 32) - 1];
    lsync();
    return total;
}

// Bases, the global outputs (block 0) and the rows of the block's pairs.
// kTotalsGiven: s.total / s.base (copies in earlier blocks) are already set.
template <bool kCoherent, bool kRankKeys, int CH = kChunks, bool kTotalsGiven = false, int NT = kThreads,
          int U = kColUnroll>
__device__ void bases_and_rows(const int32_t *ws_e, const int32_t *ws_r, int64_t n, int k, int E, int R,
                               int cap, int64_t recv_rows, int32_t *__restrict__ tokens_per_expert,
                               int32_t *__restrict__ tokens_per_rank, int32_t *__restrict__ expert_offset,
                               int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                               int32_t *__restrict__ recv_src, uint32_t *status, const Smem &s,
                               const PairsT<CH> &P, int32_t *scan_tmp, int32_t *s_dst = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = gridDim.x, b = blockIdx.x;
    // tokens_per_rank from the table (unless this is the only block and it has
    // its own counts): rank column r is summed by warp (r / nb) % 8 of block
    // r % nb.  The loads of a warp's first column are issued before the expert
    // column sums and added after them, so both wait out the same round trip.
    const bool rank_sums = !kTotalsGiven && tokens_per_rank != nullptr && !(nb == 1 && s.hr != nullptr);
    const int rcol = b + warp * nb;
    int32_t rv[4] = {0, 0, 0, 0};
    if (rank_sums && rcol < R) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = lane + 32 * q;
            if (i < nb) rv[q] = ld_col1<kCoherent>(ws_r + (int64_t)i * R + rcol);
        }
        for (int i = lane + 128; i < nb; i += 32) rv[0] += ld_col1<kCoherent>(ws_r + (int64_t)i * R + rcol);
    }
    if constexpr (kTotalsGiven) {
    } else if (nb == 1) {   // one block: its own counts are the totals
        for (int e = tid; e < E; e += NT) {
            s.total[e] = s.he[e];
            s.base[e] = 0;
        }
        lsync();
    } else {
        column_sums<kCoherent, U>(ws_e, nb, E, b, s.total, s.base, s.part);
    }
    if (rank_sums) {
        for (int r = rcol; r < R; r += nb * (NT / 32)) {   // warp-uniform
            int32_t v = 0;
            if (r == rcol) {
                v = rv[0] + rv[1] + rv[2] + rv[3];
            } else {
                for (int i = lane; i < nb; i += 32) v += ld_col1<kCoherent>(ws_r + (int64_t)i * R + r);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            if (lane == 0) tokens_per_rank[r] = v;
        }
    }
    const int32_t m_total = block_exclusive_scan<NT>(s.total, s.off, E, scan_tmp);
    for (int e = tid; e < E; e += NT) s.base[e] += cap > 0 ? e * cap : s.off[e];

    if (b == 0) {
        int32_t mx = 0;
        for (int e = tid; e < E; e += NT) {
            tokens_per_expert[e] = s.total[e];
            expert_offset[e] = s.off[e];
            mx = max(mx, s.total[e]);
        }
        if (tid == 0) expert_offset[E] = m_total;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if (lane == 0) scan_tmp[warp] = mx;
        lsync();
        if (tid == 0) {
            int32_t m = 0;
            for (int w = 0; w < (NT / 32); ++w) m = max(m, scan_tmp[w]);
            *max_count = m;
        }
        // tokens_per_rank of a single block: its own distinct-token counts
        if constexpr (!kTotalsGiven) {
            if (tokens_per_rank != nullptr && nb == 1 && s.hr != nullptr)
                for (int r = tid; r < R; r += NT) tokens_per_rank[r] = s.hr[r];
        }
    }

    const int64_t step = (int64_t)nb * NT;
    if (cap > 0) {
        const int64_t rows = (int64_t)E * cap;
        for (int64_t i = (int64_t)b * NT + tid; i < rows; i += step) {
            const int e = (int)(i / cap);
            if (i - (int64_t)e * cap >= s.total[e]) recv_src[i] = -1;
        }
    } else {
        for (int64_t i = m_total + (int64_t)b * NT + tid; i < n * k; i += step) recv_src[i] = -1;
    }
    lsync();

    bool over = false, bad_row = false;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int p = pair_of<CH>(i);
        if (p >= P.np) continue;
        const int32_t e = P.e[i];
        int32_t d = -1;
        if (e >= 0) {
            const int32_t pos = s.base[e] + s.wc[warp * E + e] + P.rk[i];
            if (cap > 0 && pos - e * cap >= cap) over = true;
            else if (pos >= recv_rows) bad_row = true;
            else d = pos;
        }
        const int64_t q = P.t0 * k + p;
        dst_pos[q] = d;
        if (s_dst) s_dst[p] = d;
        // expert mode: the row's source slot t*k + j; rank mode: its source token t
        if (d >= 0) recv_src[d] = kRankKeys ? (int32_t)(P.t0 + p / k) : (int32_t)q;
    }
    if (over) report(status, kErrCapacity);
    if (bad_row) report(status, kErrRange);
}

// Wait until flags[0..nb) all hold `tag`, for at most kWaitCycles (~1 s).
// Warp 0 polls: each round, lane l reads flags l, l + 32, ... with relaxed
// loads (one L2 read each, no L1 invalidation, all in flight together) until
// every lane has seen its flags; then a gpu-scope fence makes the other
// blocks' earlier writes visible, and the block barrier hands that on to the
// whole block.  On the way out the launch's generation advances from g0 (the
// value this block read at its start) to g0 + 1 by compare-and-swap: block 0
// does it after a successful wait (every block has read the generation by
// then, since every flag is published), and every block that gave up does it
// too, so a timed-out launch also leaves the next launch a new tag.  The first
// swap wins; later ones find the word changed and do nothing.  Returns true
// for the whole block when every flag was seen; otherwise reports
// CGL_ETIMEOUT and returns false for the whole block.  All threads of the
// block must call it.
__device__ bool wait_for_flags(uint64_t *gen, uint64_t g0, const uint64_t *flags, int nb, uint64_t tag,
                               uint32_t *status) {
    bool timed_out = false;
    if (threadIdx.x < 32) {
        const long long start = clock64();
        for (;;) {
            bool seen = true;
            for (int bb = threadIdx.x; bb < nb; bb += 32) seen &= ld_relaxed_u64(flags + bb) == tag;
            if (__all_sync(0xFFFFFFFFu, seen)) break;
            if (__any_sync(0xFFFFFFFFu, clock64() - start > kWaitCycles)) { timed_out = true; break; }
        }
        __threadfence();
    }
    const bool failed = lsync_or(timed_out);
    if (threadIdx.x == 0 && (failed || blockIdx.x == 0))
        atomicCAS(reinterpret_cast<unsigned long long *>(gen), (unsigned long long)g0,
                  (unsigned long long)(g0 + 1));
    if (failed) {
        if (threadIdx.x == 0) report(status, 1u << CGL_ETIMEOUT);
        return false;
    }
    return true;
}

// Self-test of the bounded wait: one block takes `ws` as a layout workspace
// header (word 0 the generation, then nflags flags) and waits for the tag of
// salt 0, which no layout launch uses (their salts have the top bit set), so
// on zeroed or layout-written flags it must give up after ~1 s, report
// CGL_ETIMEOUT and advance the generation, exactly as a layout block that
// timed out does.
__global__ void __launch_bounds__(kThreads) wait_probe_kernel(uint64_t *ws, int nflags, uint32_t *status) {
    const uint64_t g0 = ld_relaxed_u64(ws);
    wait_for_flags(ws, g0, ws + 1, nflags, launch_tag(0u, g0), status);
}

template <int NT = kThreads>
__device__ void zero_words(int32_t *p, int n) {
    for (int i = threadIdx.x; i < n; i += NT) p[i] = 0;
}

// ------------------------------------------------------------------ kernels

// One layout block's whole part of the one-launch layout, run by the 256
// threads of warps 0-7 (every barrier in it is lsync): block b = blockIdx.x of
// gridDim.x owns tokens [b T, b T + T).  E = number of keys (experts, or ranks
// in rank mode), E_ids / key_div = valid id range and expert-to-rank divisor
// for the key transform; in_rank == nullptr skips the rank sets (rank mode).
// s_dst (optional, shared memory, T k words) also receives the block's rows.
// Returns false (the whole group of 256) when the inter-block wait timed out.
template <bool kRankKeys, int CH, int U = kColUnroll>
__device__ bool layout_block(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int E_ids,
                             int key_div, int T, uint64_t *flags, uint32_t salt, int32_t *ws_e, int32_t *ws_r,
                             int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                             uint8_t *__restrict__ in_rank, int32_t *__restrict__ expert_offset,
                             int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                             int32_t *__restrict__ recv_src, int64_t recv_rows, uint32_t *status,
                             const Smem &s, int32_t *scan_tmp, int32_t *s_dst) {
    const int tid = threadIdx.x;
    const int nb = gridDim.x, b = blockIdx.x;
    const bool with_ranks = in_rank != nullptr;

    // This launch's tag: the host's salt and generation + 1.  Every block reads
    // the generation before it publishes its flag, and it advances only when a
    // block leaves the wait (wait_for_flags), so all blocks of a launch agree and
    // the next launch (a graph replay too, or one after a timeout) gets a new tag.
    uint64_t *gen = flags;
    flags += 1;
    const uint64_t g0 = ld_relaxed_u64(gen);
    const uint64_t tag = launch_tag(salt, g0);
    PairsT<CH> P;
    const bool bad = load_pairs<CH>(idx, n, k, E_ids, b, T, P);   // in flight while zeroing
    zero_words(s.wc, kWarps * E);
    zero_words(reinterpret_cast<int32_t *>(s.mask), T * mask_words(R));
    zero_words(s.hr, R);
    lsync();
    key_and_rank<kRankKeys, CH>(idx, k, E_ids, key_div, E, s, P);
    if (with_ranks) rank_sets<CH>(k, E, R, s, P);
    lsync();
    warp_offsets(E, s);
    if (with_ranks) rank_counts<CH>(k, R, s, P);
    lsync();
    if (nb == 1) {   // nothing to exchange
        if (with_ranks) write_rank_rows<CH>(R, in_rank, s, P);
        if (lsync_or(bad) && tid == 0) report(status, kErrRange);
        bases_and_rows<true, kRankKeys, CH, false, kThreads, U>(ws_e, ws_r, n, k, E, R, cap, recv_rows,
                                                                tokens_per_expert, tokens_per_rank, expert_offset,
                                                                max_count, dst_pos, recv_src, status, s, P,
                                                                scan_tmp, s_dst);
        return true;
    }
    for (int i = tid; i < E; i += kThreads) ws_e[(int64_t)b * E + i] = s.he[i];
    for (int i = tid; i < R; i += kThreads) ws_r[(int64_t)b * R + i] = s.hr[i];
    const bool any_bad = lsync_or(bad);   // also orders the workspace writes before the flag
    if (tid == 0) {
        __threadfence();
        st_release_u64(flags + b, tag);
        if (any_bad) report(status, kErrRange);
    }
    // no other block reads these rows: written after the flag, so the fence above
    // does not wait for them
    if (with_ranks) write_rank_rows<CH>(R, in_rank, s, P);

    // every block's counts must be visible before the bases
    if (!wait_for_flags(gen, g0, flags, nb, tag, status)) return false;

    bases_and_rows<true, kRankKeys, CH, false, kThreads, U>(ws_e, ws_r, n, k, E, R, cap, recv_rows,
                                                            tokens_per_expert, tokens_per_rank, expert_offset,
                                                            max_count, dst_pos, recv_src, status, s, P, scan_tmp,
                                                            s_dst);
    return true;
}

template <bool kRankKeys, int CH>
__global__ void __launch_bounds__(kThreads)
layout_fused_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int E_ids,
                    int key_div, uint64_t *flags, uint32_t salt, int32_t *ws_e, int32_t *ws_r,
                    int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                    uint8_t *__restrict__ in_rank, int32_t *__restrict__ expert_offset,
                    int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                    int32_t *__restrict__ recv_src, int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_fused[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve(0, smem_fused, k, E, R);
    layout_block<kRankKeys, CH>(idx, n, k, E, R, cap, E_ids, key_div, tokens_per_block(k, CH), flags, salt, ws_e, ws_r,
                                tokens_per_expert, tokens_per_rank, in_rank, expert_offset, max_count, dst_pos,
                                recv_src, recv_rows, status, s, scan_tmp, nullptr);
}

template <bool kRankKeys, int CH>
__global__ void __launch_bounds__(kThreads)
layout_count_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int E_ids, int key_div,
                    int32_t *__restrict__ ws_e, int32_t *__restrict__ ws_r,
                    uint8_t *__restrict__ in_rank, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_count[];
    const Smem s = carve(1, smem_count, k, E, R);
    const int tid = threadIdx.x;
    const bool with_ranks = in_rank != nullptr;
    zero_words(s.wc, kWarps * E);
    zero_words(reinterpret_cast<int32_t *>(s.mask), tokens_per_block(k, CH) * mask_words(R));
    zero_words(s.hr, R);
    __syncthreads();
    PairsT<CH> P;
    const bool bad =
        load_and_rank<kRankKeys, CH>(idx, n, k, E_ids, key_div, E, blockIdx.x, tokens_per_block(k, CH), s, P);
    if (with_ranks) rank_sets<CH>(k, E, R, s, P);
    __syncthreads();
    warp_offsets(E, s);
    if (with_ranks) {
        rank_counts<CH>(k, R, s, P);
        write_rank_rows<CH>(R, in_rank, s, P);
    }
    __syncthreads();
    for (int i = tid; i < E; i += kThreads) ws_e[(int64_t)blockIdx.x * E + i] = s.he[i];
    for (int i = tid; i < R; i += kThreads) ws_r[(int64_t)blockIdx.x * R + i] = s.hr[i];
    if (__syncthreads_or(bad) && tid == 0) report(status, kErrRange);
}

template <bool kRankKeys, int CH>
__global__ void __launch_bounds__(kThreads)
layout_rows_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int E_ids,
                   int key_div, const int32_t *__restrict__ ws_e, const int32_t *__restrict__ ws_r,
                   int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                   int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                   int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                   uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_rows[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve(2, smem_rows, k, E, R);
    zero_words(s.wc, kWarps * E);
    __syncthreads();
    // topk_idx is not written by the counts kernel, which started only after
    // everything before it in the stream had finished: it may be read before the wait
    PairsT<CH> P;
    load_and_rank<kRankKeys, CH>(idx, n, k, E_ids, key_div, E, blockIdx.x, tokens_per_block(k, CH), s, P);
    __syncthreads();
    warp_offsets(E, s);
    griddep_wait();
    __syncthreads();
    bases_and_rows<false, kRankKeys, CH>(ws_e, ws_r, n, k, E, R, cap, recv_rows, tokens_per_expert,
                                     tokens_per_rank, expert_offset, max_count, dst_pos, recv_src, status,
                                     s, P, scan_tmp);
}

// ---------------------------------------------------------- cluster layout
//
// Small batches (2 to 8 blocks of one chunk per warp: up to 256 tokens at
// top-8): the blocks run as one thread-block cluster and exchange their
// counts through distributed shared memory instead of the workspace.  After a
// hardware cluster barrier every CTA reads the other CTAs' per-key counts
// (mapa + ld.shared::cluster) for its prefix over earlier CTAs and the
// totals; CTA 0 also sums the distinct-token counts per rank.  A CTA arrives
// at a second cluster barrier once its peer reads are done and waits on it
// only before it exits, so no CTA's shared memory goes away while a peer may
// still read it.  No global round trip between the phases.

constexpr int kMaxClusterCtas = 8;   // portable cluster size

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The int32 at the same shared-memory offset as `local` in cluster CTA `rank`.
__device__ __forceinline__ int32_t ld_cluster_peer(const int32_t *local, uint32_t rank) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(local);
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    int32_t v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
    return v;
}

// Grid = exactly one cluster of C = gridDim.x CTAs (cluster rank = blockIdx.x);
// CTA b owns tokens [b T, b T + T), T = tokens_per_block(k, 1).
template <bool kRankKeys>
__global__ void __launch_bounds__(kThreads)
layout_cluster_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int E_ids,
                      int key_div, int32_t *__restrict__ tokens_per_key, int32_t *__restrict__ tokens_per_rank,
                      uint8_t *__restrict__ in_rank, int32_t *__restrict__ key_offset,
                      int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                      int32_t *__restrict__ recv_src, int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_cl[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve(0, smem_cl, k, E, R);
    const int tid = threadIdx.x;
    const int C = gridDim.x, b = blockIdx.x;
    const int T = tokens_per_block(k, 1);
    const bool with_ranks = in_rank != nullptr;
    PairsT<1> P;
    const bool bad = load_pairs<1>(idx, n, k, E_ids, b, T, P);   // in flight while zeroing
    zero_words(s.wc, kWarps * E);
    zero_words(reinterpret_cast<int32_t *>(s.mask), T * mask_words(R));
    zero_words(s.hr, R);
    lsync();
    key_and_rank<kRankKeys, 1>(idx, k, E_ids, key_div, E, s, P);
    if (with_ranks) rank_sets<1>(k, E, R, s, P);
    lsync();
    warp_offsets(E, s);
    if (with_ranks) rank_counts<1>(k, R, s, P);
    if (bad) report(status, kErrRange);
    cluster_arrive_release();   // this CTA's counts are final; its rank rows go out while peers catch up
    if (with_ranks) write_rank_rows<1>(R, in_rank, s, P);
    cluster_wait_acquire();     // every CTA's counts are visible cluster-wide
    for (int e = tid; e < E; e += kThreads) {
        int32_t tot = 0, pre = 0;
#pragma unroll
        for (int c = 0; c < kMaxClusterCtas; ++c) {
            if (c < C) {
                const int32_t v = ld_cluster_peer(s.he + e, (uint32_t)c);
                tot += v;
                pre += c < b ? v : 0;
            }
        }
        s.total[e] = tot;
        s.base[e] = pre;
    }
    if (b == 0 && with_ranks && tokens_per_rank != nullptr) {
        for (int r = tid; r < R; r += kThreads) {
            int32_t tot = 0;
#pragma unroll
            for (int c = 0; c < kMaxClusterCtas; ++c)
                if (c < C) tot += ld_cluster_peer(s.hr + r, (uint32_t)c);
            tokens_per_rank[r] = tot;
        }
    }
    cluster_arrive_release();   // this CTA reads no peer shared memory after this point
    lsync();
    bases_and_rows<true, kRankKeys, 1, true>(nullptr, nullptr, n, k, E, R, cap, recv_rows, tokens_per_key,
                                             nullptr, key_offset, max_count, dst_pos, recv_src, status, s, P,
                                             scan_tmp);
    cluster_wait_acquire();     // the peers have finished reading this CTA's shared memory
}

// ------------------------------------------------- replicated-count layout
//
// Batches up to a few thousand tokens: no exchange between blocks at all.
// Block b of G owns tokens [b T, b T + T) as above, and learns the global
// counts by reading every id of the batch itself (N k ids, from L2 after the
// first block has read them: 128 KiB at 4096 tokens, top-8) into two
// shared-memory histograms with shared atomics, one per id: copies in tokens
// before its own (before[e]) and the rest (rest[e]).  total = before + rest
// gives the expert offsets by one scan over E; a copy's row is expert base +
// before[e] + the block's own in-order rank (warp offsets + in-warp rank, as
// above).  The same pass counts distinct tokens for the block's designated
// ranks r = b, b + G, ... (at most 32 of them; one ballot per rank per 32
// tokens).  The redundant reads cost every block the same ~N k atomics, which
// is why it is kept to small and medium batches; in exchange nothing waits on
// another block, so no cooperative launch, no workspace and no bounded wait.

// Measured on B200 (graph of 20 back-to-back layouts, E = 256, R = 64, top-8):
// 1024 / 2048 / 4096 tokens take 6.7 / 7.5 / 9.9 us this way against
// 8.8 / 9.5 / 10.2 us with the exchange; at 6144 tokens the blocks no longer
// fit on the GPU at once and it loses (18.9 against 12.1).  Batches of at
// most one token per SM take the one-CTA-per-token kernel instead.
#ifndef CGL_REP_MAX_PAIRS
#define CGL_REP_MAX_PAIRS 32768
#endif
constexpr int64_t kRepMaxPairs = CGL_REP_MAX_PAIRS;   // (token, slot) pairs of the batch
constexpr int64_t kRepWidePairs = 4096;   // above this, standalone blocks scan with kRepThreads threads

// Shared memory of a replicated-count layout block with T tokens (words):
// warp counts [8][E], block counts [E], rank sets [T][mask_words(R)], own
// rank counts [R], total (rest) [E], before / base [E], offsets [E], and 32
// designated-rank counts.
__host__ __device__ __forceinline__ size_t rep_smem_words(int T, int E, int R) {
    return (size_t)kWarps * E + E + (size_t)T * mask_words(R) + R + 3 * (size_t)E + 32;
}

__device__ Smem carve_rep(int32_t *p, int T, int E, int R) {
    Smem s = {};
    s.wc = p; p += kWarps * E;
    s.he = p; p += E;
    s.mask = reinterpret_cast<uint32_t *>(p); p += T * mask_words(R);
    s.hr = p; p += R;
    s.total = p; p += E;
    s.base = p; p += E;
    s.off = p; p += E;
    s.part = p;   // 32 designated-rank counts
    return s;
}

// Designated ranks of block b of G: b + i G for i < rep_designated(b, G, R).
__host__ __device__ __forceinline__ int rep_designated(int b, int G, int R) {
    return b < R ? (R - 1 - b) / G + 1 : 0;
}

// Ask the TMA engine to bring the ids of the block's tokens [t0, t0 + T) into
// L2 (one thread).  Every block reads every id in its scan; with each block
// fetching its own share first, those reads hit L2 instead of queueing in HBM
// behind the block's other traffic.  kVec-aligned ids only (16-byte aligned,
// k % 4 == 0), so the range is 16-byte aligned and sized.
__device__ __forceinline__ void prefetch_own_ids(const int32_t *idx, int64_t n, int k, int64_t t0, int T,
                                                 bool vec) {
    const int64_t nt = t0 < n ? (n - t0 < T ? n - t0 : T) : 0;
    if (vec && threadIdx.x == 0 && nt > 0) prefetch_l2_bulk(idx + t0 * k, (uint32_t)(nt * k * 4));
}

// Every id of the batch into before[] (tokens < t0) / rest[] (tokens >= t0),
// and distinct tokens of the designated ranks b + i G (i < nd <= 32) into
// dcnt[i].  Warp-uniform loop over groups of 32 tokens, one token per lane;
// the ids of U groups are loaded before any of them is counted.  KM >= k ids
// per token are held in registers; kVec: k % 4 == 0 and idx 16-byte aligned
// (int4 loads).  All 256 layout threads call it.
template <bool kVec, int KM, int NT>
__device__ void rep_scan_ids(const int32_t *__restrict__ idx, int64_t n, int k, int E, int64_t t0,
                             int32_t *before, int32_t *rest, uint32_t rank_magic, int b, int G, int nd,
                             int32_t *dcnt) {
    constexpr int U = KM <= 8 ? 2 : 1;   // token groups in flight per warp
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t gmag = div_magic(G);
    int32_t dc = 0;   // lane i < nd: this warp's count for designated rank i
    for (int64_t g0 = (int64_t)warp * 32; g0 < n; g0 += (int64_t)NT * U) {
        int32_t ids[U][KM];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = g0 + (int64_t)u * NT + lane;
            const int32_t *src = idx + t * k;
            if (kVec) {
#pragma unroll
                for (int q = 0; q < KM / 4; ++q) {
                    int4 v = make_int4(-1, -1, -1, -1);
                    if (t < n && q * 4 < k) v = __ldg(reinterpret_cast<const int4 *>(src) + q);
                    ids[u][4 * q] = v.x; ids[u][4 * q + 1] = v.y; ids[u][4 * q + 2] = v.z; ids[u][4 * q + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < KM; ++j) ids[u][j] = (t < n && j < k) ? __ldg(src + j) : -1;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = g0 + (int64_t)u * NT + lane;
            int32_t *cnt = t < t0 ? before : rest;
            uint32_t hits = 0;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                const int32_t e = ids[u][j];
                if (j < k && (uint32_t)e < (uint32_t)E) {
                    red_shared_add(cnt + e, 1);
                    const int d = div_small(e, rank_magic) - b;
                    if (d >= 0) {
                        const int q = div_small(d, gmag);
                        if (q * G == d && q < nd) hits |= 1u << q;
                    }
                }
            }
            if (g0 + (int64_t)u * NT < n) {   // warp-uniform
                for (int i = 0; i < nd; ++i) {
                    const int c = __popc(__ballot_sync(0xFFFFFFFFu, (hits >> i) & 1u));
                    if (lane == i) dc += c;
                }
            }
        }
    }
    if (lane < nd && dc) red_shared_add(dcnt + lane, dc);
}

// The scan over every id by NT threads (all of them must call it).
template <int NT>
__device__ void rep_scan(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int64_t t0, bool vec,
                         const Smem &s) {
    const int G = gridDim.x, b = blockIdx.x;
    const int nd = G > 1 ? rep_designated(b, G, R) : 0;
    const uint32_t rm = div_magic(E / R);
    if (k <= 8) {
        if (vec) rep_scan_ids<true, 8, NT>(idx, n, k, E, t0, s.base, s.total, rm, b, G, nd, s.part);
        else rep_scan_ids<false, 8, NT>(idx, n, k, E, t0, s.base, s.total, rm, b, G, nd, s.part);
    } else {
        if (vec) rep_scan_ids<true, kMaxTopk, NT>(idx, n, k, E, t0, s.base, s.total, rm, b, G, nd, s.part);
        else rep_scan_ids<false, kMaxTopk, NT>(idx, n, k, E, t0, s.base, s.total, rm, b, G, nd, s.part);
    }
}

// Zero a replicated-count block's shared counters (NT threads).
template <int NT>
__device__ void rep_zero(int T, int E, int R, const Smem &s) {
    zero_words<NT>(s.wc, kWarps * E);
    zero_words<NT>(reinterpret_cast<int32_t *>(s.mask), T * mask_words(R));
    zero_words<NT>(s.hr, R);
    zero_words<NT>(s.total, E);
    zero_words<NT>(s.base, E);
    zero_words<NT>(s.part, 32);
}

// The block's own part of a replicated-count layout once the scan's counts are
// in shared memory (s.base: copies before the block, s.total: the rest, s.part:
// designated-rank counts), run by the 256 threads of warps 0-7 (barrier 1):
// block b = blockIdx.x of G = gridDim.x owns tokens [b T, b T + T).  Ranks its
// own copies, writes every layout output of its own tokens, its designated
// ranks' tokens_per_rank, its share of the recv_src fill, and (block 0) the
// expert counts, offsets and max; s_dst (optional, shared, T k words) also
// receives its rows.  P holds the block's ids (load_pairs_only, then checked
// here).  Three barriers: after the warp ranks and rank sets; after the warp
// offsets, the warps' scans of the expert totals and the is_token_in_rank
// rows; after the bases.  scan_tmp: 2 kWarps words.
// Requires G == 1 or rep_designated(0, G, R) <= 32.
template <int CH>
__device__ void rep_finish(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, bool bad,
                           PairsT<CH> &P, int32_t *__restrict__ tokens_per_expert,
                           int32_t *__restrict__ tokens_per_rank, uint8_t *__restrict__ in_rank,
                           int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                           int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                           uint32_t *status, const Smem &s, int32_t *scan_tmp, int32_t *s_dst) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    const int nd = G > 1 ? rep_designated(b, G, R) : 0;
    key_and_rank<false, CH>(idx, k, E, E / R, E, s, P);
    rank_sets<CH>(k, E, R, s, P);
    if (lsync_or(bad) && tid == 0) report(status, kErrRange);
    warp_offsets(E, s);
    // expert totals (rest + before) and their exclusive scan: thread tid takes
    // experts [i0, i1), a warp scans its threads' sums, scan_tmp[w] holds warp
    // w's total and scan_tmp[kWarps + w] its largest count
    const int per = (E + kThreads - 1) / kThreads;
    const int i0 = min(E, tid * per), i1 = min(E, i0 + per);
    int32_t local = 0, mx = 0;
    for (int i = i0; i < i1; ++i) {
        const int32_t t = s.total[i] + s.base[i];
        s.total[i] = t;
        local += t;
        mx = max(mx, t);
    }
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 31) scan_tmp[warp] = incl;
    if (lane == 0) scan_tmp[kWarps + warp] = mx;
    if (G == 1) rank_counts<CH>(k, R, s, P);   // one block: its own tokens are all tokens
    else if (tid < nd) tokens_per_rank[b + tid * G] = s.part[tid];
    write_rank_rows<CH>(R, in_rank, s, P);
    lsync();
    int32_t run = incl - local, m_total = 0, m_max = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int32_t v = scan_tmp[w];
        if (w < warp) run += v;
        m_total += v;
        m_max = max(m_max, scan_tmp[kWarps + w]);
    }
    for (int i = i0; i < i1; ++i) {
        const int32_t t = s.total[i];
        s.base[i] += cap > 0 ? i * cap : run;
        if (b == 0) {
            tokens_per_expert[i] = t;
            expert_offset[i] = run;
        }
        run += t;
    }
    if (b == 0 && tid == 0) {
        expert_offset[E] = m_total;
        *max_count = m_max;
    }
    if (G == 1)
        for (int r = tid; r < R; r += kThreads) tokens_per_rank[r] = s.hr[r];
    lsync();
    const int64_t step = (int64_t)G * kThreads;
    if (cap > 0) {   // rows past an expert's copies
        const int64_t rows = (int64_t)E * cap;
        for (int64_t i = (int64_t)b * kThreads + tid; i < rows; i += step) {
            const int e = (int)(i / cap);
            if (i - (int64_t)e * cap >= s.total[e]) recv_src[i] = -1;
        }
    } else {         // rows past the last copy (ids of -1)
        for (int64_t i = m_total + (int64_t)b * kThreads + tid; i < n * k; i += step) recv_src[i] = -1;
    }
    bool over = false, bad_row = false;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int p = pair_of<CH>(i);
        if (p >= P.np) continue;
        const int32_t e = P.e[i];
        int32_t d = -1;
        if (e >= 0) {
            const int32_t pos = s.base[e] + s.wc[warp * E + e] + P.rk[i];
            if (cap > 0 && pos - e * cap >= cap) over = true;
            else if (pos >= recv_rows) bad_row = true;
            else d = pos;
        }
        const int64_t q = P.t0 * k + p;
        dst_pos[q] = d;
        if (s_dst) s_dst[p] = d;
        if (d >= 0) recv_src[d] = (int32_t)q;   // the row's source slot t k + j
    }
    if (over) report(status, kErrCapacity);
    if (bad_row) report(status, kErrRange);
}

// A whole replicated-count layout block run by the 256 threads of warps 0-7.
template <int CH>
__device__ void rep_layout_block(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int T,
                                 bool vec, int32_t *__restrict__ tokens_per_expert,
                                 int32_t *__restrict__ tokens_per_rank, uint8_t *__restrict__ in_rank,
                                 int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                                 int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                                 uint32_t *status, const Smem &s, int32_t *scan_tmp, int32_t *s_dst) {
    PairsT<CH> P;
    load_pairs_only<CH>(idx, n, k, blockIdx.x, T, P);   // in flight while zeroing and scanning
    rep_zero<kThreads>(T, E, R, s);
    lsync();
    rep_scan<kThreads>(idx, n, k, E, R, P.t0, vec, s);
    const bool bad = check_pairs<CH>(E, P);
    rep_finish<CH>(idx, n, k, E, R, cap, bad, P, tokens_per_expert, tokens_per_rank, in_rank, expert_offset,
                   max_count, dst_pos, recv_src, recv_rows, status, s, scan_tmp, s_dst);
}

// Standalone replicated-count layout: CTAs of NT threads, all of which zero
// the counters and scan the ids (the scan is latency-bound, so past a few
// thousand ids it wants every warp the SM can hold: NT = kRepThreads); warps
// 0-7 then finish the block.
constexpr int kRepThreads = 1024;

template <int CH, int NT>
__global__ void __launch_bounds__(NT)
layout_rep_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int vec,
                  int32_t *__restrict__ tokens_per_expert, int32_t *__restrict__ tokens_per_rank,
                  uint8_t *__restrict__ in_rank, int32_t *__restrict__ expert_offset,
                  int32_t *__restrict__ max_count, int32_t *__restrict__ dst_pos,
                  int32_t *__restrict__ recv_src, int64_t recv_rows, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_rep[];
    __shared__ int32_t scan_tmp[32];
    const int T = tokens_per_block(k, CH);
    const Smem s = carve_rep(smem_rep, T, E, R);
    griddep_wait();   // the ids, and readers of the outputs, may be the kernels just before
    PairsT<CH> P;
    if (threadIdx.x < kThreads) load_pairs_only<CH>(idx, n, k, blockIdx.x, T, P);   // in flight
    rep_zero<NT>(T, E, R, s);
    __syncthreads();
    rep_scan<NT>(idx, n, k, E, R, (int64_t)blockIdx.x * T, vec != 0, s);
    __syncthreads();
    if (threadIdx.x < kThreads)
        rep_finish<CH>(idx, n, k, E, R, cap, check_pairs<CH>(E, P), P, tokens_per_expert, tokens_per_rank, in_rank,
                       expert_offset, max_count, dst_pos, recv_src, recv_rows, status, s, scan_tmp, nullptr);
}

// Fused decode path: the layout and the FP8 dispatch of a small batch (at most
// 1024 (token, slot) pairs) in one launch, no workspace.  CTA b owns tokens
// [b T, b T + T) (one token per CTA when there are as many SMs as tokens) as a
// replicated-count layout block: it reads the batch's ids for the global
// counts, ranks its own copies and keeps their rows in shared memory, then
// quantises its tokens and writes their copies with 16-byte stores (one
// thread per 16 values of the CTA's flattened (token, chunk) range; the 8
// lanes of a 128-value block share one scale).
template <int CH>
__global__ void __launch_bounds__(kThreads)
decode_fused_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int T, int vec,
                    const uint16_t *__restrict__ x, int h, int32_t *__restrict__ tokens_per_expert,
                    int32_t *__restrict__ tokens_per_rank, uint8_t *__restrict__ in_rank,
                    int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                    int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                    uint8_t *__restrict__ recv_x, float *__restrict__ recv_scale, int pow2, uint32_t *status) {
    extern __shared__ __align__(16) int32_t smem_decode[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve_rep(smem_decode, T, E, R);
    int32_t *s_dst = smem_decode + rep_smem_words(T, E, R);   // [T k] receive row per own pair
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    griddep_wait();                // ids and x may come from the kernels just before
    rep_layout_block<CH>(idx, n, k, E, R, cap, T, vec != 0, tokens_per_expert, tokens_per_rank, in_rank,
                         expert_offset, max_count, dst_pos, recv_src, recv_rows, status, s, scan_tmp, s_dst);
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * T;
    const int nt = t0 < n ? (int)(n - t0 < T ? n - t0 : T) : 0;
    const int chunks = h >> 4, nblk = h >> 7;
    const int total = nt * chunks;   // a multiple of 8: a scale block never straddles tokens
    for (int g0 = warp * 32; g0 < total; g0 += kThreads) {   // warp-uniform
        const int g = g0 + lane;
        const bool active = g < total;
        const int tl = active ? g / chunks : 0, c = active ? g - tl * chunks : 0;
        uint4 a = make_uint4(0, 0, 0, 0), b = a;
        if (active) {
            const uint16_t *src = x + (t0 + tl) * h + (int64_t)c * 16;
            a = ld_nc_v4(src);
            b = ld_nc_v4(src + 8);
        }
        float m = absmax16(a, b);
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        if (!active) continue;
        const float amax_c = fmaxf(m, 1e-4f);
        float scale, inv;
        block_scale(amax_c, pow2 != 0, scale, inv);
        const uint4 q = quant16(a, b, inv);
        for (int j = 0; j < k; ++j) {
            const int32_t row = s_dst[tl * k + j];
            if (row < 0) continue;
            st_cs_v4(recv_x + (int64_t)row * h + (int64_t)c * 16, q);
            if ((c & 7) == 0) recv_scale[(int64_t)row * nblk + (c >> 3)] = scale;
        }
    }
}

// Decode batches of at most one token per SM: one CTA per token.  CTA t
// needs, for its own k copies, the copies of each expert in tokens before t
// and the expert offsets; everything else is the block's share of the global
// outputs.  Each of the first n threads reads one token's ids (one round of
// loads) and counts them into before[] / rest[] (shared reductions), the
// batch's valid ids, and distinct tokens of the CTA's designated ranks (t, t +
// n, ...: one ballot per rank).  Then each own slot j is ranked by one warp:
// offset = the sum of totals below its expert (a warp reduction, so no block
// scan outside CTA 0), rank = before[e] + the earlier slots of the token with
// that expert.  CTA 0 writes the expert counts, offsets and max; every CTA
// writes its token's rows, is_token_in_rank row and share of the recv_src
// fill, then (kDispatch) quantises the token as the fused decode kernel does.
// About five block barriers where the general block takes a dozen.  The
// dispatching instance runs 512 threads, so one pass quantises a 7168-value
// token (the layout phases use threads 0-255); the layout-only instance (256
// threads) serves cgl_get_layout for such batches.
template <int KM, bool kDispatch, int NT>
__global__ void __launch_bounds__(NT, 1)
decode_token_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int vec,
                    const uint16_t *__restrict__ x, int h, int32_t *__restrict__ tokens_per_expert,
                    int32_t *__restrict__ tokens_per_rank, uint8_t *__restrict__ in_rank,
                    int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                    int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                    uint8_t *__restrict__ recv_x, float *__restrict__ recv_scale, int pow2, uint32_t *status) {
    __shared__ int32_t s_before[kMaxExperts];   // copies in tokens before this CTA's
    __shared__ int32_t s_total[kMaxExperts];    // copies in the rest, then in all tokens
    __shared__ int32_t s_off[kMaxExperts];      // CTA 0: exclusive prefix of s_total
    __shared__ int32_t s_own[kMaxTopk];         // this token's ids
    __shared__ int32_t s_row[kMaxTopk];         // their receive rows
    __shared__ uint32_t s_mask[32];             // this token's rank set (R <= 1024)
    __shared__ int32_t s_cnt[1 + 32];           // [0]: valid ids of the batch; [1 + i]: designated rank i
    __shared__ int32_t scan_tmp[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    const int64_t t = b;
    const bool has_tok = t < n;
    const int nd = G > 1 ? rep_designated(b, G, R) : 0;
    const uint32_t rm = div_magic(E / R), gm = div_magic(G);
    griddep_wait();   // ids and x may come from the kernels just before
    // the dispatch's first pass over the CTA's token: its x loads are in flight
    // through the layout (16 values per thread)
    uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
    if (kDispatch && has_tok && tid < (h >> 4)) {
        xa = ld_nc_v4(x + t * h + (int64_t)tid * 16);
        xb = ld_nc_v4(x + t * h + (int64_t)tid * 16 + 8);
    }
    // this thread's token (n <= 256 = the block size): its ids, in flight while zeroing
    int32_t ids[KM];
    const int64_t tp = tid;
    {
        const int32_t *src = idx + tp * k;
        if (vec) {
#pragma unroll
            for (int q = 0; q < KM / 4; ++q) {
                int4 v = make_int4(-1, -1, -1, -1);
                if (tp < n && q * 4 < k) v = __ldg(reinterpret_cast<const int4 *>(src) + q);
                ids[4 * q] = v.x; ids[4 * q + 1] = v.y; ids[4 * q + 2] = v.z; ids[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < KM; ++j) ids[j] = (tp < n && j < k) ? __ldg(src + j) : -1;
        }
    }
    for (int e = tid; e < E; e += NT) {
        s_before[e] = 0;
        s_total[e] = 0;
    }
    if (tid < 32) s_mask[tid] = 0;
    if (tid < 33) s_cnt[tid] = 0;
    __syncthreads();
    uint32_t hits = 0;
    int valid = 0;
    if (tp < n) {
        int32_t *cnt = tp < t ? s_before : s_total;
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            const int32_t e = ids[j];
            if (j < k && (uint32_t)e < (uint32_t)E) {
                red_shared_add(cnt + e, 1);
                ++valid;
                const int r = div_small(e, rm);
                const int d = r - b;
                if (d >= 0) {
                    const int q = div_small(d, gm);
                    if (q * G == d && q < nd) hits |= 1u << q;
                }
                if (tp == t) atomicOr(&s_mask[r >> 5], 1u << (r & 31));
            }
        }
        if (tp == t) {
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j < k) s_own[j] = ids[j];
        }
    }
    valid = __reduce_add_sync(0xFFFFFFFFu, valid);
    if (lane == 0 && valid) red_shared_add(&s_cnt[0], valid);
    for (int i = 0; i < nd; ++i) {   // block-uniform
        const int c = __popc(__ballot_sync(0xFFFFFFFFu, (hits >> i) & 1u));
        if (lane == 0 && c) red_shared_add(&s_cnt[1 + i], c);
    }
    __syncthreads();
    for (int e = tid; e < E; e += NT) s_total[e] += s_before[e];
    if (G > 1) {
        if (tid < nd) tokens_per_rank[b + tid * G] = s_cnt[1 + tid];
    } else {
        for (int r = tid; r < R; r += NT) tokens_per_rank[r] = (int32_t)((s_mask[r >> 5] >> (r & 31)) & 1u);
    }
    if (has_tok)
        for (int r = tid; r < R; r += NT)
            in_rank[t * R + r] = (uint8_t)((s_mask[r >> 5] >> (r & 31)) & 1u);
    __syncthreads();
    const int32_t m_total = s_cnt[0];

    // own rows: slot j ranked by warp j % 8 (an empty batch's single CTA has none)
    bool over = false, bad = false;
    for (int j = warp; has_tok && j < k; j += NT / 32) {   // warp-uniform
        const int32_t e = s_own[j];
        int32_t row = -1;
        if ((uint32_t)e < (uint32_t)E) {
            int32_t below = 0;
            if (cap == 0)
                for (int q = lane; q < e; q += 32) below += s_total[q];
            below = __reduce_add_sync(0xFFFFFFFFu, below);
            int dup = 0;
            for (int jj = 0; jj < j; ++jj) dup += s_own[jj] == e ? 1 : 0;
            const int32_t rank = s_before[e] + dup;
            if (cap > 0) {
                if (rank >= cap) over = true;
                else row = e * cap + rank;
            } else {
                row = below + rank;
            }
            if (row >= recv_rows) { bad = true; row = -1; }
        } else if (e != -1) {
            bad = true;
        }
        if (lane == 0) {
            s_row[j] = row;
            dst_pos[t * k + j] = row;
            if (row >= 0) recv_src[row] = (int32_t)(t * k + j);
        }
    }
    if (lane == 0 && over) report(status, kErrCapacity);
    if (lane == 0 && bad) report(status, kErrRange);

    // CTA 0: counts, offsets, max (threads 0-255: the scan's barrier is hardware barrier 1)
    if (b == 0) {
        if (tid < kThreads) {
            const int32_t tot = block_exclusive_scan(s_total, s_off, E, scan_tmp);
            int32_t mx = 0;
            for (int e = tid; e < E; e += kThreads) {
                tokens_per_expert[e] = s_total[e];
                expert_offset[e] = s_off[e];
                mx = max(mx, s_total[e]);
            }
            if (tid == 0) expert_offset[E] = tot;
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
            if (lane == 0) scan_tmp[warp] = mx;
        }
        __syncthreads();
        if (tid == 0) {
            int32_t m = 0;
            for (int w = 0; w < kWarps; ++w) m = max(m, scan_tmp[w]);
            *max_count = m;
        }
    }
    // this CTA's share of the rows that receive nothing
    const int64_t fstep = (int64_t)G * NT;
    if (cap > 0) {
        for (int64_t i = (int64_t)b * NT + tid; i < (int64_t)E * cap; i += fstep) {
            const int e = (int)(i / cap);
            if (i - (int64_t)e * cap >= s_total[e]) recv_src[i] = -1;
        }
    } else {
        for (int64_t i = m_total + (int64_t)b * NT + tid; i < n * k; i += fstep) recv_src[i] = -1;
    }
    __syncthreads();   // s_row

    // the token's FP8 rows: 16 values per thread per pass, 8 lanes per scale block
    if (!kDispatch || !has_tok) return;
    const int chunks = h >> 4, nblk = h >> 7;
    for (int c0 = warp * 32; c0 < chunks; c0 += NT) {   // warp-uniform
        const int c = c0 + lane;
        const bool active = c < chunks;
        uint4 a = xa, bb = xb;   // the first pass was loaded at the start (c == tid)
        if (c0 != warp * 32 && active) {
            a = ld_nc_v4(x + t * h + (int64_t)c * 16);
            bb = ld_nc_v4(x + t * h + (int64_t)c * 16 + 8);
        }
        float m = absmax16(a, bb);
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        if (!active) continue;
        const float amax_c = fmaxf(m, 1e-4f);
        float scale, inv;
        block_scale(amax_c, pow2 != 0, scale, inv);
        const uint4 q = quant16(a, bb, inv);
        for (int j = 0; j < k; ++j) {
            const int32_t row = s_row[j];
            if (row < 0) continue;
            st_cs_v4(recv_x + (int64_t)row * h + (int64_t)c * 16, q);
            if ((c & 7) == 0) recv_scale[(int64_t)row * nblk + (c >> 3)] = scale;
        }
    }
}

// ------------------------------------------- fused layout + FP8 dispatch
//
// Prefill-sized batches: the layout and the FP8 dispatch in one launch, one
// CTA of 768 threads per SM.  CTA b owns tokens [b T, b T + T) both as a
// replicated-count layout block and for the dispatch.
//   1. All 24 warps read every id of the batch into the block's shared
//      histograms (before / rest, designated ranks): the one phase whose cost
//      grows with the batch, done first with every warp so it is short and
//      nothing competes with it.
//   2. Warps 0-7 then finish the layout block (own ranks, rows, outputs; their
//      barriers are hardware barrier 1 with 256 threads) and keep the block's
//      receive rows in shared memory, while warps 8-23 read the CTA's tokens
//      and stage their FP8 codes and scales in shared memory, in token order.
//      The tokens form up to kMaxGroups groups; every warp but warp 0 arrives
//      on a group's hardware barrier (2 + g) once it has no chunk left in it.
//   3. As soon as the rows are known, the lanes of warp 0 wait on each group's
//      barrier in turn and hand its staged rows to the TMA engine, one bulk copy
//      per receive row (and one per scale row), so the HBM writes of early
//      tokens overlap the reads of later ones; warps 1-7 stage the CTA's last
//      tokens.
// At kernel start the TMA engine is also asked to bring the CTA's own ids,
// then its x rows (one contiguous range), into L2, so that the id scan and the
// staging reads hit L2; the block's own ids are checked only after the scan.
// No CTA waits on another.  It runs only when a CTA's whole share fits in
// shared memory (at hidden 7168 up to 28 tokens per CTA, 4144 on 148 SMs).

constexpr int kLdThreads = 768;
constexpr int kStageUnroll = 2;    // thread-chunks per batch; two batches in registers
constexpr int kGroupBar = 2;       // hardware barriers 2 .. 2 + kMaxGroups - 1: staged token groups
constexpr int kMaxGroups = 14;
// Share of a CTA's tokens staged by layout warps 1-7 once the layout is done
// (they start a few microseconds after the 16 staging warps).
constexpr int kLateShareNum = 5, kLateShareDen = 28;
constexpr int64_t kPrefetchBytes = 32 * 1024;   // bytes per L2 prefetch instruction

__device__ __forceinline__ void bar_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Tokens [group_begin(g), group_begin(g + 1)) of cnt form staging group g of ng.
__device__ __forceinline__ int group_begin(int g, int cnt, int ng) { return (int)(((int64_t)g * cnt) / ng); }

__host__ __device__ __forceinline__ size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Dynamic shared memory of the fused layout + dispatch kernel: the layout
// block's region, its receive rows (T k words), then B staged rows of h codes
// and h / 128 fp32 scales.
__host__ __device__ __forceinline__ size_t ld_fixed_bytes(int k, int E, int R, int T) {
    return align16(rep_smem_words(T, E, R) * sizeof(int32_t) + (size_t)T * k * sizeof(int32_t));
}
__host__ __device__ __forceinline__ size_t ld_row_bytes(int h) { return (size_t)h + (size_t)(h >> 7) * 4; }

// Quantise staged tokens: thread-chunks of kStageV consecutive values of one
// token (one 16-byte load per 8 values), kStageLanes = 128 / kStageV lanes per
// 128-value scale block, which combine their block maximum with xor-shuffles.
// The arithmetic is the dispatch kernel's: block absmax, amax_c = max(amax,
// 1e-4), scale = amax_c / 448 and inv = 448 / amax_c (IEEE divisions), codes =
// e4m3_rn_satfinite(x * inv), written to qbuf[t][h]; the block's first lane
// writes the scale to sbuf[t][h / 128].  (32 values per thread, with half the
// shuffles and divisions per value, measured slower on B200: 72.6 against
// 63 us for the whole kernel at 4096 tokens.)
constexpr int kStageV = 16;
constexpr int kStageLanes = 128 / kStageV;
constexpr int kStageLoads = kStageV / 8;     // 16-byte loads per thread-chunk

struct StageBatch {
    uint4 d[kStageUnroll][kStageLoads];
    int t[kStageUnroll], c[kStageUnroll];
};

// Issue the loads of the next kStageUnroll chunks of this thread ((t, c)
// advanced by nth chunks per step).  The loads allocate in L1: the two 16-byte
// halves of a lane's 32-byte sector come from consecutive instructions.
__device__ __forceinline__ void stage_load(const uint16_t *__restrict__ x, int h, int64_t t_first, int cnt,
                                           int chunks, int dt, int dc, int &t, int &c, StageBatch &B) {
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u) {
        B.t[u] = t;
        B.c[u] = c;
        const uint16_t *src = x + (t_first + t) * h + (int64_t)c * kStageV;
#pragma unroll
        for (int i = 0; i < kStageLoads; ++i) B.d[u][i] = t < cnt ? ld_nc_l1_v4(src + 8 * i) : make_uint4(0, 0, 0, 0);
        t += dt;
        c += dc;
        if (c >= chunks) { c -= chunks; ++t; }
    }
}

__device__ __forceinline__ void stage_quantise(int h, int cnt, const StageBatch &B, uint8_t *qbuf, float *sbuf,
                                               int pow2) {
    const int nblk = h >> 7;
#pragma unroll
    for (int u = 0; u < kStageUnroll; ++u) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < kStageLoads; i += 2) m = fmaxf(m, absmax16(B.d[u][i], B.d[u][i + 1]));
#pragma unroll
        for (int o = kStageLanes / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (B.t[u] < cnt) {
            const float amax_c = fmaxf(m, 1e-4f);
            float scale, inv;
            block_scale(amax_c, pow2 != 0, scale, inv);
            uint4 *dst = reinterpret_cast<uint4 *>(qbuf + (size_t)B.t[u] * h + (size_t)B.c[u] * kStageV);
#pragma unroll
            for (int i = 0; i < kStageLoads; i += 2) dst[i / 2] = quant16(B.d[u][i], B.d[u][i + 1], inv);
            if ((B.c[u] & (kStageLanes - 1)) == 0) sbuf[B.t[u] * nblk + B.c[u] / kStageLanes] = scale;
        }
    }
}

// Stage tokens [tok_begin, tok_end) of the CTA's cnt tokens (global tokens
// t_first + ...; see stage_quantise) with threads [th0, th0 + nth), and signal
// the store issuer group by group: the CTA's tokens form ng groups, and a warp
// arrives on barrier kGroupBar + g (bar_count threads in all) once its next
// chunk lies past group g (a thread's chunks come in increasing order, and
// lane 0's is the warp's lowest), after a proxy fence so that the bulk copies
// see its codes.  Groups before the range are arrived on at once, those after
// it at the end: every calling warp arrives on every group exactly once.
__device__ void stage_fp8_rows_grouped(const uint16_t *__restrict__ x, int h, int64_t t_first, int cnt,
                                       int tok_begin, int tok_end, uint8_t *qbuf, float *sbuf, int th0, int nth,
                                       int ng, int bar_count, int pow2) {
    const int chunks = h / kStageV;    // a multiple of kStageLanes: a scale block never straddles tokens
    const int q0 = tok_begin * chunks, q1 = tok_end * chunks;
    const int me = (int)threadIdx.x - th0;
    const int wme = me & ~31;          // lane 0's offset
    // (token, chunk) of this thread's next chunk, advanced by nth per step
    const int dt = nth / chunks, dc = nth - dt * chunks;
    int t = (q0 + me) / chunks, c = (q0 + me) - t * chunks;
    int g_next = 0;                    // next group this warp arrives on
    auto arrive_below = [&](int64_t next_min) {
        while (g_next < ng && (int64_t)group_begin(g_next + 1, cnt, ng) * chunks <= next_min) {
            fence_proxy_async();
            bar_arrive(kGroupBar + g_next, bar_count);
            ++g_next;
        }
    };
    arrive_below((int64_t)q0 + wme);
    // two batches in registers: the next batch's loads are in flight while
    // the current one is quantised (uniform loop: every lane joins the shuffles)
    const int step = nth * kStageUnroll;
    StageBatch b0, b1;
    if (q0 < q1) stage_load(x, h, t_first, tok_end, chunks, dt, dc, t, c, b0);
    for (int base = q0; base < q1;) {
        const bool has1 = base + step < q1;
        if (has1) stage_load(x, h, t_first, tok_end, chunks, dt, dc, t, c, b1);
        stage_quantise(h, tok_end, b0, qbuf, sbuf, pow2);
        base += step;
        arrive_below((int64_t)wme + base);
        if (!has1) break;
        const bool has2 = base + step < q1;
        if (has2) stage_load(x, h, t_first, tok_end, chunks, dt, dc, t, c, b0);
        stage_quantise(h, tok_end, b1, qbuf, sbuf, pow2);
        base += step;
        arrive_below((int64_t)wme + base);
        if (!has2) break;
    }
    arrive_below(INT64_MAX);
}

// Write staged tokens [t_begin, t_end) of this CTA to their receive rows: one
// bulk copy per (token, slot) with a row, issued by the 32 lanes of the
// calling warp; scales by bulk copy when their row is a multiple of 16 bytes
// and 16-byte aligned, else by plain stores.  Each lane commits its own bulk
// group.
__device__ void issue_fp8_rows(int k, int h, int t_begin, int t_end, const int32_t *s_dst, const uint8_t *qbuf,
                               const float *sbuf, uint8_t *__restrict__ recv_x, float *__restrict__ recv_scale,
                               bool scale_bulk) {
    const int nblk = h >> 7;
    const int lane = threadIdx.x & 31;
    for (int p = t_begin * k + lane; p < t_end * k; p += 32) {
        const int t = p / k;
        const int32_t row = s_dst[p];
        if (row < 0) continue;
        bulk_store(recv_x + (int64_t)row * h, qbuf + (size_t)t * h, (uint32_t)h);
        if (scale_bulk) {
            bulk_store(recv_scale + (int64_t)row * nblk, sbuf + t * nblk, (uint32_t)(nblk * 4));
        } else {
            for (int i = 0; i < nblk; ++i) recv_scale[(int64_t)row * nblk + i] = sbuf[t * nblk + i];
        }
    }
    bulk_commit();
}

template <int CH>
__global__ void __launch_bounds__(kLdThreads, 1)
layout_dispatch_fp8_kernel(const int32_t *__restrict__ idx, int64_t n, int k, int E, int R, int cap, int T,
                           int B, int vec, int32_t *__restrict__ tokens_per_expert,
                           int32_t *__restrict__ tokens_per_rank, uint8_t *__restrict__ in_rank,
                           int32_t *__restrict__ expert_offset, int32_t *__restrict__ max_count,
                           int32_t *__restrict__ dst_pos, int32_t *__restrict__ recv_src, int64_t recv_rows,
                           const uint16_t *__restrict__ x, int h, uint8_t *__restrict__ recv_x,
                           float *__restrict__ recv_scale, int scale_bulk, int pow2, uint32_t *status) {
    extern __shared__ __align__(128) int32_t smem_ld[];
    __shared__ int32_t scan_tmp[32];
    const Smem s = carve_rep(smem_ld, T, E, R);
    int32_t *s_dst = smem_ld + rep_smem_words(T, E, R);
    uint8_t *qbuf = reinterpret_cast<uint8_t *>(smem_ld) + ld_fixed_bytes(k, E, R, T);
    float *sbuf = reinterpret_cast<float *>(qbuf + (size_t)B * h);
    const int64_t t0 = (int64_t)blockIdx.x * T;
    const int nt = t0 < n ? (int)(n - t0 < T ? n - t0 : T) : 0;
    const int cnt0 = nt < B ? nt : B;   // == nt: the host launches this kernel only when B >= T
    const int ng = cnt0 < kMaxGroups ? (cnt0 > 0 ? cnt0 : 1) : kMaxGroups;
    const int split = cnt0 - (cnt0 * kLateShareNum) / kLateShareDen;   // warps 1-7 stage [split, cnt0)
    griddep_wait();   // ids and x may come from the kernels just before, which may still read our outputs
    prefetch_own_ids(idx, n, k, t0, T, vec != 0);   // ahead of x in the memory queues
    if (threadIdx.x < 32 && cnt0 > 0) {
        // the CTA's x rows are one contiguous range: the TMA engine streams it from
        // HBM into L2 while the ids are scanned, so the staging loads hit L2
        const char *src = reinterpret_cast<const char *>(x + t0 * h);
        const int64_t bytes = (int64_t)cnt0 * h * 2;
        for (int64_t off = (int64_t)threadIdx.x * kPrefetchBytes; off < bytes; off += 32 * kPrefetchBytes)
            prefetch_l2_bulk(src + off, (uint32_t)(bytes - off < kPrefetchBytes ? bytes - off : kPrefetchBytes));
    }
    PairsT<CH> P;
    if (threadIdx.x < kThreads) load_pairs_only<CH>(idx, n, k, blockIdx.x, T, P);   // in flight
    rep_zero<kLdThreads>(T, E, R, s);
    __syncthreads();
    rep_scan<kLdThreads>(idx, n, k, E, R, t0, vec != 0, s);
    __syncthreads();
    if (threadIdx.x < kThreads) {
        rep_finish<CH>(idx, n, k, E, R, cap, check_pairs<CH>(E, P), P, tokens_per_expert, tokens_per_rank, in_rank,
                       expert_offset, max_count, dst_pos, recv_src, recv_rows, status, s, scan_tmp, s_dst);
        lsync();   // every row of the block is in s_dst
        if (threadIdx.x < 32) {
            for (int g = 0; g < ng; ++g) {
                bar_sync(kGroupBar + g, kLdThreads);   // group g is staged
                issue_fp8_rows(k, h, group_begin(g, cnt0, ng), group_begin(g + 1, cnt0, ng), s_dst, qbuf, sbuf,
                               recv_x, recv_scale, scale_bulk != 0);
            }
            bulk_wait_all();
        } else {   // warps 1-7, free after the layout: the CTA's last tokens
            stage_fp8_rows_grouped(x, h, t0, cnt0, split, cnt0, qbuf, sbuf, 32, kThreads - 32, ng, kLdThreads, pow2);
        }
    } else {
        stage_fp8_rows_grouped(x, h, t0, cnt0, 0, split, qbuf, sbuf, kThreads, kLdThreads - kThreads, ng, kLdThreads,
                               pow2);
    }
}

// ------------------------------------------------------------------ host side

std::mutex g_mu;

// Per-call salt for the exchange tags: a process-wide call counter, spread
// over 31 bits by an odd multiplier (a bijection), with the top bit set.
std::atomic<uint32_t> g_calls{0};
uint32_t next_salt() {
    const uint32_t c = g_calls.fetch_add(1, std::memory_order_relaxed);
    return 0x80000000u | ((c * 0x9E3779B1u) & 0x7FFFFFFFu);
}

int g_fused_ctas_per_sm[2][3][64] = {{{0}}};   // fused-kernel occupancy at kSmemDefault, per mode, CH, device

__host__ __device__ constexpr int ch_slot(int ch) { return ch == 1 ? 0 : (ch == 2 ? 1 : 2); }

// Largest grid of the fused kernel that is certain to be co-resident; 0 if none.
template <bool kRankKeys, int CH>
int fused_capacity() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    int &slot = g_fused_ctas_per_sm[kRankKeys ? 1 : 0][ch_slot(CH)][dev];
    if (slot == 0) {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, layout_fused_kernel<kRankKeys, CH>, kThreads,
                                                          kSmemDefault) != cudaSuccess)
            return 0;
        slot = v > 0 ? v : -1;
    }
    return slot > 0 ? slot * device_sm_count() : 0;
}

int g_cluster_ok[2][64][kMaxClusterCtas + 1] = {{{0}}};   // per mode, device, size: 1 ok, -1 no

// CTAs of the cluster layout for n tokens (2..8 blocks of tokens_per_block(k, 1)
// tokens whose shared memory needs no opt-in and that the device can
// schedule as one cluster; queried once per size), else 0.
template <bool kRankKeys>
int cluster_ctas_for(int64_t n, int k, int nkeys, int R) {
    const int T = tokens_per_block(k, 1);
    const int64_t C = (n + T - 1) / T;
    if (C < 2 || C > kMaxClusterCtas) return 0;
    const size_t smem = smem_words(0, k, nkeys, R) * sizeof(int32_t);
    if (smem > kSmemDefault) return 0;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    int &ok = g_cluster_ok[kRankKeys ? 1 : 0][dev][C];
    if (ok == 0) {
        ok = -1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)C);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemDefault;   // the most this path uses
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, layout_cluster_kernel<kRankKeys>, &cfg) == cudaSuccess &&
            clusters >= 1)
            ok = 1;
        cudaGetLastError();   // a refused query must not linger as a sticky launch error
    }
    return ok == 1 ? (int)C : 0;
}

// Blocks of the replicated-count layout for n tokens (one chunk per warp, T =
// tokens_per_block(k, 1) tokens per block), or 0 when it does not apply: more
// than kRepMaxPairs pairs, more than 32 designated ranks per block, or more
// shared memory than a kernel gets without opting in.
int rep_grid(int64_t n, int k, int E, int R) {
    if (n * k > kRepMaxPairs) return 0;
    const int T = tokens_per_block(k, 1);
    const int64_t G = n > 0 ? (n + T - 1) / T : 1;
    if (G > 1 && rep_designated(0, (int)G, R) > 32) return 0;
    if (rep_smem_words(T, E, R) * sizeof(int32_t) > kSmemDefault) return 0;
    return (int)G;
}

template <bool kRankKeys>
bool fused_fits(int64_t n, int k, int nkeys, int R) {
    const WsLayout w = ws_layout(n, k, nkeys, R);
    if (smem_words(0, k, nkeys, R) * sizeof(int32_t) > kSmemDefault) return false;
    switch (layout_chunks(n, k)) {
        case 1: return w.blocks <= fused_capacity<kRankKeys, 1>();
        case 2: return w.blocks <= fused_capacity<kRankKeys, 2>();
        default: return w.blocks <= fused_capacity<kRankKeys, 4>();
    }
}

// Fused layout + FP8 dispatch: launch shape for n tokens.  T = tokens per CTA
// (one CTA per SM, at least 64 pairs each), CH = chunks per warp of its layout
// block, B = tokens the shared memory can stage (>= T, else ok = false and the
// layout and the dispatch run separately).
constexpr int kLdMaxBlocks = 256;

int g_optin_smem[64] = {0};   // per device: largest dynamic shared memory a block may opt in to

int optin_smem_bytes() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_optin_smem[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
        g_optin_smem[dev] = v > 0 ? v : -1;
    }
    return g_optin_smem[dev];
}

struct LdShape {
    bool ok;
    int T, CH, B, G;
    size_t smem;
};

LdShape ld_shape(int64_t n, int k, int E, int R, int h, int num_sms) {
    LdShape r = {false, 0, 0, 0, 0, 0};
    int sms = device_sm_count();
    if (num_sms > 0 && num_sms < sms) sms = num_sms;
    if (n <= 0 || sms <= 0 || h <= 0 || h % 128 != 0) return r;
    if (n * k < 64 * (int64_t)sms) return r;   // small batches: a few CTAs would carry the whole dispatch
    if (n * k > kRepMaxPairs) return r;         // every CTA reads all ids
    int64_t T = (n + sms - 1) / sms;
    const int t_min = 64 / k > 0 ? 64 / k : 1;
    if (T < t_min) T = t_min;
    if (T > tokens_per_block(k, kChunks)) return r;
    const int64_t pairs = T * k;
    r.T = (int)T;
    r.CH = pairs <= 256 ? 1 : (pairs <= 512 ? 2 : 4);
    r.G = (int)((n + T - 1) / T);
    if (r.G > kLdMaxBlocks) return r;
    if (rep_designated(0, r.G, R) > 32) return r;
    const int optin = optin_smem_bytes();
    if (optin <= 0) return r;
    const size_t avail = optin > 1024 ? (size_t)optin - 1024 : 0;   // room for the static shared memory
    const size_t fixed = ld_fixed_bytes(k, E, R, r.T), row = ld_row_bytes(h);
    if (avail <= fixed) return r;
    const size_t b = (avail - fixed) / row;
    if (b < (size_t)r.T) return r;   // one staging round only
    r.B = r.T;
    r.smem = fixed + (size_t)r.B * row;
    r.ok = true;
    return r;
}

// CTAs per SM of the fused kernel at this shared memory, cached per device, CH
// and size (the shared memory only takes a few values: one per tokens per CTA).
struct LdOcc {
    int dev, ch;
    size_t smem;
    int occ;
};
LdOcc g_ld_occ[64];
int g_ld_occ_n = 0;

template <int CH>
bool ld_launchable(const LdShape &sh) {
    if (!ensure_smem_attr((const void *)layout_dispatch_fp8_kernel<CH>, sh.smem)) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    int occ = -1;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (int i = 0; i < g_ld_occ_n; ++i)
            if (g_ld_occ[i].dev == dev && g_ld_occ[i].ch == CH && g_ld_occ[i].smem == sh.smem) occ = g_ld_occ[i].occ;
    }
    if (occ < 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, layout_dispatch_fp8_kernel<CH>, kLdThreads,
                                                          sh.smem) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_ld_occ_n < 64) g_ld_occ[g_ld_occ_n++] = {dev, CH, sh.smem, occ};
    }
    return occ >= 1;   // no co-residency needed: the CTAs never wait on one another
}

bool ld_fits(const LdShape &sh) {
    if (!sh.ok) return false;
    switch (sh.CH) {
        case 1: return ld_launchable<1>(sh);
        case 2: return ld_launchable<2>(sh);
        default: return ld_launchable<4>(sh);
    }
}

template <int CH>
cgl_status ld_launch(const LdShape &sh, const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                     const uint16_t *x, int h, int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                     uint8_t *in_rank, int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                     int32_t *recv_src, uint8_t *recv_x, float *recv_scale, bool pow2, uint32_t *status,
                     cudaStream_t stream) {
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;
    const int scale_bulk = ((h >> 7) % 4 == 0) && (reinterpret_cast<uintptr_t>(recv_scale) % 16 == 0);
    const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
    const cudaError_t err = launch_pdl(layout_dispatch_fp8_kernel<CH>, dim3((unsigned)sh.G), dim3(kLdThreads), sh.smem,
                                       stream, idx, n, k, E, R, cap, sh.T, sh.B, vec, tokens_per_expert,
                                       tokens_per_rank, in_rank, expert_offset, max_count, dst_pos, recv_src,
                                       recv_rows, x, h, recv_x, recv_scale, scale_bulk, (int)pow2, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace

// One CTA per token: at most one token per SM in use (and per thread of the
// scanning block), at most 32 designated ranks per CTA, E within the static
// shared histograms.
bool token_layout_fits(int64_t n, int k, int E, int R, int use_sms) {
    (void)k;
    return n <= use_sms && n <= kThreads && E <= kMaxExperts && (n <= 1 || rep_designated(0, (int)n, R) <= 32);
}

template <bool kDispatch>
cgl_status launch_token_kernel(const int32_t *idx, int64_t n, int k, int E, int R, int cap, int vec,
                               const uint16_t *x, int h, int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                               uint8_t *in_rank, int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                               int32_t *recv_src, int64_t recv_rows, uint8_t *recv_x, float *recv_scale, bool pow2,
                               uint32_t *status, cudaStream_t stream) {
    constexpr int NT = kDispatch ? 2 * kThreads : kThreads;
    const dim3 grid((unsigned)(n < 1 ? 1 : n));
    const cudaError_t err =
        k <= 8 ? launch_pdl(decode_token_kernel<8, kDispatch, NT>, grid, dim3(NT), 0, stream, idx, n, k, E, R, cap,
                            vec, x, h, tokens_per_expert, tokens_per_rank, in_rank, expert_offset, max_count, dst_pos,
                            recv_src, recv_rows, recv_x, recv_scale, (int)pow2, status)
               : launch_pdl(decode_token_kernel<kMaxTopk, kDispatch, NT>, grid, dim3(NT), 0, stream, idx, n, k, E, R,
                            cap, vec, x, h, tokens_per_expert, tokens_per_rank, in_rank, expert_offset, max_count,
                            dst_pos, recv_src, recv_rows, recv_x, recv_scale, (int)pow2, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

size_t layout_workspace_bytes(int64_t n, int k, int E, int R) { return ws_layout(n, k, E, R).bytes; }

// Workspace of cgl_layout_dispatch_fp8: the layout's, then (16-byte aligned) a
// 64-bit token counter for the dispatch kernel when the layout and the
// dispatch run as two kernels; the fused kernel needs none.
size_t ld_claim_offset(int64_t n, int k, int E, int R) { return align16(ws_layout(n, k, E, R).bytes); }

size_t layout_dispatch_workspace_bytes(int64_t n, int k, int E, int R) {
    return ld_claim_offset(n, k, E, R) + 16;
}

bool layout_dispatch_fused_fits(int64_t n, int k, int E, int R, int h, int num_sms) {
    const int sms = device_sm_count();
    const int use_sms = (num_sms > 0 && num_sms < sms) ? num_sms : sms;
    if (sms > 0 && token_layout_fits(n, k, E, R, use_sms)) return true;
    return ld_fits(ld_shape(n, k, E, R, h, num_sms));
}

cgl_status launch_layout_dispatch_fp8(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                                      const uint16_t *x, int h, int32_t *tokens_per_expert,
                                      int32_t *tokens_per_rank, uint8_t *in_rank, int32_t *expert_offset,
                                      int32_t *max_count, int32_t *dst_pos, int32_t *recv_src, uint8_t *recv_x,
                                      float *recv_scale, void *ws, int num_sms, bool pow2, uint32_t *status,
                                      cudaStream_t stream) {
    {   // at most one token per SM: one CTA per token does both
        const int sms = device_sm_count();
        if (sms <= 0) return CGL_ECUDA;
        const int use_sms = (num_sms > 0 && num_sms < sms) ? num_sms : sms;
        if (token_layout_fits(n, k, E, R, use_sms)) {
            const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;
            const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
            return launch_token_kernel<true>(idx, n, k, E, R, cap, vec, x, h, tokens_per_expert, tokens_per_rank,
                                             in_rank, expert_offset, max_count, dst_pos, recv_src, recv_rows, recv_x,
                                             recv_scale, pow2, status, stream);
        }
    }
    const LdShape sh = ld_shape(n, k, E, R, h, num_sms);
    if (ld_fits(sh)) {
        switch (sh.CH) {
            case 1:
                return ld_launch<1>(sh, idx, n, k, E, R, cap, x, h, tokens_per_expert, tokens_per_rank, in_rank,
                                    expert_offset, max_count, dst_pos, recv_src, recv_x, recv_scale, pow2, status,
                                    stream);
            case 2:
                return ld_launch<2>(sh, idx, n, k, E, R, cap, x, h, tokens_per_expert, tokens_per_rank, in_rank,
                                    expert_offset, max_count, dst_pos, recv_src, recv_x, recv_scale, pow2, status,
                                    stream);
            default:
                return ld_launch<4>(sh, idx, n, k, E, R, cap, x, h, tokens_per_expert, tokens_per_rank, in_rank,
                                    expert_offset, max_count, dst_pos, recv_src, recv_x, recv_scale, pow2, status,
                                    stream);
        }
    }
    // two kernels: the dispatch hands its tokens out from a counter at the
    // workspace's tail, zeroed here first (before the layout, so that nothing
    // comes between the two kernels)
    unsigned long long *claim =
        reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) + ld_claim_offset(n, k, E, R));
    if (cudaMemsetAsync(claim, 0, 2 * sizeof(unsigned long long), stream) != cudaSuccess) return CGL_ECUDA;
    const cgl_status st = launch_layout(idx, n, k, E, R, cap, tokens_per_expert, tokens_per_rank, in_rank,
                                        expert_offset, max_count, dst_pos, recv_src, ws, status, stream);
    if (st != CGL_OK) return st;
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;
    return launch_dispatch_fp8(x, n, h, k, dst_pos, recv_x, recv_scale, recv_rows, num_sms, pow2, status, stream,
                               claim);
}

bool layout_needs_smem_optin(int E, int R, int k) {
    return smem_words(0, k, E, R) * sizeof(int32_t) > kSmemDefault;
}

bool layout_fused_fits(int64_t n, int k, int E, int R) {
    const int sms = device_sm_count();
    return (sms > 0 && token_layout_fits(n, k, E, R, sms)) || rep_grid(n, k, E, R) > 0 || fused_fits<false>(n, k, E, R);
}

template <bool kRankKeys, int CH>
cgl_status launch_layout_ch(const int32_t *idx, int64_t n, int k, int E_ids, int R, int cap,
                            int32_t *tokens_per_key, int32_t *tokens_per_rank, uint8_t *in_rank,
                            int32_t *key_offset, int32_t *max_count, int32_t *dst_pos, int32_t *recv_src,
                            void *ws, uint32_t *status, cudaStream_t stream) {
    const int E = kRankKeys ? R : E_ids;        // number of keys
    const int key_div = E_ids / R;
    const WsLayout w = ws_layout(n, k, E, R);
    uint64_t *flags = static_cast<uint64_t *>(ws);
    int32_t *ws_e = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.e_off);
    int32_t *ws_r = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + w.r_off);
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;

    if (fused_fits<kRankKeys>(n, k, E, R)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)w.blocks);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem_words(0, k, E, R) * sizeof(int32_t);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t err = cudaLaunchKernelEx(
            &cfg, layout_fused_kernel<kRankKeys, CH>, idx, n, k, E, R, cap, E_ids, key_div, flags, next_salt(),
            ws_e, ws_r,
            tokens_per_key, tokens_per_rank, in_rank, key_offset, max_count, dst_pos, recv_src, recv_rows,
            status);
        if (err == cudaSuccess) return CGL_OK;
        if (err != cudaErrorCooperativeLaunchTooLarge) return CGL_ECUDA;
        cudaGetLastError();   // fewer SMs free than the occupancy query counted: use the two kernels
    }

    const size_t smem1 = smem_words(1, k, E, R) * sizeof(int32_t);
    const size_t smem2 = smem_words(2, k, E, R) * sizeof(int32_t);
    if (smem1 > kSmemDefault && !ensure_smem_attr((const void *)layout_count_kernel<kRankKeys, CH>, smem1))
        return CGL_ECUDA;
    if (smem2 > kSmemDefault && !ensure_smem_attr((const void *)layout_rows_kernel<kRankKeys, CH>, smem2))
        return CGL_ECUDA;
    layout_count_kernel<kRankKeys, CH><<<(unsigned)w.blocks, kThreads, smem1, stream>>>(
        idx, n, k, E, R, E_ids, key_div, ws_e, ws_r, in_rank, status);
    if (cudaGetLastError() != cudaSuccess) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(layout_rows_kernel<kRankKeys, CH>, dim3((unsigned)w.blocks), dim3(kThreads),
                                       smem2, stream, idx, n, k, E, R, cap, E_ids, key_div,
                                       (const int32_t *)ws_e, (const int32_t *)ws_r, tokens_per_key,
                                       tokens_per_rank, key_offset, max_count, dst_pos, recv_src, recv_rows,
                                       status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

template <bool kRankKeys>
cgl_status launch_layout_impl(const int32_t *idx, int64_t n, int k, int E_ids, int R, int cap,
                              int32_t *tokens_per_key, int32_t *tokens_per_rank, uint8_t *in_rank,
                              int32_t *key_offset, int32_t *max_count, int32_t *dst_pos,
                              int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream) {
    const int nkeys = kRankKeys ? R : E_ids;
    if constexpr (!kRankKeys) {
        const int sms = device_sm_count();
        if (sms > 0 && token_layout_fits(n, k, E_ids, R, sms)) {
            const int64_t recv_rows = cap > 0 ? (int64_t)E_ids * cap : n * k;
            const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
            return launch_token_kernel<false>(idx, n, k, E_ids, R, cap, vec, nullptr, 0, tokens_per_key,
                                              tokens_per_rank, in_rank, key_offset, max_count, dst_pos, recv_src,
                                              recv_rows, nullptr, nullptr, false, status, stream);
        }
        const int G = rep_grid(n, k, E_ids, R);
        if (G > 0) {
            const int T = tokens_per_block(k, 1);
            const int64_t recv_rows = cap > 0 ? (int64_t)E_ids * cap : n * k;
            const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
            const size_t smem = rep_smem_words(T, E_ids, R) * sizeof(int32_t);
            const cudaError_t err =
                n * k > kRepWidePairs
                    ? launch_pdl(layout_rep_kernel<1, kRepThreads>, dim3((unsigned)G), dim3(kRepThreads), smem, stream,
                                 idx, n, k, E_ids, R, cap, vec, tokens_per_key, tokens_per_rank, in_rank, key_offset,
                                 max_count, dst_pos, recv_src, recv_rows, status)
                    : launch_pdl(layout_rep_kernel<1, kThreads>, dim3((unsigned)G), dim3(kThreads), smem, stream, idx,
                                 n, k, E_ids, R, cap, vec, tokens_per_key, tokens_per_rank, in_rank, key_offset,
                                 max_count, dst_pos, recv_src, recv_rows, status);
            return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
        }
    }
    const int C = cluster_ctas_for<kRankKeys>(n, k, nkeys, R);
    if (C > 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)C);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem_words(0, k, nkeys, R) * sizeof(int32_t);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const int64_t recv_rows = cap > 0 ? (int64_t)nkeys * cap : n * k;
        const cudaError_t err = cudaLaunchKernelEx(&cfg, layout_cluster_kernel<kRankKeys>, idx, n, k, nkeys, R, cap,
                                                   E_ids, E_ids / R, tokens_per_key, tokens_per_rank, in_rank,
                                                   key_offset, max_count, dst_pos, recv_src, recv_rows, status);
        return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
    }
    switch (layout_chunks(n, k)) {
        case 1:
            return launch_layout_ch<kRankKeys, 1>(idx, n, k, E_ids, R, cap, tokens_per_key, tokens_per_rank,
                                                  in_rank, key_offset, max_count, dst_pos, recv_src, ws, status,
                                                  stream);
        case 2:
            return launch_layout_ch<kRankKeys, 2>(idx, n, k, E_ids, R, cap, tokens_per_key, tokens_per_rank,
                                                  in_rank, key_offset, max_count, dst_pos, recv_src, ws, status,
                                                  stream);
        default:
            return launch_layout_ch<kRankKeys, 4>(idx, n, k, E_ids, R, cap, tokens_per_key, tokens_per_rank,
                                                  in_rank, key_offset, max_count, dst_pos, recv_src, ws, status,
                                                  stream);
    }
}

cgl_status launch_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                         int32_t *tokens_per_expert, int32_t *tokens_per_rank, uint8_t *in_rank,
                         int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                         int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream) {
    return launch_layout_impl<false>(idx, n, k, E, R, cap, tokens_per_expert, tokens_per_rank, in_rank,
                                     expert_offset, max_count, dst_pos, recv_src, ws, status, stream);
}

cgl_status launch_rank_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                              int32_t *tokens_per_rank, int32_t *rank_offset, int32_t *max_count,
                              int32_t *rank_dst, int32_t *recv_token, void *ws, uint32_t *status,
                              cudaStream_t stream) {
    return launch_layout_impl<true>(idx, n, k, E, R, cap, tokens_per_rank, nullptr, nullptr, rank_offset,
                                    max_count, rank_dst, recv_token, ws, status, stream);
}

cgl_status launch_wait_probe(uint64_t *ws, int nflags, uint32_t *status, cudaStream_t stream) {
    wait_probe_kernel<<<1, kThreads, 0, stream>>>(ws, nflags, status);
    return cudaGetLastError() == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

// Launch shape of the fused decode kernel: G CTAs of T tokens (at most one CTA
// per SM in use, and T k <= 1024 pairs); one CTA for everything when more
// CTAs would give one of them more than 32 designated ranks.
struct DecodeShape {
    int G, T, CH;
};
DecodeShape decode_shape(int64_t n, int k, int R, int use_sms) {
    DecodeShape d;
    const int64_t g = n < 1 ? 1 : (n < use_sms ? n : use_sms);
    d.T = n < 1 ? 1 : (int)((n + g - 1) / g);
    d.G = n < 1 ? 1 : (int)((n + d.T - 1) / d.T);
    if (d.G > 1 && rep_designated(0, d.G, R) > 32) {
        d.G = 1;
        d.T = n < 1 ? 1 : (int)n;
    }
    const int64_t pairs = (int64_t)d.T * k;
    d.CH = pairs <= 256 ? 1 : (pairs <= 512 ? 2 : 4);
    return d;
}

size_t decode_fused_smem_bytes(int64_t n, int k, int E, int R) {
    // the largest T any launch shape uses is n (a single CTA)
    const int T = n < 1 ? 1 : (int)n;
    return (rep_smem_words(T, E, R) + (size_t)T * k) * sizeof(int32_t);
}

cgl_status launch_decode_dispatch_fp8(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                                      const uint16_t *x, int h, int32_t *tokens_per_expert,
                                      int32_t *tokens_per_rank, uint8_t *in_rank, int32_t *expert_offset,
                                      int32_t *max_count, int32_t *dst_pos, int32_t *recv_src,
                                      uint8_t *recv_x, float *recv_scale, int num_sms, bool pow2, uint32_t *status,
                                      cudaStream_t stream) {
    const int64_t recv_rows = cap > 0 ? (int64_t)E * cap : n * k;
    const int sms = device_sm_count();
    if (sms <= 0) return CGL_ECUDA;
    const int use_sms = (num_sms > 0 && num_sms < sms) ? num_sms : sms;
    const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0);
    if (token_layout_fits(n, k, E, R, use_sms))
        return launch_token_kernel<true>(idx, n, k, E, R, cap, vec, x, h, tokens_per_expert, tokens_per_rank, in_rank,
                                         expert_offset, max_count, dst_pos, recv_src, recv_rows, recv_x, recv_scale,
                                         pow2, status, stream);
    const DecodeShape d = decode_shape(n, k, R, use_sms);
    const size_t smem = (rep_smem_words(d.T, E, R) + (size_t)d.T * k) * sizeof(int32_t);
    cudaError_t err;
    switch (d.CH) {
        case 1:
            err = launch_pdl(decode_fused_kernel<1>, dim3((unsigned)d.G), dim3(kThreads), smem, stream, idx, n, k, E,
                             R, cap, d.T, vec, x, h, tokens_per_expert, tokens_per_rank, in_rank, expert_offset,
                             max_count, dst_pos, recv_src, recv_rows, recv_x, recv_scale, (int)pow2, status);
            break;
        case 2:
            err = launch_pdl(decode_fused_kernel<2>, dim3((unsigned)d.G), dim3(kThreads), smem, stream, idx, n, k, E,
                             R, cap, d.T, vec, x, h, tokens_per_expert, tokens_per_rank, in_rank, expert_offset,
                             max_count, dst_pos, recv_src, recv_rows, recv_x, recv_scale, (int)pow2, status);
            break;
        default:
            err = launch_pdl(decode_fused_kernel<4>, dim3((unsigned)d.G), dim3(kThreads), smem, stream, idx, n, k, E,
                             R, cap, d.T, vec, x, h, tokens_per_expert, tokens_per_rank, in_rank, expert_offset,
                             max_count, dst_pos, recv_src, recv_rows, recv_x, recv_scale, (int)pow2, status);
    }
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
