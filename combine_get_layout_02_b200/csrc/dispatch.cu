// Dispatch: each token's row is read once and written to its k receive rows,
// quantised to FP8 E4M3 with one fp32 scale per 128 values, or copied as BF16.
//
// Pages: FP8 dispatch and BF16 combine are the benchmark settings of DeepEP's
// normal kernels (news article "具体性能方面", brainleap "DeepEP 的性能表现",
// flashmla.org/de); "原生FP8 调度支持" is item 5 of brainleap's key techniques.
// The kernels here copy inside one GPU's HBM instead of over NVLink/RDMA.
// The scale is amax_c / 448 by IEEE division, or with `pow2` the smallest
// power of two 2^e with 448 * 2^e >= amax_c (block_scale in common.cuh).
//
// FP8, hidden <= 16384 (the bulk kernel).  A CTA owns one token at a time
// (persistent over tokens), one thread per 16 hidden values: the thread loads
// its 32 bytes of the row (the next token's 32 bytes are already in flight),
// the 8 lanes of each 128-value block combine their absmax with xor-shuffles,
// and the codes go to a shared-memory row (two buffers, alternating).  One
// thread then hands the row to the TMA engine: k bulk copies, shared ->
// global, each one whole 7168-byte receive row at hidden 7168, so the copies
// leave the SM as long contiguous writes without holding registers.  Before a
// buffer is rewritten, the copies issued from it two tokens earlier must have
// read it (bulk wait_group.read).  One lane of each 128-value block stores its
// fp32 scale.
//
// BF16, hidden <= 8192 and a multiple of 16: the same staging with BF16 rows.
// FP8 above 16384 and BF16 otherwise: one thread per 16 or 8 values of the
// flattened (token, chunk) grid, 16-byte loads and one 16-byte store per copy.  Every
// kernel launches with programmatic dependent launch: blocks start while the
// layout drains and wait (griddepcontrol) before their first global read.
#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxBulkHidden = 16384;    // one thread per 16 values: at most 1024 threads
constexpr int kBulkThreadsPerSM = 1024;  // CTAs per SM of the bulk kernels = this / block size
constexpr int kMaxBulkHiddenBf16 = 8192; // two staged BF16 rows stay within 32 KiB of shared memory

// Dynamic token order: thread 0 of each CTA claims tokens from a 64-bit word,
// one ahead of the token being loaded.  Bits 0-39 count the tokens handed out,
// bits 40-63 the CTAs that have finished: claims and counts are atomics on the
// one word, so its modification order holds every CTA's claims before that
// CTA's count, and the CTA whose count completes the grid can set the word
// back to zero for the next launch with no fence.  A claim's raw value is only
// looked at where it is used (take_claim), so the atomic's round trip overlaps
// the token's copies.  take_claim clamps it to n: a word that did not start at
// zero can at worst leave tokens out, never send a load or a copy outside the
// batch.  A launch that starts from zero hands out at most n + 2 G tokens (no
// CTA makes more than two claims past n); a claim of n + 3 G or more means the
// scratch was not zero, and sets `bad` (reported as kErrRange).
constexpr int kDoneShift = 40;
constexpr unsigned long long kClaimMask = (1ull << kDoneShift) - 1;

__device__ __forceinline__ int64_t take_claim(unsigned long long word, int64_t n, bool &bad) {
    const unsigned long long v = word & kClaimMask;
    if (v >= (unsigned long long)n + 3ull * gridDim.x) bad = true;
    return v < (unsigned long long)n ? (int64_t)v : n;
}

// After the CTA's last claim: count it finished; the last CTA resets the word.
__device__ __forceinline__ void claims_done(unsigned long long *claim) {
    const unsigned long long old = atomicAdd(claim, 1ull << kDoneShift);
    if ((old >> kDoneShift) == (unsigned long long)gridDim.x - 1) *claim = 0;
}

__global__ void __launch_bounds__(1024)
dispatch_fp8_bulk_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                         const int32_t *__restrict__ dst_pos, uint8_t *__restrict__ recv_x,
                         float *__restrict__ recv_scale, int64_t recv_rows, int pow2,
                         unsigned long long *claim, uint32_t *status) {
    extern __shared__ __align__(128) uint8_t rows_smem[];   // [2][h] staged code rows
    __shared__ int64_t s_next[2];      // claimed tokens (dynamic order)
    griddep_wait();                   // dst_pos (and x) may come from the kernels just before
    const int chunks = h >> 4, nblk = h >> 7;
    const int c = threadIdx.x;        // this thread's 16 values
    const bool active = c < chunks;   // only lanes of the last warp can be idle
    const bool scale_lane = active && (c & 7) == 0;
    bool bad = false;
    int buf = 0;
    // Token order.  Static: CTA b takes tokens b, b + G, ...  Dynamic (claim
    // != null: the claim word above, zero at launch): thread 0 claims the
    // CTA's tokens from the counter, one token ahead of the
    // one being loaded, so CTAs on SMs that stream faster take more tokens (on
    // B200 some SMs, by where they sit, are consistently slower).
    int64_t t = blockIdx.x, tn = t + gridDim.x;
    unsigned long long pend = (unsigned long long)n;   // thread 0: the claim in flight (raw)
    if (claim != nullptr) {
        if (threadIdx.x == 0) {
            s_next[0] = take_claim(atomicAdd(claim, 1ull), n, bad);
            s_next[1] = take_claim(atomicAdd(claim, 1ull), n, bad);
        }
        __syncthreads();
        t = s_next[0];
        tn = t < n ? s_next[1] : n;
        if (threadIdx.x == 0 && tn < n) pend = atomicAdd(claim, 1ull);
    }
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (t < n && active) {
        a = ld_nc_v4(x + t * h + (int64_t)c * 16);
        b = ld_nc_v4(x + t * h + (int64_t)c * 16 + 8);
    }
    for (int it = 0; t < n; buf ^= 1, ++it) {
        uint4 an = make_uint4(0, 0, 0, 0), bn = an;   // the next token's chunk, in flight
        if (tn < n && active) {
            an = ld_nc_v4(x + tn * h + (int64_t)c * 16);
            bn = ld_nc_v4(x + tn * h + (int64_t)c * 16 + 8);
        }
        float m = absmax16(a, b);
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        const float amax_c = fmaxf(m, 1e-4f);
        float scale, inv;
        block_scale(amax_c, pow2 != 0, scale, inv);
        const uint4 q = quant16(a, b, inv);
        uint8_t *row = rows_smem + buf * h;
        if (threadIdx.x == 0) {
            bulk_wait_read<1>();   // copies from two tokens ago have read `row`
            if (claim != nullptr) s_next[it & 1] = take_claim(pend, n, bad);
        }
        __syncthreads();
        if (active) *reinterpret_cast<uint4 *>(row + c * 16) = q;
        fence_proxy_async();
        __syncthreads();
        int64_t tnn = tn + gridDim.x;   // the token after the next one
        if (claim != nullptr) {
            tnn = tn < n ? s_next[it & 1] : n;
            if (threadIdx.x == 0) pend = tnn < n ? atomicAdd(claim, 1ull) : (unsigned long long)n;
        }
        const int32_t *dp = dst_pos + t * k;
        if (threadIdx.x == 0) {
            for (int j = 0; j < k; ++j) {
                const int32_t r = __ldg(dp + j);
                if (r < 0) continue;
                if (r >= recv_rows) { bad = true; continue; }
                bulk_store(recv_x + (int64_t)r * h, row, (uint32_t)h);
            }
            bulk_commit();
        }
        if (scale_lane) {
            for (int j = 0; j < k; ++j) {
                const int32_t r = __ldg(dp + j);
                if (r >= 0 && r < recv_rows) recv_scale[(int64_t)r * nblk + (c >> 3)] = scale;
            }
        }
        a = an;
        b = bn;
        t = tn;
        tn = tnn;
    }
    if (threadIdx.x == 0) {
        if (claim != nullptr) claims_done(claim);   // before the wait, which hides the atomic
        bulk_wait_all();
    }
    if (bad) report(status, kErrRange);
}

__global__ void __launch_bounds__(kThreads)
dispatch_fp8_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                    const int32_t *__restrict__ dst_pos, uint8_t *__restrict__ recv_x,
                    float *__restrict__ recv_scale, int64_t recv_rows, int pow2, uint32_t *status) {
    griddep_wait();                   // dst_pos (and x) may come from the kernels just before
    const int chunks = h >> 4;        // 16 values per thread
    const int nblk = h >> 7;          // 128-value scale blocks per row
    const int64_t total = n * chunks; // a multiple of 8: scale groups never straddle
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    bool bad = false;
    // warp-uniform loop: all 32 lanes take part in every shuffle
    for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < total;
         base += stride) {
        const int64_t g = base + lane;
        const bool active = g < total;
        int64_t t = 0;
        int c = 0;
        uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
        if (active) {
            t = g / chunks;
            c = (int)(g - t * chunks);
            const uint16_t *src = x + t * h + (int64_t)c * 16;
            a = ld_nc_v4(src);
            b = ld_nc_v4(src + 8);
        }
        float v[16];
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = bf16_lo(wv[i]);
            v[2 * i + 1] = bf16_hi(wv[i]);
        }
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        if (!active) continue;
        const float amax_c = fmaxf(m, 1e-4f);
        float scale, inv;
        block_scale(amax_c, pow2 != 0, scale, inv);
        uint32_t qw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = cvt_e4m3x2(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv));
            const uint32_t hi = cvt_e4m3x2(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv));
            qw[i] = lo | (hi << 16);
        }
        const uint4 q = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        const int32_t *dp = dst_pos + t * k;
        const bool scale_lane = (c & 7) == 0;
        for (int j = 0; j < k; ++j) {
            const int32_t row = __ldg(dp + j);
            if (row < 0) continue;
            if (row >= recv_rows) { bad = true; continue; }
            st_cs_v4(recv_x + (int64_t)row * h + (int64_t)c * 16, q);
            if (scale_lane) recv_scale[(int64_t)row * nblk + (c >> 3)] = scale;
        }
    }
    if (bad) report(status, kErrRange);
}

// BF16 rows through the same staging: one thread per 16 values, k bulk copies per token.
__global__ void __launch_bounds__(1024)
dispatch_bf16_bulk_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                          const int32_t *__restrict__ dst_pos, uint16_t *__restrict__ recv_x,
                          int64_t recv_rows, unsigned long long *claim, uint32_t *status) {
    extern __shared__ __align__(128) uint8_t rows_smem[];   // [2][2h] staged rows
    __shared__ int64_t s_next[2];      // claimed tokens (dynamic order, as in the FP8 kernel)
    griddep_wait();
    const int chunks = h >> 4;
    const int c = threadIdx.x;
    const bool active = c < chunks;
    const uint32_t row_bytes = (uint32_t)h * 2;
    bool bad = false;
    int buf = 0;
    int64_t t = blockIdx.x, tn = t + gridDim.x;
    unsigned long long pend = (unsigned long long)n;   // thread 0: the claim in flight (raw)
    if (claim != nullptr) {
        if (threadIdx.x == 0) {
            s_next[0] = take_claim(atomicAdd(claim, 1ull), n, bad);
            s_next[1] = take_claim(atomicAdd(claim, 1ull), n, bad);
        }
        __syncthreads();
        t = s_next[0];
        tn = t < n ? s_next[1] : n;
        if (threadIdx.x == 0 && tn < n) pend = atomicAdd(claim, 1ull);
    }
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (t < n && active) {
        a = ld_nc_v4(x + t * h + (int64_t)c * 16);
        b = ld_nc_v4(x + t * h + (int64_t)c * 16 + 8);
    }
    for (int it = 0; t < n; buf ^= 1, ++it) {
        uint4 an = make_uint4(0, 0, 0, 0), bn = an;   // the next token's chunk, in flight
        if (tn < n && active) {
            an = ld_nc_v4(x + tn * h + (int64_t)c * 16);
            bn = ld_nc_v4(x + tn * h + (int64_t)c * 16 + 8);
        }
        uint8_t *row = rows_smem + (size_t)buf * row_bytes;
        if (threadIdx.x == 0) {
            bulk_wait_read<1>();
            if (claim != nullptr) s_next[it & 1] = take_claim(pend, n, bad);
        }
        __syncthreads();
        if (active) {
            reinterpret_cast<uint4 *>(row)[2 * c] = a;
            reinterpret_cast<uint4 *>(row)[2 * c + 1] = b;
        }
        fence_proxy_async();
        __syncthreads();
        int64_t tnn = tn + gridDim.x;   // the token after the next one
        if (claim != nullptr) {
            tnn = tn < n ? s_next[it & 1] : n;
            if (threadIdx.x == 0) pend = tnn < n ? atomicAdd(claim, 1ull) : (unsigned long long)n;
        }
        if (threadIdx.x == 0) {
            const int32_t *dp = dst_pos + t * k;
            for (int j = 0; j < k; ++j) {
                const int32_t r = __ldg(dp + j);
                if (r < 0) continue;
                if (r >= recv_rows) { bad = true; continue; }
                bulk_store(recv_x + (int64_t)r * h, row, row_bytes);
            }
            bulk_commit();
        }
        a = an;
        b = bn;
        t = tn;
        tn = tnn;
    }
    if (threadIdx.x == 0) {
        if (claim != nullptr) claims_done(claim);   // before the wait, which hides the atomic
        bulk_wait_all();
    }
    if (bad) report(status, kErrRange);
}

__global__ void __launch_bounds__(kThreads)
dispatch_bf16_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                     const int32_t *__restrict__ dst_pos, uint16_t *__restrict__ recv_x,
                     int64_t recv_rows, uint32_t *status) {
    griddep_wait();
    const int chunks = h >> 3;        // 8 values per thread
    const int64_t total = n * chunks;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    bool bad = false;
    for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < total; g += stride) {
        const int64_t t = g / chunks;
        const int c = (int)(g - t * chunks);
        const uint4 a = ld_nc_v4(x + t * h + (int64_t)c * 8);
        const int32_t *dp = dst_pos + t * k;
        for (int j = 0; j < k; ++j) {
            const int32_t row = __ldg(dp + j);
            if (row < 0) continue;
            if (row >= recv_rows) { bad = true; continue; }
            st_cs_v4(recv_x + (int64_t)row * h + (int64_t)c * 8, a);
        }
    }
    if (bad) report(status, kErrRange);
}

}  // namespace

cgl_status launch_dispatch_fp8(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                               uint8_t *recv_x, float *recv_scale, int64_t recv_rows,
                               int num_sms, bool pow2, uint32_t *status, cudaStream_t stream,
                               unsigned long long *claim) {
    if (n * (h / 16) == 0) return CGL_OK;
    if (h <= kMaxBulkHidden) {
        const int threads = (h / 16 + 31) / 32 * 32;
        const int grid = persistent_grid((const void *)dispatch_fp8_bulk_kernel, threads, (size_t)2 * h,
                                         kBulkThreadsPerSM / threads, num_sms, n);
        if (grid <= 0) return CGL_ECUDA;
        if (n <= grid) claim = nullptr;   // one token per CTA either way: the counter would only add latency
        const cudaError_t err = launch_pdl(dispatch_fp8_bulk_kernel, dim3(grid), dim3(threads),
                                           (size_t)2 * h, stream, x, n, h, k, dst_pos, recv_x,
                                           recv_scale, recv_rows, (int)pow2, claim, status);
        return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
    }
    const int64_t work = n * (h / 16);
    const int grid = copy_grid((const void *)dispatch_fp8_kernel, kThreads,
                               (work + kThreads - 1) / kThreads, num_sms);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(dispatch_fp8_kernel, dim3(grid), dim3(kThreads), 0, stream, x, n, h,
                                       k, dst_pos, recv_x, recv_scale, recv_rows, (int)pow2, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

cgl_status launch_dispatch_bf16(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                                uint16_t *recv_x, int64_t recv_rows, int num_sms, uint32_t *status,
                                cudaStream_t stream, unsigned long long *claim) {
    if (n * (h / 8) == 0) return CGL_OK;
    if (h % 16 == 0 && h <= kMaxBulkHiddenBf16) {
        const int threads = (h / 16 + 31) / 32 * 32;
        const int grid = persistent_grid((const void *)dispatch_bf16_bulk_kernel, threads, (size_t)4 * h,
                                         kBulkThreadsPerSM / threads, num_sms, n);
        if (grid <= 0) return CGL_ECUDA;
        if (n <= grid) claim = nullptr;   // one token per CTA either way
        const cudaError_t err = launch_pdl(dispatch_bf16_bulk_kernel, dim3(grid), dim3(threads),
                                           (size_t)4 * h, stream, x, n, h, k, dst_pos, recv_x,
                                           recv_rows, claim, status);
        return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
    }
    const int64_t work = n * (h / 8);
    const int grid = copy_grid((const void *)dispatch_bf16_kernel, kThreads,
                               (work + kThreads - 1) / kThreads, num_sms);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(dispatch_bf16_kernel, dim3(grid), dim3(kThreads), 0, stream, x, n,
                                       h, k, dst_pos, recv_x, recv_rows, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
