// Dispatch: each token's row is read once and written to its k receive rows,
// quantised to FP8 E4M3 with one fp32 scale per 128 values, or copied as BF16.
//
// Pages: FP8 dispatch and BF16 combine are the benchmark settings of DeepEP's
// normal kernels (news article "具体性能方面", brainleap "DeepEP 的性能表现",
// flashmla.org/de); "原生FP8 调度支持" is item 5 of brainleap's key techniques.
// The kernels here copy inside one GPU's HBM instead of over NVLink/RDMA.
//
// Work unit: one thread owns 16 consecutive hidden values of one token (FP8:
// two 16-byte loads in, one 16-byte store per copy out) or 8 values (BF16: one
// 16-byte load, one 16-byte store per copy).  Threads are numbered over the
// flattened (token, chunk) grid, so a warp reads 512 or 1024 contiguous bytes
// and every store of a warp covers 512 contiguous bytes of one receive row.
// For FP8 a 128-value scale block is 8 adjacent lanes; their absmax is
// combined with three xor-shuffles.  The grid is a multiple of the resident
// CTAs per SM and loops grid-stride.  Launches use programmatic dependent
// launch: blocks start while the layout kernels drain and wait (griddepcontrol)
// before their first global read.
#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
dispatch_fp8_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                    const int32_t *__restrict__ dst_pos, uint8_t *__restrict__ recv_x,
                    float *__restrict__ recv_scale, int64_t recv_rows, uint32_t *status) {
    griddep_launch_dependents();
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
        const float scale = __fdiv_rn(amax_c, 448.0f);
        const float inv = __fdiv_rn(448.0f, amax_c);
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

__global__ void __launch_bounds__(kThreads)
dispatch_bf16_kernel(const uint16_t *__restrict__ x, int64_t n, int h, int k,
                     const int32_t *__restrict__ dst_pos, uint16_t *__restrict__ recv_x,
                     int64_t recv_rows, uint32_t *status) {
    griddep_launch_dependents();
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
                               int num_sms, uint32_t *status, cudaStream_t stream) {
    const int64_t work = n * (h / 16);
    if (work == 0) return CGL_OK;
    const int grid = copy_grid((const void *)dispatch_fp8_kernel, kThreads,
                               (work + kThreads - 1) / kThreads, num_sms);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(dispatch_fp8_kernel, dim3(grid), dim3(kThreads), 0, stream, x, n, h,
                                       k, dst_pos, recv_x, recv_scale, recv_rows, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

cgl_status launch_dispatch_bf16(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                                uint16_t *recv_x, int64_t recv_rows, int num_sms, uint32_t *status,
                                cudaStream_t stream) {
    const int64_t work = n * (h / 8);
    if (work == 0) return CGL_OK;
    const int grid = copy_grid((const void *)dispatch_bf16_kernel, kThreads,
                               (work + kThreads - 1) / kThreads, num_sms);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(dispatch_bf16_kernel, dim3(grid), dim3(kThreads), 0, stream, x, n,
                                       h, k, dst_pos, recv_x, recv_rows, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
