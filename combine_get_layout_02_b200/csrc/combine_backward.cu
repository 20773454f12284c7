// Combine backward: for out[t] = sum_j w[t,j] * y[dst_pos[t,j]] and an output
// gradient g = dL/dout,
//   grad_y[dst_pos[t,j], :] = bf16(w[t,j] * g[t, :])      (one fp32 product, RNE)
//   grad_w[t, j]            = <g[t, :], y[dst_pos[t,j], :]> (fp32)
//
// Pages: combine accumulates the experts' outputs (brainleap "Day2 DeepEP",
// "All-to-All通信"); its gradient is the training-side counterpart.
//
// Work unit: a CTA owns one token at a time (persistent over tokens), one
// thread per 16 hidden values (every 512th chunk when the row is longer).  Per
// batch of 4 slots a thread loads its 32 bytes of g and of each slot's y row
// (all loads in flight before any math), writes
// the 4 scaled gradient chunks with 16-byte stores and keeps 4 partial dot
// products (fused multiply-adds over its values in order).  Batches of 4 keep
// the kernel at 64 registers, so two CTAs share an SM and one's loads cover
// the other's block reduction (batches of 8 needed 117 registers: one CTA
// per SM, idle HBM during every reduction).  The block then
// reduces the partial dots with xor-shuffles and one pass over the warps in
// warp order, so grad_w does not depend on timing.  Launches use programmatic
// dependent launch.
#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kBatch = 4;                // slots whose rows are loaded together
constexpr int kThreadsPerSM = 1024;      // CTAs per SM = this / block size (at least 1)
constexpr int kMaxThreads = 512;         // larger rows loop: each thread takes every 512th chunk

__global__ void __launch_bounds__(kMaxThreads, 2)
combine_backward_kernel(const uint16_t *__restrict__ g, const uint16_t *__restrict__ y, int64_t recv_rows,
                        const int32_t *__restrict__ dst_pos, const float *__restrict__ w, int64_t n, int h,
                        int k, uint16_t *__restrict__ grad_y, float *__restrict__ grad_w, uint32_t *status) {
    __shared__ float red[kMaxThreads / 32][kBatch];   // per-warp partial dots of one batch
    griddep_wait();
    const int chunks = h >> 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    bool bad = false;
    for (int64_t t = blockIdx.x; t < n; t += gridDim.x) {
        const int32_t *dp = dst_pos + t * k;
        const float *wp = w + t * k;
        for (int j0 = 0; j0 < k; j0 += kBatch) {
            int32_t rows[kBatch];
            float wt[kBatch], part[kBatch];
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                const int j = j0 + jj;
                rows[jj] = -1;
                wt[jj] = 0.0f;
                part[jj] = 0.0f;
                if (j < k) {
                    const int32_t r = __ldg(dp + j);
                    if (r >= 0 && r < recv_rows) {
                        rows[jj] = r;
                        wt[jj] = __ldg(wp + j);
                    } else if (r >= recv_rows) {
                        bad = true;
                    }
                }
            }
            for (int c = tid; c < chunks; c += blockDim.x) {
                const uint16_t *gs = g + t * h + (int64_t)c * 16;
                const uint4 ga = ld_nc_v4(gs), gb = ld_nc_v4(gs + 8);
                uint4 ya[kBatch], yb[kBatch];
#pragma unroll
                for (int jj = 0; jj < kBatch; ++jj) {
                    ya[jj] = make_uint4(0, 0, 0, 0);
                    yb[jj] = ya[jj];
                    if (rows[jj] >= 0) {
                        const uint16_t *ys = y + (int64_t)rows[jj] * h + (int64_t)c * 16;
                        ya[jj] = ld_nc_v4(ys);
                        yb[jj] = ld_nc_v4(ys + 8);
                    }
                }
                float gv[16];
                const uint32_t gw[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    gv[2 * i] = bf16_lo(gw[i]);
                    gv[2 * i + 1] = bf16_hi(gw[i]);
                }
#pragma unroll
                for (int jj = 0; jj < kBatch; ++jj) {
                    if (rows[jj] < 0) continue;
                    const uint32_t yw[8] = {ya[jj].x, ya[jj].y, ya[jj].z, ya[jj].w,
                                            yb[jj].x, yb[jj].y, yb[jj].z, yb[jj].w};
                    float d = part[jj];
                    uint32_t o[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        d = fmaf(gv[2 * i], bf16_lo(yw[i]), d);
                        d = fmaf(gv[2 * i + 1], bf16_hi(yw[i]), d);
                        o[i] = cvt_bf16x2(__fmul_rn(wt[jj], gv[2 * i]), __fmul_rn(wt[jj], gv[2 * i + 1]));
                    }
                    part[jj] = d;
                    uint16_t *dst = grad_y + (int64_t)rows[jj] * h + (int64_t)c * 16;
                    st_cs_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
                    st_cs_v4(dst + 8, make_uint4(o[4], o[5], o[6], o[7]));
                }
            }
            // block reduction of the partial dots: shuffles, then warps in order
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                float v = part[jj];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (lane == 0) red[warp][jj] = v;
            }
            __syncthreads();
            if (tid < kBatch && j0 + tid < k) {
                const int32_t r = __ldg(dp + j0 + tid);
                float s = 0.0f;
                for (int wi = 0; wi < nwarps; ++wi) s += red[wi][tid];
                grad_w[t * k + j0 + tid] = (r >= 0 && r < recv_rows) ? s : 0.0f;
            }
            __syncthreads();
        }
    }
    if (bad) report(status, kErrRange);
}

}  // namespace

cgl_status launch_combine_backward(const uint16_t *g, const uint16_t *y, int64_t recv_rows,
                                   const int32_t *dst_pos, const float *w, int64_t n, int h, int k,
                                   uint16_t *grad_y, float *grad_w, int num_sms, uint32_t *status,
                                   cudaStream_t stream) {
    if (n == 0) return CGL_OK;
    int threads = (h / 16 + 31) / 32 * 32;
    if (threads > kMaxThreads) threads = kMaxThreads;
    const int grid = persistent_grid((const void *)combine_backward_kernel, threads, 0,
                                     kThreadsPerSM / threads, num_sms, n);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(combine_backward_kernel, dim3(grid), dim3(threads), 0, stream, g, y,
                                       recv_rows, dst_pos, w, n, h, k, grad_y, grad_w, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
