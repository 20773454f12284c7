// Combine: gather each token's k expert-output rows and reduce them with the
// top-k weights, in slot order, in fp32, into one BF16 row.
//
// Pages: combine merges the experts' outputs and accumulates (brainleap "Day2
// DeepEP", "All-to-All通信", the combine bullet); BF16 combine is the
// benchmark setting (news article "具体性能方面", flashmla.org/de).  Here the
// k rows are read from this GPU's HBM instead of received over NVLink/RDMA.
//
// Work unit: one thread owns 8 consecutive hidden values of one token.  It
// issues the loads of up to 8 slots before it adds anything (8 x 16 bytes in
// flight per thread), then accumulates acc = acc + w_j * y_j with separate
// round-to-nearest multiply and add (no contraction to FMA), j ascending,
// and stores one 16-byte BF16 vector.  A warp reads 512 contiguous bytes of
// each of the token's k rows and writes 512 contiguous output bytes.  The
// launch uses programmatic dependent launch (blocks wait in griddepcontrol
// before their first global read).
#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;   // slots whose loads are in flight together

__global__ void __launch_bounds__(kThreads)
combine_kernel(const uint16_t *__restrict__ y, int64_t recv_rows,
               const int32_t *__restrict__ dst_pos, const float *__restrict__ w, int64_t n, int h,
               int k, uint16_t *__restrict__ out, uint32_t *status) {
    griddep_wait();                   // y and dst_pos may come from the kernels just before
    const int chunks = h >> 3;
    const int64_t total = n * chunks;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    bool bad = false;
    for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < total; g += stride) {
        const int64_t t = g / chunks;
        const int c = (int)(g - t * chunks);
        const int32_t *dp = dst_pos + t * k;
        const float *wp = w + t * k;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += kBatch) {
            uint4 val[kBatch];
            float wt[kBatch];
            bool use[kBatch];
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                const int j = j0 + jj;
                use[jj] = false;
                wt[jj] = 0.0f;
                val[jj] = make_uint4(0, 0, 0, 0);
                if (j < k) {
                    const int32_t row = __ldg(dp + j);
                    if (row >= 0 && row < recv_rows) {
                        use[jj] = true;
                        wt[jj] = __ldg(wp + j);
                        val[jj] = ld_nc_v4(y + (int64_t)row * h + (int64_t)c * 8);
                    } else if (row >= recv_rows) {
                        bad = true;
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < kBatch; ++jj) {
                if (!use[jj]) continue;
                const uint32_t wv[4] = {val[jj].x, val[jj].y, val[jj].z, val[jj].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wt[jj], bf16_lo(wv[i])));
                    acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wt[jj], bf16_hi(wv[i])));
                }
            }
        }
        const uint4 o = make_uint4(cvt_bf16x2(acc[0], acc[1]), cvt_bf16x2(acc[2], acc[3]),
                                   cvt_bf16x2(acc[4], acc[5]), cvt_bf16x2(acc[6], acc[7]));
        st_cs_v4(out + t * h + (int64_t)c * 8, o);
    }
    if (bad) report(status, kErrRange);
}

}  // namespace

cgl_status launch_combine(const uint16_t *y, int64_t recv_rows, const int32_t *dst_pos,
                          const float *w, int64_t n, int h, int k, uint16_t *out, int num_sms,
                          uint32_t *status, cudaStream_t stream) {
    const int64_t work = n * (h / 8);
    if (work == 0) return CGL_OK;
    const int grid = copy_grid((const void *)combine_kernel, kThreads,
                               (work + kThreads - 1) / kThreads, num_sms);
    if (grid <= 0) return CGL_ECUDA;
    const cudaError_t err = launch_pdl(combine_kernel, dim3(grid), dim3(kThreads), 0, stream, y, recv_rows,
                                       dst_pos, w, n, h, k, out, status);
    return err == cudaSuccess ? CGL_OK : CGL_ECUDA;
}

}  // namespace cgl
