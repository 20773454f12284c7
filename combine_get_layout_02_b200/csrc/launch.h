// Internal launchers behind the C ABI (not exported).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "cgl.h"

namespace cgl {

// Raise a kernel's dynamic shared-memory limit once per device; false on error.
bool ensure_smem_attr(const void *kernel, size_t bytes);

// SMs on the current device (cached per device); 0 on error.
int device_sm_count();

// Grid for a persistent kernel (CTAs loop over `work` items): SMs in use x
// min(target CTAs per SM, CTAs per SM that fit), at most `work`; 0 on error.
int persistent_grid(const void *kernel, int threads, size_t smem, int target_per_sm, int num_sms_cap,
                    int64_t work);

// Grid for a grid-stride copy kernel: enough CTAs for `work_ctas`, capped at
// (SMs in use) x (resident CTAs per SM).
int copy_grid(const void *kernel, int threads, int64_t work_ctas, int num_sms_cap);

// Launch `kernel` with programmatic stream serialisation: it may start while
// the previous kernel in the stream is finishing, and must griddep_wait()
// before reading anything that kernel (or an earlier one) wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

size_t layout_workspace_bytes(int64_t n, int k, int E, int R);

// True if some layout kernel for these sizes needs more shared memory than a
// kernel gets without raising its attribute (host-side bookkeeping on first use).
bool layout_needs_smem_optin(int E, int R, int k);

// True if the layout for these sizes runs as one cooperative kernel on the current device.
bool layout_fused_fits(int64_t n, int k, int E, int R);

cgl_status launch_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                         int32_t *tokens_per_expert, int32_t *tokens_per_rank, uint8_t *in_rank,
                         int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                         int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream);

// Per-rank layout: keys are destination ranks (one row per token and rank).
cgl_status launch_rank_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                              int32_t *tokens_per_rank, int32_t *rank_offset, int32_t *max_count,
                              int32_t *rank_dst, int32_t *recv_token, void *ws, uint32_t *status,
                              cudaStream_t stream);

// pow2: power-of-two (UE8M0) scales instead of amax_c / 448 (cgl_opts.flags).
// claim: null (static token order), or two 64-bit words that are zero when
// the kernel starts (a token counter the CTAs claim from, and a count of
// finished CTAs); the last CTA to finish zeroes both again.
cgl_status launch_dispatch_fp8(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                               uint8_t *recv_x, float *recv_scale, int64_t recv_rows,
                               int num_sms, bool pow2, uint32_t *status, cudaStream_t stream,
                               unsigned long long *claim = nullptr);

cgl_status launch_dispatch_bf16(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                                uint16_t *recv_x, int64_t recv_rows, int num_sms, uint32_t *status,
                                cudaStream_t stream, unsigned long long *claim = nullptr);

cgl_status launch_combine(const uint16_t *y, int64_t recv_rows, const int32_t *dst_pos,
                          const float *w, int64_t n, int h, int k, uint16_t *out, int num_sms,
                          uint32_t *status, cudaStream_t stream);

// One block running the layout's bounded inter-block wait, with its exit path
// (generation advance), on a workspace header whose flags hold no tag it waits for.
cgl_status launch_wait_probe(uint64_t *ws, int nflags, uint32_t *status, cudaStream_t stream);

// Dynamic shared memory of the fused decode kernel (bytes).
size_t decode_fused_smem_bytes(int64_t n, int k, int E, int R);

cgl_status launch_decode_dispatch_fp8(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                                      const uint16_t *x, int h, int32_t *tokens_per_expert,
                                      int32_t *tokens_per_rank, uint8_t *in_rank, int32_t *expert_offset,
                                      int32_t *max_count, int32_t *dst_pos, int32_t *recv_src,
                                      uint8_t *recv_x, float *recv_scale, int num_sms, bool pow2,
                                      uint32_t *status, cudaStream_t stream);

// Fused layout + FP8 dispatch (one cooperative launch when it applies, else
// the layout and the dispatch kernels in turn).
size_t layout_dispatch_workspace_bytes(int64_t n, int k, int E, int R);
bool layout_dispatch_fused_fits(int64_t n, int k, int E, int R, int h, int num_sms);
cgl_status launch_layout_dispatch_fp8(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                                      const uint16_t *x, int h, int32_t *tokens_per_expert,
                                      int32_t *tokens_per_rank, uint8_t *in_rank, int32_t *expert_offset,
                                      int32_t *max_count, int32_t *dst_pos, int32_t *recv_src, uint8_t *recv_x,
                                      float *recv_scale, void *ws, int num_sms, bool pow2, uint32_t *status,
                                      cudaStream_t stream);

cgl_status launch_combine_backward(const uint16_t *g, const uint16_t *y, int64_t recv_rows,
                                   const int32_t *dst_pos, const float *w, int64_t n, int h, int k,
                                   uint16_t *grad_y, float *grad_w, int num_sms, uint32_t *status,
                                   cudaStream_t stream);

}  // namespace cgl
