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

// Grid for a grid-stride copy kernel: enough CTAs for `work_ctas`, capped at
// (SMs in use) x (resident CTAs per SM).
int copy_grid(const void *kernel, int threads, int64_t work_ctas, int num_sms_cap);

size_t layout_workspace_bytes(int64_t n, int E, int R);

// Dynamic shared memory of the layout assign kernel per block (bytes).
size_t layout_assign_smem_bytes(int E, int k);

cgl_status launch_layout(const int32_t *idx, int64_t n, int k, int E, int R, int cap,
                         int32_t *tokens_per_expert, int32_t *tokens_per_rank, uint8_t *in_rank,
                         int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                         int32_t *recv_src, void *ws, uint32_t *status, cudaStream_t stream);

cgl_status launch_dispatch_fp8(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                               uint8_t *recv_x, float *recv_scale, int64_t recv_rows,
                               int num_sms, uint32_t *status, cudaStream_t stream);

cgl_status launch_dispatch_bf16(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                                uint16_t *recv_x, int64_t recv_rows, int num_sms, uint32_t *status,
                                cudaStream_t stream);

cgl_status launch_combine(const uint16_t *y, int64_t recv_rows, const int32_t *dst_pos,
                          const float *w, int64_t n, int h, int k, uint16_t *out, int num_sms,
                          uint32_t *status, cudaStream_t stream);

}  // namespace cgl
