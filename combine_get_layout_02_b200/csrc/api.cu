// The exported C ABI (declared in include/cgl.h): argument checks, then one
// call into the launchers.  Host-visible errors return before any launch.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "launch.h"

namespace cgl {

namespace {

std::mutex g_mu;

struct KernelCache {
    const void *kernel;
    int device;
    size_t smem;         // dynamic shared memory limit set so far
    int ctas_per_sm;     // occupancy at kThreads, 0 = not computed
};
std::vector<KernelCache> g_kernels;
int g_sms[256] = {0};

KernelCache &entry(const void *kernel, int device) {
    for (auto &e : g_kernels)
        if (e.kernel == kernel && e.device == device) return e;
    g_kernels.push_back({kernel, device, 48 * 1024, 0});
    return g_kernels.back();
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int opt_sms(const cgl_opts *o) { return o ? o->num_sms : 0; }
int opt_cap(const cgl_opts *o) { return o ? o->capacity : 0; }
uint32_t opt_flags(const cgl_opts *o) { return o ? o->flags : 0u; }
bool flags_ok(const cgl_opts *o) { return (opt_flags(o) & ~CGL_OPT_UE8M0_SCALES) == 0; }
bool opt_pow2(const cgl_opts *o) { return (opt_flags(o) & CGL_OPT_UE8M0_SCALES) != 0; }
unsigned long long *opt_scratch(const cgl_opts *o) {
    return o ? static_cast<unsigned long long *>(o->scratch) : nullptr;
}

}  // namespace

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 0;
    if (g_sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g_sms[dev] = v;
    }
    return g_sms[dev];
}

bool ensure_smem_attr(const void *kernel, size_t bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    KernelCache &e = entry(kernel, dev);
    if (bytes <= e.smem) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return false;
    e.smem = bytes;
    return true;
}

namespace {
struct OccEntry {
    const void *kernel;
    int device, threads;
    size_t smem;
    int ctas;
};
OccEntry g_occ[64];
int g_occ_n = 0;
}  // namespace

int persistent_grid(const void *kernel, int threads, size_t smem, int target_per_sm, int num_sms_cap,
                    int64_t work) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const int sms = device_sm_count();
    if (sms <= 0) return 0;
    int fit = 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (int i = 0; i < g_occ_n; ++i)
            if (g_occ[i].kernel == kernel && g_occ[i].device == dev && g_occ[i].threads == threads &&
                g_occ[i].smem == smem)
                fit = g_occ[i].ctas;
        if (fit == 0) {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, kernel, threads, smem) != cudaSuccess)
                return 0;
            if (fit < 1) fit = 1;
            if (g_occ_n < 64) g_occ[g_occ_n++] = {kernel, dev, threads, smem, fit};
        }
    }
    int per_sm = target_per_sm < fit ? target_per_sm : fit;
    if (per_sm < 1) per_sm = 1;
    const int use_sms = (num_sms_cap > 0 && num_sms_cap < sms) ? num_sms_cap : sms;
    const int64_t want = (int64_t)use_sms * per_sm;
    return (int)(work < want ? work : want);
}

int copy_grid(const void *kernel, int threads, int64_t work_ctas, int num_sms_cap) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const int sms = device_sm_count();
    if (sms <= 0) return 0;
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        KernelCache &e = entry(kernel, dev);
        if (e.ctas_per_sm == 0) {
            int v = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, threads, 0) != cudaSuccess)
                return 0;
            e.ctas_per_sm = v > 0 ? v : 1;
        }
        per_sm = e.ctas_per_sm;
    }
    const int use_sms = (num_sms_cap > 0 && num_sms_cap < sms) ? num_sms_cap : sms;
    const int64_t cap = (int64_t)use_sms * per_sm;
    return (int)(work_ctas < cap ? work_ctas : cap);
}

}  // namespace cgl

using namespace cgl;

extern "C" {

int cgl_version(void) { return 300; }

const char *cgl_status_string(int s) {
    switch (s) {
        case CGL_OK: return "ok";
        case CGL_EINVAL: return "invalid argument";
        case CGL_EALIGN: return "misaligned pointer";
        case CGL_ERANGE: return "expert id or receive row out of range";
        case CGL_ECAPACITY: return "padded expert capacity exceeded";
        case CGL_ETIMEOUT: return "bounded wait timed out";
        case CGL_ECUDA: return "CUDA runtime error";
        case CGL_ENOTIMPL: return "not implemented";
        default: return "unknown status";
    }
}

static bool layout_sizes_ok(int64_t n, int k, int E, int R) {
    return n >= 0 && k >= 1 && k <= kMaxTopk && E >= 1 && E <= kMaxExperts && R >= 1 && R <= E &&
           E % R == 0 && n * (int64_t)k < ((int64_t)1 << 31);
}

size_t cgl_layout_workspace_bytes(int64_t n, int k, int E, int R) {
    if (!layout_sizes_ok(n, k, E, R)) return 0;
    return layout_workspace_bytes(n, k, E, R);
}

int cgl_layout_kernel_count(int64_t n, int k, int E, int R) {
    if (!layout_sizes_ok(n, k, E, R)) return -1;
    return layout_fused_fits(n, k, E, R) ? 1 : 2;
}

cgl_status cgl_get_layout(const int32_t *topk_idx, int64_t n, int k, int E, int R,
                          const cgl_opts *opts, int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                          uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count,
                          int32_t *dst_pos, int32_t *recv_src, void *workspace,
                          size_t workspace_bytes, uint32_t *status_dev, void *stream) {
    if (!layout_sizes_ok(n, k, E, R) || !flags_ok(opts)) return CGL_EINVAL;
    const int cap = opt_cap(opts);
    if (cap < 0 || (int64_t)E * cap >= ((int64_t)1 << 31)) return CGL_EINVAL;
    const int64_t rows = cap > 0 ? (int64_t)E * cap : n * k;
    if (!tokens_per_expert || !tokens_per_rank || !expert_offset || !max_count || !workspace)
        return CGL_EINVAL;
    if (n > 0 && (!topk_idx || !dst_pos || !is_token_in_rank)) return CGL_EINVAL;
    if (rows > 0 && !recv_src) return CGL_EINVAL;
    if (workspace_bytes < layout_workspace_bytes(n, k, E, R)) return CGL_EINVAL;
    if (!aligned(topk_idx, 4) || !aligned(tokens_per_expert, 4) || !aligned(tokens_per_rank, 4) ||
        !aligned(expert_offset, 4) || !aligned(max_count, 4) || !aligned(dst_pos, 4) ||
        !aligned(recv_src, 4) || !aligned(status_dev, 4) || !aligned(is_token_in_rank, 16) ||
        !aligned(workspace, 16))
        return CGL_EALIGN;
    return launch_layout(topk_idx, n, k, E, R, cap, tokens_per_expert, tokens_per_rank,
                         is_token_in_rank, expert_offset, max_count, dst_pos, recv_src, workspace,
                         status_dev, static_cast<cudaStream_t>(stream));
}

cgl_status cgl_get_rank_layout(const int32_t *topk_idx, int64_t n, int k, int E, int R,
                               const cgl_opts *opts, int32_t *tokens_per_rank, int32_t *rank_offset,
                               int32_t *max_count, int32_t *rank_dst, int32_t *recv_token,
                               void *workspace, size_t workspace_bytes, uint32_t *status_dev,
                               void *stream) {
    if (!layout_sizes_ok(n, k, E, R) || !flags_ok(opts)) return CGL_EINVAL;
    const int cap = opt_cap(opts);
    if (cap < 0 || (int64_t)R * cap >= ((int64_t)1 << 31)) return CGL_EINVAL;
    const int64_t rows = cap > 0 ? (int64_t)R * cap : n * k;
    if (!tokens_per_rank || !rank_offset || !max_count || !workspace) return CGL_EINVAL;
    if (n > 0 && (!topk_idx || !rank_dst)) return CGL_EINVAL;
    if (rows > 0 && !recv_token) return CGL_EINVAL;
    if (workspace_bytes < layout_workspace_bytes(n, k, R, R)) return CGL_EINVAL;
    if (!aligned(topk_idx, 4) || !aligned(tokens_per_rank, 4) || !aligned(rank_offset, 4) ||
        !aligned(max_count, 4) || !aligned(rank_dst, 4) || !aligned(recv_token, 4) ||
        !aligned(status_dev, 4) || !aligned(workspace, 16))
        return CGL_EALIGN;
    return launch_rank_layout(topk_idx, n, k, E, R, cap, tokens_per_rank, rank_offset, max_count,
                              rank_dst, recv_token, workspace, status_dev,
                              static_cast<cudaStream_t>(stream));
}

cgl_status cgl_dispatch_fp8(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                            uint8_t *recv_x, float *recv_scale, int64_t recv_rows,
                            const cgl_opts *opts, uint32_t *status_dev, void *stream) {
    if (n < 0 || h <= 0 || h % 128 != 0 || k < 1 || k > kMaxTopk || recv_rows < 0)
        return CGL_EINVAL;
    if (opt_sms(opts) < 0 || !flags_ok(opts)) return CGL_EINVAL;
    if (n > 0 && (!x || !dst_pos)) return CGL_EINVAL;
    if (n > 0 && recv_rows > 0 && (!recv_x || !recv_scale)) return CGL_EINVAL;
    if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(dst_pos, 4) ||
        !aligned(recv_scale, 4) || !aligned(status_dev, 4) || !aligned(opt_scratch(opts), 8))
        return CGL_EALIGN;
    return launch_dispatch_fp8(x, n, h, k, dst_pos, recv_x, recv_scale, recv_rows, opt_sms(opts), opt_pow2(opts),
                               status_dev, static_cast<cudaStream_t>(stream), opt_scratch(opts));
}

cgl_status cgl_dispatch_bf16(const uint16_t *x, int64_t n, int h, int k, const int32_t *dst_pos,
                             uint16_t *recv_x, int64_t recv_rows, const cgl_opts *opts,
                             uint32_t *status_dev, void *stream) {
    if (n < 0 || h <= 0 || h % 8 != 0 || k < 1 || k > kMaxTopk || recv_rows < 0) return CGL_EINVAL;
    if (opt_sms(opts) < 0 || !flags_ok(opts)) return CGL_EINVAL;
    if (n > 0 && (!x || !dst_pos)) return CGL_EINVAL;
    if (n > 0 && recv_rows > 0 && !recv_x) return CGL_EINVAL;
    if (!aligned(x, 16) || !aligned(recv_x, 16) || !aligned(dst_pos, 4) || !aligned(status_dev, 4) ||
        !aligned(opt_scratch(opts), 8))
        return CGL_EALIGN;
    return launch_dispatch_bf16(x, n, h, k, dst_pos, recv_x, recv_rows, opt_sms(opts), status_dev,
                                static_cast<cudaStream_t>(stream), opt_scratch(opts));
}

cgl_status cgl_combine(const uint16_t *y, int64_t recv_rows, const int32_t *dst_pos,
                       const float *topk_weights, int64_t n, int h, int k, uint16_t *out,
                       const cgl_opts *opts, uint32_t *status_dev, void *stream) {
    if (n < 0 || h <= 0 || h % 8 != 0 || k < 1 || k > kMaxTopk || recv_rows < 0) return CGL_EINVAL;
    if (opt_sms(opts) < 0 || !flags_ok(opts)) return CGL_EINVAL;
    if (n > 0 && (!dst_pos || !topk_weights || !out)) return CGL_EINVAL;
    if (n > 0 && recv_rows > 0 && !y) return CGL_EINVAL;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(dst_pos, 4) ||
        !aligned(topk_weights, 4) || !aligned(status_dev, 4))
        return CGL_EALIGN;
    return launch_combine(y, recv_rows, dst_pos, topk_weights, n, h, k, out, opt_sms(opts),
                          status_dev, static_cast<cudaStream_t>(stream));
}

cgl_status cgl_combine_backward(const uint16_t *grad_out, const uint16_t *y, int64_t recv_rows,
                                const int32_t *dst_pos, const float *topk_weights, int64_t n, int h,
                                int k, uint16_t *grad_y, float *grad_w, const cgl_opts *opts,
                                uint32_t *status_dev, void *stream) {
    if (n < 0 || h <= 0 || h % 16 != 0 || h > 16384 || k < 1 || k > kMaxTopk || recv_rows < 0)
        return CGL_EINVAL;
    if (opt_sms(opts) < 0 || !flags_ok(opts)) return CGL_EINVAL;
    if (n > 0 && (!grad_out || !dst_pos || !topk_weights || !grad_w)) return CGL_EINVAL;
    if (n > 0 && recv_rows > 0 && (!y || !grad_y)) return CGL_EINVAL;
    if (!aligned(grad_out, 16) || !aligned(y, 16) || !aligned(grad_y, 16) || !aligned(dst_pos, 4) ||
        !aligned(topk_weights, 4) || !aligned(grad_w, 4) || !aligned(status_dev, 4))
        return CGL_EALIGN;
    return launch_combine_backward(grad_out, y, recv_rows, dst_pos, topk_weights, n, h, k, grad_y, grad_w,
                                   opt_sms(opts), status_dev, static_cast<cudaStream_t>(stream));
}

cgl_status cgl_decode_dispatch_fp8(const int32_t *topk_idx, int64_t n, int k, int E, int R,
                                   const cgl_opts *opts, const uint16_t *x, int h,
                                   int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                                   uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count,
                                   int32_t *dst_pos, int32_t *recv_src, uint8_t *recv_x,
                                   float *recv_scale, uint32_t *status_dev, void *stream) {
    if (!layout_sizes_ok(n, k, E, R) || h <= 0 || h % 128 != 0 || !flags_ok(opts)) return CGL_EINVAL;
    const int per_block = 1024 / k < 256 ? 1024 / k : 256;   // tokens one layout block holds
    if (n > per_block) return CGL_EINVAL;
    if (decode_fused_smem_bytes(n, k, E, R) > 47 * 1024) return CGL_EINVAL;
    const int cap = opt_cap(opts);
    if (cap < 0 || (int64_t)E * cap >= ((int64_t)1 << 31) || opt_sms(opts) < 0) return CGL_EINVAL;
    const int64_t rows = cap > 0 ? (int64_t)E * cap : n * k;
    if (!tokens_per_expert || !tokens_per_rank || !expert_offset || !max_count) return CGL_EINVAL;
    if (n > 0 && (!topk_idx || !x || !dst_pos || !is_token_in_rank)) return CGL_EINVAL;
    if (rows > 0 && (!recv_src || !recv_x || !recv_scale)) return CGL_EINVAL;
    if (!aligned(topk_idx, 4) || !aligned(x, 16) || !aligned(tokens_per_expert, 4) ||
        !aligned(tokens_per_rank, 4) || !aligned(is_token_in_rank, 16) || !aligned(expert_offset, 4) ||
        !aligned(max_count, 4) || !aligned(dst_pos, 4) || !aligned(recv_src, 4) ||
        !aligned(recv_x, 16) || !aligned(recv_scale, 4) || !aligned(status_dev, 4))
        return CGL_EALIGN;
    return launch_decode_dispatch_fp8(topk_idx, n, k, E, R, cap, x, h, tokens_per_expert, tokens_per_rank,
                                      is_token_in_rank, expert_offset, max_count, dst_pos, recv_src, recv_x,
                                      recv_scale, opt_sms(opts), opt_pow2(opts), status_dev,
                                      static_cast<cudaStream_t>(stream));
}

size_t cgl_layout_dispatch_workspace_bytes(int64_t n, int k, int E, int R) {
    if (!layout_sizes_ok(n, k, E, R)) return 0;
    return layout_dispatch_workspace_bytes(n, k, E, R);
}

int cgl_layout_dispatch_kernel_count(int64_t n, int k, int E, int R, int h, const cgl_opts *opts) {
    if (!layout_sizes_ok(n, k, E, R) || h <= 0 || h % 128 != 0 || opt_sms(opts) < 0) return -1;
    if (layout_dispatch_fused_fits(n, k, E, R, h, opt_sms(opts))) return 1;
    return (layout_fused_fits(n, k, E, R) ? 1 : 2) + 1;
}

cgl_status cgl_layout_dispatch_fp8(const int32_t *topk_idx, int64_t n, int k, int E, int R,
                                   const cgl_opts *opts, const uint16_t *x, int h,
                                   int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                                   uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count,
                                   int32_t *dst_pos, int32_t *recv_src, uint8_t *recv_x, float *recv_scale,
                                   void *workspace, size_t workspace_bytes, uint32_t *status_dev,
                                   void *stream) {
    if (!layout_sizes_ok(n, k, E, R) || h <= 0 || h % 128 != 0 || !flags_ok(opts)) return CGL_EINVAL;
    const int cap = opt_cap(opts);
    if (cap < 0 || (int64_t)E * cap >= ((int64_t)1 << 31) || opt_sms(opts) < 0) return CGL_EINVAL;
    const int64_t rows = cap > 0 ? (int64_t)E * cap : n * k;
    if (!tokens_per_expert || !tokens_per_rank || !expert_offset || !max_count || !workspace)
        return CGL_EINVAL;
    if (n > 0 && (!topk_idx || !x || !dst_pos || !is_token_in_rank)) return CGL_EINVAL;
    if (rows > 0 && (!recv_src || !recv_x || !recv_scale)) return CGL_EINVAL;
    if (workspace_bytes < layout_dispatch_workspace_bytes(n, k, E, R)) return CGL_EINVAL;
    if (!aligned(topk_idx, 4) || !aligned(x, 16) || !aligned(tokens_per_expert, 4) ||
        !aligned(tokens_per_rank, 4) || !aligned(is_token_in_rank, 16) || !aligned(expert_offset, 4) ||
        !aligned(max_count, 4) || !aligned(dst_pos, 4) || !aligned(recv_src, 4) ||
        !aligned(recv_x, 16) || !aligned(recv_scale, 4) || !aligned(status_dev, 4) || !aligned(workspace, 16))
        return CGL_EALIGN;
    return launch_layout_dispatch_fp8(topk_idx, n, k, E, R, cap, x, h, tokens_per_expert, tokens_per_rank,
                                      is_token_in_rank, expert_offset, max_count, dst_pos, recv_src, recv_x,
                                      recv_scale, workspace, opt_sms(opts), opt_pow2(opts), status_dev,
                                      static_cast<cudaStream_t>(stream));
}

cgl_status cgl_selftest_bounded_wait(uint64_t *workspace, int nflags, uint32_t *status_dev, void *stream) {
    if (!workspace || !status_dev || nflags < 1 || nflags > 4096) return CGL_EINVAL;
    if (!aligned(workspace, 8) || !aligned(status_dev, 4)) return CGL_EALIGN;
    return launch_wait_probe(workspace, nflags, status_dev, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
