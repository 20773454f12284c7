// cgl_get_layout_noalloc: the dispatch layout for callers that cannot allocate
// device memory.
//
// cgl_get_layout needs a few tens of KiB of device scratch (per-block expert
// and rank histograms) that its caller allocates.  Some callers cannot do
// that: hosts that hand the library only pre-planned input and output buffers
// and own every other byte of device memory (engine plugins, serving runtimes
// with a fixed memory plan), callers that must not add the device-wide
// synchronisation cudaFree implies, and foreign-language callers that reach
// only this C ABI and have no CUDA allocator.  For them the scratch lives in a
// file-scope device array of fixed size, which every GPU that loads this
// library holds until the process exits.
//
// Set-up: the first call on a device, with that device current, looks up the
// array's device address with cudaGetSymbolAddress and caches it for that
// device; host code must not pass the array's name itself to a kernel (on the
// host it only stands in for the symbol).  That first call should come before
// any stream capture.
//
// Every call shares the one array and it keeps whatever the last call left in
// it.  Nothing in it needs to start at zero: the count kernel overwrites every
// histogram word the assign kernel later reads.  Calls whose work overlaps on
// the GPU (different streams, or different host threads on the same device)
// race on the array and must be serialised by the caller.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = CGL_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_layout_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device; nullptr on error.
void *scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" cgl_status cgl_get_layout_noalloc(
    const int32_t *topk_idx, int64_t num_tokens, int num_topk, int num_experts, int num_ranks,
    const cgl_opts *opts, int32_t *tokens_per_expert, int32_t *tokens_per_rank,
    uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
    int32_t *recv_src, uint32_t *status_dev, void *stream) {
    const size_t need = cgl_layout_workspace_bytes(num_tokens, num_topk, num_experts, num_ranks);
    if (need == 0 || need > kScratchBytes) return CGL_EINVAL;
    // stay within the default 48 KiB of shared memory per block, so that no
    // launch here has to raise a kernel attribute first
    if (cgl::layout_needs_smem_optin(num_experts, num_ranks, num_topk)) return CGL_EINVAL;
    void *scratch = scratch_on_current_device();
    if (scratch == nullptr) return CGL_ECUDA;
    return cgl_get_layout(topk_idx, num_tokens, num_topk, num_experts, num_ranks, opts,
                          tokens_per_expert, tokens_per_rank, is_token_in_rank, expert_offset,
                          max_count, dst_pos, recv_src, scratch, kScratchBytes, status_dev, stream);
}
