/*
 * cgl.h -- C ABI of the single-GPU MoE layout / dispatch / combine library
 * (libcgl.so, CUDA kernels for B200, sm_100a).
 *
 * What the calls compute.  The DeepEP pages describe all-to-all GPU kernels
 * for MoE "dispatch" (send each token to the experts its gate picked) and
 * "combine" (merge the experts' outputs back, accumulating), FP8 dispatch and
 * BF16 combine, group-limited gating ("top-4 groups, top-8 experts"), and a
 * host that waits for a GPU-produced receive count:
 *   - "DeepEP ... CPO" GitHub-issue mirror, section "Technical Overview of DeepEP";
 *   - 智东西 news article (yunnanlong.com), the feature list and "具体性能方面";
 *   - brainleap.ai "【Day2】DeepEP", sections "DeepEP是什么", "All-to-All通信"
 *     (combine accumulates) and that section's figure caption on the host
 *     waiting for the GPU's receive counts;
 *   - flashmla.org/de "DeepEP", the feature and benchmark-setting paragraphs.
 * Here the expert-parallel ranks are logical partitions of ONE GPU: rank r owns
 * experts [r*E/R, (r+1)*E/R), every "send" is a row copy inside this GPU's
 * memory, and there is no collective.
 *
 * Conventions for every call.
 *   - Pointers named as device buffers are device (or managed) memory that the
 *     CALLER allocates and frees; the library allocates nothing and keeps no
 *     pointer after a call returns.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous: outputs are ready when the stream is.
 *   - Arrays are dense and row-major.  BF16 values are passed as their 16-bit
 *     patterns (uint16_t); FP8 values as E4M3 ("fn": no infinities, max 448)
 *     bytes.
 *   - Errors the host can see (sizes, null or misaligned pointers) are returned
 *     at once and nothing is launched.  Errors only the GPU can see are OR-ed
 *     into `*status_dev` as bits (1u << CGL_ERANGE, 1u << CGL_ECAPACITY, ...);
 *     the caller zeroes that word and reads it after synchronising.
 *     `status_dev` may be NULL, in which case those errors go unreported (the
 *     kernels still skip the offending copies).  No kernel traps or asserts.
 *   - Calls that share output buffers must not overlap on the GPU.
 *   - Workspaces take any contents.  The layout's blocks signal one another
 *     through 64-bit tags in the workspace: a per-call value from the host
 *     (unique among the process's first 2^31 calls, top bit set) and the
 *     workspace's launch count, which every launch advances, one that timed out
 *     included.  So no word that an earlier call of this library left in a
 *     workspace equals a later call's tag (graph replays of one captured call
 *     share the host value and differ in the count), and neither does zeroed
 *     memory or a count word; other data would have to equal the 64-bit tag
 *     exactly.
 *   - Limits: num_topk in [1, 32]; num_experts in [1, 1024];
 *     num_tokens * num_topk < 2^31; num_experts % num_ranks == 0.
 */
#ifndef CGL_H
#define CGL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum cgl_status {
    CGL_OK = 0,
    CGL_EINVAL = 1,     /* bad size or argument, or a required pointer is NULL */
    CGL_EALIGN = 2,     /* a pointer is not aligned as the call requires */
    CGL_ERANGE = 3,     /* (device) an expert id < -1 or >= E, or a receive row outside the buffer */
    CGL_ECAPACITY = 4,  /* (device) a padded expert received more copies than its capacity */
    CGL_ETIMEOUT = 5,   /* (device) a bounded wait between the layout's blocks gave up (~1 s) */
    CGL_ECUDA = 6,      /* the CUDA runtime refused a launch or an attribute call */
    CGL_ENOTIMPL = 7    /* not implemented */
} cgl_status;

/* Per-call options.  A NULL options pointer means all fields zero. */
typedef struct cgl_opts {
    /* Cap the grid of the copy kernels to this many SMs' worth of CTAs
     * (0 = all SMs).  This is the SM-count control the DeepEP pages list for
     * their normal kernels (news article feature list; flashmla.org/de). */
    int32_t num_sms;
    /* cgl_get_layout only.  0: compact receive rows, expert e's copies at rows
     * [expert_offset[e], expert_offset[e+1]).  > 0: padded receive buffers of
     * `capacity` rows per expert, expert e's copies at rows [e*capacity, ...);
     * the decode setting pads to the largest per-expert count, which the host
     * reads from a first, compact call (max_count). */
    int32_t capacity;
    /* Bit flags (0 = none; bits this library does not define are refused with
     * CGL_EINVAL).  CGL_OPT_UE8M0_SCALES: the FP8 dispatch calls
     * (cgl_dispatch_fp8, cgl_layout_dispatch_fp8, cgl_decode_dispatch_fp8) use
     * power-of-two scales, as an 8-bit exponent-only (UE8M0) scale format holds:
     * per 128-value block, scale = 2^e for the smallest integer e with
     * 448 * 2^e >= amax_c, inv = 2^-e, codes = e4m3_rn_satfinite(x * inv) (x * inv
     * is exact, and no value saturates).  recv_scale still holds binary32
     * values: 2^e, whose biased exponent field ((bits >> 23) & 0xFF) is the
     * UE8M0 code.  Calls that quantise nothing ignore the flag. */
    uint32_t flags;
    /* Optional device scratch for cgl_dispatch_fp8 and cgl_dispatch_bf16: 16
     * bytes, 8-byte aligned, all zero before the first call that uses them.
     * With it the dispatch kernel's CTAs claim their tokens from a counter in
     * it instead of taking a fixed share (on B200 some SMs, by where they sit,
     * stream measurably slower; the faster ones then take more tokens), with
     * results identical to the fixed order; the kernel leaves the 16 bytes
     * zero again when it finishes (batches with at most one token per CTA
     * keep the fixed order and leave it untouched).  Calls that may run at
     * the same time must not share one scratch (stream-ordered calls may),
     * and the scratch must stay allocated as long as a captured CUDA graph
     * that uses it may be replayed.  A scratch that was not zero cannot make
     * the kernel touch memory outside the call's buffers (claims past the
     * batch are clamped), but tokens may be left out: when a claim returns a
     * value that no zeroed start produces (>= num_tokens + 3 * CTAs), the
     * kernel sets the CGL_ERANGE bit in *status.
     * NULL: fixed order.  Other calls ignore it. */
    void *scratch;
} cgl_opts;

#define CGL_OPT_UE8M0_SCALES 1u

/* Library version (major * 10000 + minor * 100 + patch).  0.2.0 added
 * cgl_opts.flags and 0.3.0 cgl_opts.scratch: C callers built against an older
 * cgl.h must be rebuilt. */
int cgl_version(void);

/* A static string naming a cgl_status value (or "unknown status"). */
const char *cgl_status_string(int status);

/*
 * Bytes of device workspace cgl_get_layout needs for these sizes (per-block
 * histograms).  Host-only; returns 0 for invalid sizes.
 */
size_t cgl_layout_workspace_bytes(int64_t num_tokens, int num_topk, int num_experts, int num_ranks);

/*
 * Number of kernels cgl_get_layout launches for these sizes on the current
 * device: 1 (one thread-block cluster for 2 to 8 small blocks, else one
 * cooperative kernel) when all its blocks fit on the GPU at once, else 2.
 * -1 for invalid sizes.  Host-only (queries the device's occupancy once).
 */
int cgl_layout_kernel_count(int64_t num_tokens, int num_topk, int num_experts, int num_ranks);

/*
 * cgl_get_layout -- the dispatch layout: how many copies each expert and each
 * logical rank receives, where they start, and the receive row of every
 * (token, slot) copy.  Pages: the dispatch described under "DeepEP是什么" and
 * "All-to-All通信" (brainleap "Day2 DeepEP"), whose receive counts the host
 * waits on (the figure caption in "All-to-All通信" on the host waiting for the
 * receive counts).
 *
 * In (device):
 *   topk_idx          int32 [num_tokens, num_topk]; expert id per slot, -1 = no copy.
 * Out (device, all written in full by the call):
 *   tokens_per_expert int32 [E]: copies routed to expert e (including copies
 *                     dropped for capacity).
 *   tokens_per_rank   int32 [R]: distinct tokens with at least one copy on rank r.
 *   is_token_in_rank  uint8 [num_tokens, R]: 1 if token t has a copy on rank r, else 0.
 *   expert_offset     int32 [E + 1]: exclusive prefix sum of tokens_per_expert
 *                     (expert order, so each rank's experts are contiguous).
 *   max_count         int32 [1]: max over e of tokens_per_expert.
 *   dst_pos           int32 [num_tokens, num_topk]: receive row of the copy, -1
 *                     when the slot is masked, out of range or over capacity.
 *   recv_src          int32 [num_tokens*num_topk] (compact) or [E*capacity]
 *                     (padded): t*num_topk + j of the copy in each receive row,
 *                     -1 for rows that receive nothing.
 * Order: inside each expert, copies are in ascending token order (ascending
 * slot for a repeated expert within one token), i.e. a stable counting sort.
 * workspace: device, >= cgl_layout_workspace_bytes(...) bytes, 16-byte aligned,
 *   any contents; it is scratch for the call and may be reused afterwards
 *   (calls that overlap on the GPU must not share one).
 * Device errors: CGL_ERANGE for ids < -1 or >= E (those slots make no copy),
 *   CGL_ECAPACITY when a padded expert overflows (late copies dropped).
 * Host errors: CGL_EINVAL (sizes, NULL outputs, small workspace), CGL_EALIGN
 *   (int32 arrays not 4-byte aligned, workspace or is_token_in_rank not 16-byte aligned).
 */
cgl_status cgl_get_layout(const int32_t *topk_idx, int64_t num_tokens, int num_topk,
                          int num_experts, int num_ranks, const cgl_opts *opts,
                          int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                          uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count,
                          int32_t *dst_pos, int32_t *recv_src, void *workspace,
                          size_t workspace_bytes, uint32_t *status_dev, void *stream);

/*
 * cgl_get_rank_layout -- the per-rank (deduplicated) layout: a token sends ONE
 * copy to each logical rank that hosts at least one of its experts, instead of
 * one copy per expert.  Pages: the normal kernels' per-destination transfers
 * and their receive counts ("All-to-All通信", the dispatch bullet: send,
 * forward, receive per destination; the figure caption there on the host
 * waiting for the receive counts).
 * Reading: this is the is_token_in_rank view of dispatch; the receiving rank
 * then serves its local experts and returns one partial row per token.
 *
 * In (device): topk_idx int32 [num_tokens, num_topk] as for cgl_get_layout.
 * Out (device, all written in full):
 *   tokens_per_rank int32 [R]: distinct tokens reaching rank r.
 *   rank_offset     int32 [R + 1]: exclusive prefix sum of tokens_per_rank.
 *   max_count       int32 [1]: max over r of tokens_per_rank.
 *   rank_dst        int32 [num_tokens, num_topk]: for the FIRST slot j of token t
 *                   whose expert lies on rank r, the receive row of t on r; -1 for
 *                   later slots on the same rank and for masked / out-of-range /
 *                   over-capacity slots.
 *   recv_token      int32 [num_tokens*num_topk] (compact) or [R*capacity] (padded):
 *                   the source token of each receive row, -1 for rows with none.
 * Rows of a rank hold its tokens in ascending token order.  opts.capacity > 0
 * pads each rank to `capacity` rows (rank r at [r*capacity, ...)).
 * Use: cgl_dispatch_fp8 / cgl_dispatch_bf16 with dst_pos = rank_dst write one
 * copy per (token, rank); cgl_combine with dst_pos = rank_dst and unit weights
 * sums the ranks' partial rows back in slot order.
 * workspace: >= cgl_layout_workspace_bytes(num_tokens, num_topk, num_ranks, num_ranks)
 *   bytes (the expert layout's size also suffices), 16-byte aligned, any contents.
 * Errors as for cgl_get_layout.
 */
cgl_status cgl_get_rank_layout(const int32_t *topk_idx, int64_t num_tokens, int num_topk,
                               int num_experts, int num_ranks, const cgl_opts *opts,
                               int32_t *tokens_per_rank, int32_t *rank_offset, int32_t *max_count,
                               int32_t *rank_dst, int32_t *recv_token, void *workspace,
                               size_t workspace_bytes, uint32_t *status_dev, void *stream);

/* Size of the device scratch array behind cgl_get_layout_noalloc. */
#define CGL_NOALLOC_SCRATCH_BYTES (512u * 1024u)

/*
 * cgl_get_layout_noalloc -- cgl_get_layout for callers that cannot allocate
 * device memory.  The pages have no counterpart of this entry point.
 *
 * Who needs it: hosts that give the library only pre-planned input and output
 * buffers and own all other device memory (engine plugins, serving runtimes
 * with a fixed memory plan), callers that must not take the device-wide
 * synchronisation that cudaFree implies, and callers that reach only this C
 * ABI without a CUDA allocator.  They cannot provide the workspace that
 * cgl_get_layout takes.
 *
 * Same arguments, outputs, ordering and errors as cgl_get_layout, minus the
 * workspace: the scratch is a fixed device array of CGL_NOALLOC_SCRATCH_BYTES
 * (512 KiB) inside libcgl.so, held by every GPU that loads the library until
 * the process exits.  The call allocates nothing (no cudaMalloc or cudaFree,
 * no allocating library routine); the caller still passes every input and
 * output buffer.
 * Limits, rejected with CGL_EINVAL before anything is launched:
 *   cgl_layout_workspace_bytes(...) <= CGL_NOALLOC_SCRATCH_BYTES
 *     (at E = 256, R = 64, num_topk = 8: up to 52,096 tokens), and
 *   12 * num_experts + num_ranks + T * ceil(num_ranks / 32) <= 9984, with
 *     T = min(256, 1024 / num_topk) tokens per block (the layout kernels then
 *     fit in the default 48 KiB of shared memory per block; with
 *     num_ranks <= 64 this holds for any num_topk up to E = 784).
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address once and caches it; make that first call before any
 * stream capture.  CGL_ECUDA if the lookup fails.
 * Sharing: every call uses the same array, which keeps the last call's
 * contents (nothing in it needs to start at zero).  Calls whose work overlaps
 * on the GPU race on it: serialise them (one stream per device, or events).
 */
cgl_status cgl_get_layout_noalloc(const int32_t *topk_idx, int64_t num_tokens, int num_topk,
                                  int num_experts, int num_ranks, const cgl_opts *opts,
                                  int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                                  uint8_t *is_token_in_rank, int32_t *expert_offset,
                                  int32_t *max_count, int32_t *dst_pos, int32_t *recv_src,
                                  uint32_t *status_dev, void *stream);

/*
 * cgl_dispatch_fp8 -- FP8 dispatch: quantise each token once and write its
 * copies to the receive rows.  Pages: "FP8 dispatch, BF16 combine" in the
 * benchmark settings (news article "具体性能方面"; brainleap "DeepEP 的性能表现";
 * flashmla.org/de) and "原生FP8 调度支持" (brainleap key techniques, item 5).
 *
 * For token t and each block b of 128 consecutive hidden values:
 *   amax = max |x|, amax_c = max(amax, 1e-4), scale = amax_c / 448,
 *   inv = 448 / amax_c (IEEE binary32 divisions), q = e4m3_rn_satfinite(x * inv)
 *   (with CGL_OPT_UE8M0_SCALES: scale = 2^e, inv = 2^-e, see cgl_opts.flags);
 * then for every slot j with dst_pos[t, j] = row >= 0:
 *   recv_x[row, :] = q, recv_scale[row, b] = scale.
 * In (device): x BF16 [num_tokens, hidden]; dst_pos int32 [num_tokens, num_topk]
 *   (from cgl_get_layout).
 * Out (device): recv_x uint8 [num_recv_rows, hidden], recv_scale fp32
 *   [num_recv_rows, hidden/128].  Rows that receive no copy are NOT written.
 * Requires hidden % 128 == 0; x and recv_x 16-byte aligned; dst_pos and
 * recv_scale 4-byte aligned.
 * With opts->scratch the CTAs claim tokens dynamically (see cgl_opts.scratch);
 * the results are the same.
 * Device errors: CGL_ERANGE if some dst_pos >= num_recv_rows (that copy is skipped).
 */
cgl_status cgl_dispatch_fp8(const uint16_t *x, int64_t num_tokens, int hidden, int num_topk,
                            const int32_t *dst_pos, uint8_t *recv_x, float *recv_scale,
                            int64_t num_recv_rows, const cgl_opts *opts, uint32_t *status_dev,
                            void *stream);

/*
 * cgl_dispatch_bf16 -- BF16 dispatch: recv_x[dst_pos[t, j], :] = x[t, :] bit for
 * bit.  The same call re-dispatches gradient rows by a forward layout
 * (combine-backward, unweighted).  Pages: dispatch as above; BF16 is the
 * combine format of the benchmark settings.
 * In (device): x BF16 [num_tokens, hidden]; dst_pos int32 [num_tokens, num_topk].
 * Out (device): recv_x BF16 [num_recv_rows, hidden]; rows with no copy are not written.
 * Requires hidden % 8 == 0; x and recv_x 16-byte aligned.  With opts->scratch
 * (hidden % 16 == 0 and <= 8192) the CTAs claim tokens dynamically.
 * Device errors: CGL_ERANGE if some dst_pos >= num_recv_rows.
 */
cgl_status cgl_dispatch_bf16(const uint16_t *x, int64_t num_tokens, int hidden, int num_topk,
                             const int32_t *dst_pos, uint16_t *recv_x, int64_t num_recv_rows,
                             const cgl_opts *opts, uint32_t *status_dev, void *stream);

/*
 * cgl_combine -- BF16 combine: gather each token's expert outputs back and
 * reduce them with the top-k weights.  Pages: combine "accumulates"
 * (brainleap "All-to-All通信", the combine bullet), BF16 combine (benchmark
 * settings).
 *   out[t, h] = bf16_rn( ((+0 + w[t,0]*y0) + w[t,1]*y1) + ... ), y_j = y[dst_pos[t, j], h],
 * each product and each sum one binary32 operation (no fused multiply-add),
 * slots in order j = 0..k-1, slots with dst_pos < 0 skipped.
 * In (device): y BF16 [num_recv_rows, hidden]; dst_pos int32 [num_tokens, num_topk];
 *   topk_weights fp32 [num_tokens, num_topk] (used as given).
 * Out (device): out BF16 [num_tokens, hidden], every element written.
 * Requires hidden % 8 == 0; y and out 16-byte aligned.
 * Device errors: CGL_ERANGE if some dst_pos >= num_recv_rows (that slot is skipped).
 */
cgl_status cgl_combine(const uint16_t *y, int64_t num_recv_rows, const int32_t *dst_pos,
                       const float *topk_weights, int64_t num_tokens, int hidden, int num_topk,
                       uint16_t *out, const cgl_opts *opts, uint32_t *status_dev, void *stream);

/*
 * cgl_decode_dispatch_fp8 -- the decode path in one launch: cgl_get_layout and
 * cgl_dispatch_fp8 fused for a small batch, with no workspace.  Pages: the
 * low-latency kernels for decoding (news article feature list and
 * "具体性能方面": 128 tokens per batch, hidden 7168, top-8, FP8 dispatch, BF16
 * combine; brainleap "Pure RDMA 的低延迟内核"), here on one GPU: one launch
 * instead of two, no device-to-host count read when opts.capacity fixes the
 * per-expert capacity in advance (what a captured CUDA graph needs).
 * Same outputs, ordering and errors as cgl_get_layout followed by
 * cgl_dispatch_fp8 with the layout's dst_pos (receive rows = E*capacity when
 * opts.capacity > 0, else num_tokens*num_topk; rows past a full expert are
 * dropped with CGL_ECAPACITY).
 * Limits (CGL_EINVAL otherwise): num_tokens <= min(256, 1024 / num_topk)
 * (128 at top-8); hidden % 128 == 0; the shared memory the kernel needs
 * (per-block counts for E experts, the batch's (token, slot) rows) within
 * 47 KiB.  opts.num_sms caps the grid (one CTA per token otherwise).
 * Alignment: x, recv_x and is_token_in_rank 16-byte aligned; int32/fp32 arrays 4-byte.
 */
cgl_status cgl_decode_dispatch_fp8(const int32_t *topk_idx, int64_t num_tokens, int num_topk,
                                   int num_experts, int num_ranks, const cgl_opts *opts,
                                   const uint16_t *x, int hidden, int32_t *tokens_per_expert,
                                   int32_t *tokens_per_rank, uint8_t *is_token_in_rank,
                                   int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                                   int32_t *recv_src, uint8_t *recv_x, float *recv_scale,
                                   uint32_t *status_dev, void *stream);

/*
 * Bytes of device workspace cgl_layout_dispatch_fp8 needs for these sizes
 * (cgl_get_layout's workspace, then, 16-byte aligned, the dispatch kernel's
 * token counter).  Host-only; 0 for invalid sizes.
 */
size_t cgl_layout_dispatch_workspace_bytes(int64_t num_tokens, int num_topk, int num_experts, int num_ranks);

/*
 * Kernels cgl_layout_dispatch_fp8 launches for these sizes on the current
 * device: 1 when the fused kernel applies, else the layout's count + 1.
 * -1 for invalid sizes.  Host-only (queries the device once per shape).
 */
int cgl_layout_dispatch_kernel_count(int64_t num_tokens, int num_topk, int num_experts, int num_ranks,
                                     int hidden, const cgl_opts *opts);

/*
 * cgl_layout_dispatch_fp8 -- cgl_get_layout and cgl_dispatch_fp8 in one call
 * for any batch size.  Pages: the dispatch and its receive counts as for
 * cgl_get_layout, FP8 dispatch as for cgl_dispatch_fp8 (brainleap "Day2
 * DeepEP": the normal kernels' prefill setting, FP8 dispatch with BF16
 * combine).  The pages have no fused form; on one GPU it lets the FP8
 * dispatch's reads and quantisation run while the layout's counts are made.
 * Same outputs, ordering and errors as cgl_get_layout followed by
 * cgl_dispatch_fp8 with the layout's dst_pos (receive rows = E*capacity when
 * opts.capacity > 0, else num_tokens*num_topk).
 * One kernel when it applies: one CTA per token when there is at most one
 * token per SM in use (decode); for prefill-sized batches (every SM gets at
 * least 64 (token, slot) pairs, at most 32768 pairs, and a CTA's whole share
 * of FP8 rows fits in shared memory: at hidden 7168 up to 28 tokens per CTA,
 * 4144 tokens on 148 SMs) one CTA of 768 threads per SM, each owning
 * ceil(num_tokens / SMs) tokens, which reads every id for the counts (no CTA
 * waits on another) while it stages its tokens' FP8 rows.  Otherwise the
 * layout kernel(s), then the dispatch kernel, whose CTAs take their tokens
 * from a counter at the workspace's tail that the call zeroes first (CTAs
 * on faster SMs take more); the same results either way.
 * opts.num_sms caps the SMs used.
 * workspace: device, >= cgl_layout_dispatch_workspace_bytes(...) bytes,
 *   16-byte aligned, any contents (scratch for the call; overlapping calls
 *   must not share one).
 * Requires hidden % 128 == 0.  Alignment: x, recv_x, is_token_in_rank and the
 * workspace 16-byte aligned; int32/fp32 arrays 4-byte (a 16-byte aligned
 * recv_scale with hidden % 512 == 0 lets the scale rows go out as bulk copies).
 * Device errors: as cgl_get_layout (CGL_ERANGE, CGL_ECAPACITY, CGL_ETIMEOUT
 * for the inter-block wait, after which nothing is dispatched).
 */
cgl_status cgl_layout_dispatch_fp8(const int32_t *topk_idx, int64_t num_tokens, int num_topk,
                                   int num_experts, int num_ranks, const cgl_opts *opts,
                                   const uint16_t *x, int hidden, int32_t *tokens_per_expert,
                                   int32_t *tokens_per_rank, uint8_t *is_token_in_rank,
                                   int32_t *expert_offset, int32_t *max_count, int32_t *dst_pos,
                                   int32_t *recv_src, uint8_t *recv_x, float *recv_scale,
                                   void *workspace, size_t workspace_bytes, uint32_t *status_dev,
                                   void *stream);

/*
 * cgl_combine_backward -- the gradient of cgl_combine.  Pages: combine
 * accumulates the experts' outputs (brainleap "Day2 DeepEP", "All-to-All通信");
 * this is its derivative for training.  For an output gradient g = dL/dout:
 *   grad_y[dst_pos[t, j], h] = bf16_rn( w[t, j] * g[t, h] )   (one binary32 product)
 *   grad_w[t, j]             = sum_h g[t, h] * y[dst_pos[t, j], h]   (binary32)
 * grad_w's summation order is this library's (per-thread fused multiply-adds,
 * then a fixed tree over the block): deterministic, within a few binary32
 * roundings of the exact sum; slots with dst_pos < 0 give grad_w = 0 and write
 * no row.
 * In (device): grad_out BF16 [num_tokens, hidden]; y BF16 [num_recv_rows, hidden]
 *   (the expert outputs combine read); dst_pos, topk_weights as for cgl_combine.
 * Out (device): grad_y BF16 [num_recv_rows, hidden] (rows with no slot untouched);
 *   grad_w fp32 [num_tokens, num_topk] (every element written).
 * Requires hidden % 16 == 0 and hidden <= 16384; grad_out, y, grad_y 16-byte aligned.
 * Device errors: CGL_ERANGE if some dst_pos >= num_recv_rows (that slot is skipped).
 */
cgl_status cgl_combine_backward(const uint16_t *grad_out, const uint16_t *y, int64_t num_recv_rows,
                                const int32_t *dst_pos, const float *topk_weights, int64_t num_tokens,
                                int hidden, int num_topk, uint16_t *grad_y, float *grad_w,
                                const cgl_opts *opts, uint32_t *status_dev, void *stream);

/*
 * cgl_selftest_bounded_wait -- diagnostic for failure detection.  Runs the
 * layout's inter-block wait (the only software wait in any kernel of this
 * library) in one block, exit path included, on a layout workspace header:
 * workspace[0] is the generation word and workspace[1 .. nflags] are the flags.
 * It waits for a tag that no layout launch writes, so on zeroed memory, or on
 * a header that layout calls have used, it must give up after ~1 s (2^31 SM
 * cycles), OR 1u << CGL_ETIMEOUT into *status_dev, advance the generation word
 * by one (as a layout block that times out does, so that the next layout call
 * on that workspace gets a new tag) and return; the stream and the context
 * stay usable.  workspace: device, 8-byte aligned, 1 + nflags words;
 * nflags in [1, 4096].  The pages have no counterpart.
 */
cgl_status cgl_selftest_bounded_wait(uint64_t *workspace, int nflags, uint32_t *status_dev, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CGL_H */
