/*
 * k3moe -- one Kimi-K3-shape mixture-of-experts FFN layer computed directly on
 * packed MXFP4 expert weights, for NVIDIA B200 (sm_100a).
 *
 * The layer (per token x, hidden size d):
 *   l   = W_r x + b                              router logits over E experts
 *   p   = softmax(l)                              over all E experts
 *   idx = the k experts with the largest l, ties to the lower index, listed in
 *         descending order; w_j = p_idx_j (not renormalised over the k)
 *   o_e = W_d,e (silu(W_g,e x) * W_u,e x)         SwiGLU expert, MXFP4 weights
 *   S   = W_d,s (silu(W_g,s x) * W_u,s x)         shared expert, bf16 weights
 *   y   = S + sum_j w_j o_idx_j
 * Sources: "Kimi K3 纯 C 语言 CPU 推理实战" (chenxutan.com), section 1.2 (the
 * routing formula, K = 16 of 896 experts plus an always-on shared expert) and
 * section 2.4 (router GEMV, stable softmax over all experts, top-k, weighted
 * combine; the MoELayer/moe_forward interface); the kimi-k3-in-c project card
 * ("P053"), core features (experts multiplied directly on the packed nibbles,
 * never dequantised; MXFP4 = 4-bit E2M1 nibble + shared E8M0 scale, 0.53125
 * bytes per weight) and architecture notes (the config reader refuses
 * defaults: every argument here is explicit and validated).
 *
 * ---------------------------------------------------------------------------
 * Data formats (all device memory, little-endian, row-major):
 *   x          bf16 [T][d]
 *   w_router   fp32 [E][d]
 *   bias       fp32 [E], or NULL for no bias (added to the logits before the
 *              softmax, so it moves both the selection and the weights)
 *   expert blob, one per routed expert, 3*d*ff*17/32 bytes, 16-byte aligned:
 *     [W_g nibbles | W_g scales | W_u nibbles | W_u scales | W_d nibbles | W_d scales]
 *     W_g, W_u: ff rows x d columns; W_d: d rows x ff columns.
 *     A nibble plane holds rows*cols/2 bytes: element (r, c) is the low nibble
 *     (bits 0-3) of byte r*cols/2 + c/2 when c is even, the high nibble when c
 *     is odd.  A scale plane holds rows*cols/32 E8M0 bytes: byte r*cols/32 + c/32
 *     scales the 32 consecutive elements of row r that contain column c.
 *     E2M1 code: sign bit 3, 2 exponent bits (bias 1), 1 mantissa bit ->
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6}; E8M0 byte e -> 2^(e-127), 255 = NaN
 *     (OCP Microscaling Formats v1.0).
 *   shared expert: W_g,s, W_u,s bf16 [ff_shared][d], W_d,s bf16 [d][ff_shared]
 *   y          [T][d], bf16 (round to nearest even, once, from the fp32 sum) or
 *              fp32 with K3MOE_OUT_FP32
 *   idx        int32 [T][k], weight fp32 [T][k]
 *
 * Precision: routed-expert weights enter the tensor cores exactly, as their
 * own E2M1 codes and E8M0 scales (block-scaled MMA, E2M1 x E2M1).  The
 * activations they multiply (x, and w_j * h for the down projections, the
 * routing weight folded in) enter as sums of 6 E2M1 pieces, each 32-element
 * block of each piece with its own E8M0 scale taken from what the earlier
 * pieces left over; the pieces reproduce each activation to about 2^-19 of
 * the largest element of its 32-element block.  The bf16 shared expert runs
 * on bf16 tensor-core MMAs with x exact and its h as bf16 hi + lo.  All
 * accumulation is fp32 (the routed down projections and the shared one sum
 * into one fp32 accumulator per output).  Router logits are fp32 sums of
 * exact fp32 x bf16 products.
 *
 * Many tokens (T > 8, with a workspace sized for T): the grouped path.  The
 * router is a GEMM over all tokens (fp32, fixed summation order), the
 * (token, slot) pairs are sorted by expert and cut into groups of up to 32
 * tokens, and each group runs through the experts' packed weights on the
 * tensor cores with its activations as 4 E2M1 pieces (about 2^-10 of the
 * block's largest element); each (token, slot) output is kept in fp32 and
 * the k + 1 outputs of a token are summed in slot order (shared expert last)
 * before the one rounding.  A workspace sized for 8 tokens runs any T as
 * 8-token passes of the path above.
 *
 * Ownership and ordering: the caller owns every buffer and the stream.  Calls
 * allocate nothing, never synchronise, and are ordered on `stream`; results
 * are valid once the stream reaches them, and inputs must stay unmodified
 * until then.  `ws` is caller-owned device scratch of at least
 * k3moe_workspace_size() bytes, 256-byte aligned and zero-filled before its
 * first use (each call leaves it ready for the next); one workspace must not
 * be used by two calls that may run at the same time.
 *
 * Errors: every call validates all arguments before launching anything and
 * returns a status; on failure nothing is launched.  Launch failures return
 * K3MOE_ERR_CUDA (the CUDA error text is kept for k3moe_last_error()).
 * Conditions only the device can see (a blob pointer that is not 16-byte
 * aligned, a bounded wait that ran out) are recorded in the workspace status
 * word and read with k3moe_device_status().
 * ---------------------------------------------------------------------------
 */
#ifndef K3MOE_H
#define K3MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define K3MOE_ABI_VERSION 1

typedef enum {
    K3MOE_OK = 0,
    K3MOE_ERR_INVALID_ARGUMENT = 1,   /* null/misaligned pointer, bad count */
    K3MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* dimension outside the supported set */
    K3MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    K3MOE_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    K3MOE_ERR_DEVICE_TIMEOUT = 5,     /* a bounded device wait ran out */
    K3MOE_ERR_DEVICE_CHECK = 6        /* a device-side argument check failed */
} k3moe_status;

/* flags */
#define K3MOE_OUT_FP32 1u  /* y (and expert_ffn's out) in fp32 instead of bf16 */
#define K3MOE_NO_SHARED 2u /* skip the shared expert (its pointers may be NULL) */
/* Check every E8M0 scale byte the call reads for 0xFF (the encoding of NaN,
 * OCP Microscaling Formats v1.0): a call that meets one records
 * K3MOE_ERR_DEVICE_CHECK in the workspace status word (its outputs are then
 * undefined).  Without the flag the byte is handed to the tensor core as it
 * is, and the outputs it reaches are whatever the hardware makes of a NaN
 * scale. */
#define K3MOE_STRICT 4u
/* Routing variants (the pages' routing uses neither; both are common in MoE
 * models).  K3MOE_RENORM_TOPK: the k weights of a token are divided by their
 * sum, w_j = p_idx_j / sum_j' p_idx_j' (summed in pick order).
 * K3MOE_BIAS_SELECT_ONLY: `bias` moves only the selection -- the top-k is
 * taken on l_e + b_e, while the weights come from the softmax of the unbiased
 * logits l (without the flag the bias is part of the logits and so moves
 * both). */
#define K3MOE_RENORM_TOPK 8u
#define K3MOE_BIAS_SELECT_ONLY 16u
/* Decode passes (T <= 8 tokens per pass) as one cooperative launch (router,
 * top-k, gate/up, down and combine in one kernel, the shared expert's gate/up
 * streamed while the routing is decided) instead of the default three
 * launches (route; gate/up; down).  Same results within the output tolerance
 * (the partial sums are added in another order); the routing of the two may
 * differ only where two logits tie to the last bit.  Shapes the one-launch
 * kernel does not take (d > 8192, too many router rows per CTA) run the
 * three launches. */
#define K3MOE_ONE_LAUNCH 32u

/*
 * Layer dimensions.  d and ff: multiples of 64, 64 <= d <= 8192,
 * 64 <= ff <= 3072; 1 <= n_experts <= 1024; 1 <= top_k <= min(n_experts, 32);
 * ff_shared: 0 (no shared expert) or a multiple of 64 up to 3072.  Shapes
 * whose staging tiles do not fit in one SM's shared memory return
 * K3MOE_ERR_UNSUPPORTED_SHAPE.  Unknown flag bits are rejected.
 */
typedef struct {
    int32_t d;
    int32_t ff;
    int32_t n_experts;
    int32_t top_k;
    int32_t ff_shared;
    uint32_t flags;
} k3moe_dims;

/* ABI version of the loaded library (K3MOE_ABI_VERSION when it matches). */
int k3moe_abi_version(void);

/* Bytes of one routed expert's blob: 3*d*ff*17/32; 0 if dims are invalid. */
size_t k3moe_blob_bytes(const k3moe_dims *dims);

/* Scratch bytes a call with up to T_max tokens needs; 0 if dims are invalid.
 * For T_max > 8 this includes the grouped path's region for passes of up to
 * 8192 tokens (about 0.9 MB per token for the K3 shape, most of it the fp32
 * output of every (token, slot)); a call with more tokens than its workspace
 * was sized for falls back to 8-token passes when the workspace holds those. */
size_t k3moe_workspace_size(const k3moe_dims *dims, int32_t T_max);

/*
 * Router, softmax over all experts, top-k (tutorial page, section 2.4):
 *   idx[t][j] = j-th selected expert of token t (descending logit, ties to the
 *               lower index), weight[t][j] = its softmax probability.
 * x: bf16 [T][d]; w_router: fp32 [E][d]; bias: fp32 [E] or NULL;
 * idx: int32 [T][k]; weight: fp32 [T][k].  All pointers 16-byte aligned
 * except bias, idx and weight (4-byte aligned).  With T > 8 and a workspace
 * sized for T, the logits come from the grouped path's router GEMM.
 */
k3moe_status k3moe_route(const void *x, int32_t T, const float *w_router, const float *bias,
                         const k3moe_dims *dims, int32_t *idx, float *weight, void *ws,
                         size_t ws_bytes, void *stream);

/*
 * One routed expert applied to T tokens, unweighted (the per-expert step of
 * the tutorial page's section 2.4 loop, on the packed nibbles per the project
 * card): out[t] = W_d (silu(W_g x_t) * W_u x_t).
 * blob: one expert blob as above (16-byte aligned); out: [T][d] bf16, or fp32
 * with K3MOE_OUT_FP32.  n_experts/top_k/ff_shared in dims are not used but
 * must still be valid.
 */
k3moe_status k3moe_expert_ffn(const void *x, int32_t T, const uint8_t *blob,
                              const k3moe_dims *dims, void *out, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * The whole layer (tutorial page, sections 1.2 and 2.4):
 *   y[t] = S(x_t) + sum_j w[t][j] o_idx[t][j](x_t)
 * expert_blobs: DEVICE array of E device pointers, expert e's blob at
 *   expert_blobs[e] (each 16-byte aligned; checked on the device);
 * shared_wg/wu/wd: bf16 shared-expert matrices, or NULL with ff_shared == 0
 *   or K3MOE_NO_SHARED;
 * y: [T][d] bf16 or fp32 (K3MOE_OUT_FP32);
 * idx_out / w_out: optional copies of the routing ([T][k]), may be NULL.
 */
k3moe_status k3moe_layer(const void *x, int32_t T, const float *w_router, const float *bias,
                         const uint8_t *const *expert_blobs, const void *shared_wg,
                         const void *shared_wu, const void *shared_wd, const k3moe_dims *dims,
                         void *y, int32_t *idx_out, float *w_out, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * The layer inside a pre-norm transformer block: the step before it (RMSNorm
 * of the residual stream) and the one after it (the residual add) fused in
 * (the kimi-k3-in-c project card lists RMSNorm among its kernels; the pages
 * give no formula, so the standard one is used):
 *   x      = RNE_bf16( h * norm_w / sqrt(mean(h^2) + eps) )   per token
 *   h_out  = h + layer(x)                                      rounded once
 * h: bf16 [T][d] (the residual stream); norm_w: bf16 [d], 16-byte aligned;
 * eps >= 0; h_out: [T][d] bf16 (or fp32 with K3MOE_OUT_FP32), and may be h
 * itself (updated in place).  The normalisation runs in fp32 (1/rms as
 * 1/sqrtf of the fp32 mean of squares, each element (h * r) * w rounded to
 * bf16): up to 8 tokens per pass a norm launch writes x into the workspace
 * before the decode launches and the down pass adds h before its rounding
 * (with K3MOE_ONE_LAUNCH both are fused into the one-launch kernel, within its
 * shape limits); with a workspace sized for more tokens the grouped path
 * normalises each pass first and adds h in its final sum.  Other arguments as
 * for k3moe_layer (no routing copies).
 */
k3moe_status k3moe_layer_residual(const void *h, int32_t T, const void *norm_w, float eps,
                                  const float *w_router, const float *bias,
                                  const uint8_t *const *expert_blobs, const void *shared_wg,
                                  const void *shared_wu, const void *shared_wd,
                                  const k3moe_dims *dims, void *h_out, void *ws, size_t ws_bytes,
                                  void *stream);

/*
 * Expert cache: the routed experts live in host memory and only the most
 * recently used ones in device memory, in n_slots slots -- the pages' defining
 * idea (the kimi-k3-in-c project card: experts are streamed on demand, never
 * all resident; their engine keeps an LRU of RAM slots fed from NVMe), one
 * level up: host memory -> HBM by the copy engine.  The layer calls reach the
 * experts through their device pointer table, which the cache rewrites.
 *   k3moe_cache_slot_bytes: bytes of one slot (the blob size rounded up to 256).
 *   k3moe_cache_create: slot_mem is caller-owned device memory of at least
 *     n_slots * slot bytes, 256-byte aligned; host_blobs holds E host pointers
 *     to the experts' blobs (page-locked memory makes the copies asynchronous;
 *     it must stay valid while the cache is used).  The library allocates the
 *     small host-side bookkeeping (freed by k3moe_cache_destroy) and no device
 *     memory.  Starts empty.
 *   k3moe_cache_fetch: makes every expert in experts[0..n) (host array,
 *     repeats allowed) resident: experts already in a slot are marked used;
 *     each missing one (in order of first appearance) takes a free slot or the
 *     least recently used slot not holding a requested expert (lowest slot on
 *     ties) and is copied in with one cudaMemcpyAsync on `stream`.  Then the
 *     device pointer table ptr_table (E entries) is rewritten on `stream`:
 *     each resident expert's slot address, NULL for the others (a call that
 *     selects a non-resident expert reports K3MOE_ERR_DEVICE_CHECK through the
 *     workspace status).  K3MOE_ERR_INVALID_ARGUMENT, with nothing changed,
 *     when an id is out of range or more distinct experts than slots are asked.
 *   k3moe_cache_plan: the same bookkeeping without any copy (simulation).
 *   k3moe_layer_cached: k3moe_layer with the experts behind the cache: per
 *     pass of up to 8 tokens, the routing (the same kernel and bits as the
 *     layer's own), its picks copied to idx_host (host, [T][k] int32, page-
 *     locked preferred), a SYNCHRONISATION of `stream`, a fetch of the picks,
 *     then the layer on the fetched experts.  ws needs k3moe_workspace_size(dims, 8).
 */
typedef struct k3moe_cache k3moe_cache;
typedef struct {
    uint64_t requests;  /* distinct experts asked for, summed over fetches */
    uint64_t hits;      /* of those, already resident */
    uint64_t fills;     /* copied in */
    uint64_t evictions; /* resident experts replaced */
} k3moe_cache_stats;
size_t k3moe_cache_slot_bytes(const k3moe_dims *dims);
k3moe_status k3moe_cache_create(const k3moe_dims *dims, int32_t n_slots, void *slot_mem,
                                size_t slot_mem_bytes, const void *const *host_blobs,
                                k3moe_cache **cache);
void k3moe_cache_destroy(k3moe_cache *cache);
k3moe_status k3moe_cache_fetch(k3moe_cache *cache, const int32_t *experts, int32_t n,
                               void *ptr_table, void *stream);
k3moe_status k3moe_cache_plan(k3moe_cache *cache, const int32_t *experts, int32_t n,
                              int32_t *filled, int32_t *n_filled);
k3moe_status k3moe_cache_get_stats(const k3moe_cache *cache, k3moe_cache_stats *stats);
k3moe_status k3moe_layer_cached(k3moe_cache *cache, const void *x, int32_t T, const float *w_router,
                                const float *bias, void *ptr_table, const void *shared_wg,
                                const void *shared_wu, const void *shared_wd,
                                const k3moe_dims *dims, void *y, int32_t *idx_host, void *ws,
                                size_t ws_bytes, void *stream);

/*
 * k3moe_layer with the activations in HOST memory: copies x_host ([T][d]
 * bf16) into the workspace, runs the layer, and copies y back to y_host
 * ([T][d], bf16 or fp32 per flags), all ordered on `stream` (the copies are
 * asynchronous when the host buffers are page-locked).  Weights stay in
 * device memory as for k3moe_layer.  The host buffers must stay valid until
 * the stream reaches the end of the call.  Needs
 * k3moe_workspace_size(dims, T) + k3moe_host_staging_bytes(dims, T) bytes.
 */
size_t k3moe_host_staging_bytes(const k3moe_dims *dims, int32_t T);
k3moe_status k3moe_layer_from_host(const void *x_host, int32_t T, const float *w_router,
                                   const float *bias, const uint8_t *const *expert_blobs,
                                   const void *shared_wg, const void *shared_wu,
                                   const void *shared_wd, const k3moe_dims *dims, void *y_host,
                                   void *ws, size_t ws_bytes, void *stream);

/*
 * k3moe_layer for per-kernel timing (device input and output, up to 8 tokens,
 * i.e. one pass of the kernels): `events` are n_events cudaEvent_t handles
 * created by the caller; events[0] is recorded on `stream` before the first
 * kernel and events[i] after the i-th kernel, for i up to the number of
 * kernels the call launches, which is written to *n_kernels (3: router with
 * softmax, top-k and dispatch; gate/up of the routed and shared experts;
 * down projections with the weighted combine).
 * The computation and its result are those of k3moe_layer.
 */
k3moe_status k3moe_layer_timed(const void *x, int32_t T, const float *w_router, const float *bias,
                               const uint8_t *const *expert_blobs, const void *shared_wg,
                               const void *shared_wu, const void *shared_wd,
                               const k3moe_dims *dims, void *y, void *ws, size_t ws_bytes,
                               void *stream, void *const *events, int32_t n_events,
                               int32_t *n_kernels);

/*
 * k3moe_layer without a caller-supplied workspace.  The pages this library
 * follows have no counterpart of this call; it exists for callers that cannot
 * allocate device memory at the point where they run the layer (code that
 * must not call an allocator on its hot path, or a host framework whose
 * allocator is not reachable through a C ABI).  Neither the library nor the
 * caller allocates anything: the scratch is a fixed 16 MiB buffer in the
 * library's own device data, one per device.
 *   - The first call on a device looks up that buffer's device address for
 *     the current device (cudaGetSymbolAddress) and clears it on `stream`;
 *     make that first call before any stream capture begins.  A call whose
 *     shape (d, ff, n_experts, top_k, ff_shared) differs from the previous
 *     call's on that device also clears it first (the scratch layout and the
 *     counters in it that must start at zero depend on the shape).
 *   - Shapes whose scratch (k3moe_workspace_size(dims, 8)) exceeds 16 MiB are
 *     rejected with K3MOE_ERR_WORKSPACE_TOO_SMALL before anything runs; the
 *     K3 shape (d=7168, ff=1536, 896 experts, top-16, shared ff=1536) needs
 *     about 14.8 MiB.
 *   - All calls on one device share the buffer: two calls that may overlap
 *     (other streams, other host threads) race and give wrong results.
 *     Serialise them, or use k3moe_layer with a workspace per stream.
 *   - Conditions only the device can see (misaligned blob pointers, a
 *     bounded wait that ran out) are recorded in the buffer's status word,
 *     which this interface does not read back; k3moe_layer reports them
 *     through k3moe_device_status.
 * Arguments, layouts, results and ordering are those of k3moe_layer without
 * the routing copies (idx_out, w_out).
 */
k3moe_status k3moe_layer_noalloc(const void *x, int32_t T, const float *w_router, const float *bias,
                                 const uint8_t *const *expert_blobs, const void *shared_wg,
                                 const void *shared_wu, const void *shared_wd,
                                 const k3moe_dims *dims, void *y, void *stream);

/*
 * Synchronises `stream`, then reads and clears the workspace status word:
 * K3MOE_OK, K3MOE_ERR_DEVICE_CHECK or K3MOE_ERR_DEVICE_TIMEOUT.  After
 * K3MOE_ERR_DEVICE_TIMEOUT the outputs of the calls since the last check are
 * undefined and the workspace must be zero-filled again before its next use.
 * ws == NULL reads the built-in scratch of k3moe_layer_noalloc on the
 * current device instead; there, after K3MOE_ERR_DEVICE_TIMEOUT, this call
 * itself zero-fills the whole built-in buffer (synchronously), so the next
 * k3moe_layer_noalloc call starts clean.
 */
k3moe_status k3moe_device_status(void *ws, void *stream);

/*
 * For tests of the failure paths only (process-wide; leave at 0, 0 in
 * production).  Makes a bounded device wait run out without any GPU fault:
 *   mode 0: normal operation;
 *   mode 1: the routed gate/up work of every later layer call waits for a
 *           "routing loaded" signal that is never given, so its waits run
 *           out and the call records K3MOE_ERR_DEVICE_TIMEOUT (the kernels
 *           then finish early with undefined outputs; nothing faults).
 * wait_limit_ns bounds every device wait of later calls (0: the default of
 * 2 seconds).  Returns K3MOE_ERR_INVALID_ARGUMENT for an unknown mode.
 */
k3moe_status k3moe_debug_set_fault(int32_t mode, uint64_t wait_limit_ns);

/* Static text for a status code. */
const char *k3moe_status_string(k3moe_status status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char *k3moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* K3MOE_H */
