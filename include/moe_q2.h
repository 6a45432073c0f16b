/*
 * moe_q2.h -- C ABI of a B200 (sm_100a) library for one routed
 * mixture-of-experts FFN layer whose experts are stored as 2-bit block
 * ("Q2") quantized weights.
 *
 * The problem, as the pages state it: a sparse MoE model of 48 layers x 512
 * routed experts in which every token is sent to 10 routed experts plus 1
 * shared expert (Strata tuning page, section 2, model table; devlabs page,
 * section 1 "MoE 专家分流"); the expert matmuls run directly from the
 * quantized blocks, which are never densified at load (strata-mlx page, "它是
 * 什么", first bullet); the 2-bit format decodes through an affine codebook
 * with bias -1 (devlabs page, section 4, second validation layer).  Prompts
 * arrive in 1024-token chunks (devlabs page, section 1) or larger chunks such
 * as 32768 (Strata tuning page, section 4), decode/verify windows hold 1-3
 * tokens (guess-and-check, devlabs page, section 1).
 *
 * Conventions for every call
 *  - Every pointer is a DEVICE pointer unless the comment says otherwise.  The
 *    caller allocates and owns all memory (weights, activations, outputs,
 *    workspace); the library allocates nothing in these calls and keeps no
 *    mutable global state (apart from the per-thread profiling switch
 *    moe_trace_kernel), so calls on different streams with different
 *    workspaces are independent.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Argument checks run on the host before any
 *    launch and return an error with nothing enqueued.
 *  - Activations are bfloat16, passed as uint16_t bit patterns, row-major
 *    [T, hidden].  Router weights are fp32 [n_experts, hidden] row-major.
 *  - Kernels never trap or assert.  An inconsistency found on the device sets
 *    a sticky status word in the workspace; moe_check_status() reads it.
 */
#ifndef MOE_Q2_H
#define MOE_Q2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st *moe_stream_t;

/* Layer dimensions.  The Q2 block is fixed at 32 weights.
 * Limits checked by every call (MOE_ERR_ARG otherwise, sizes report 0):
 *  - hidden and inter are multiples of 128 in [128, 4096].  The packed layout
 *    groups four 32-weight blocks (128 weights) along the contraction
 *    dimension: that group is one lane-fragment load, one TMA box and one
 *    tensor-core K chunk, so a remainder of one to three blocks has no place
 *    in it.  The pages' model (hidden 2048, expert intermediate 512 in this
 *    library's synthetic stand-in) is far inside both bounds.
 *  - 1 <= n_experts <= 65535 (the pages' model routes over 512 per layer).
 *  - 1 <= top_k <= min(n_experts, 32): the selection keeps one warp lane per
 *    selected expert (the pages' model selects 10).
 * Which kernels run: T <= 8 with inter = 512, T * top_k <= 128 and
 * n_experts <= 1024 takes one fused persistent kernel for the whole layer;
 * other T <= 8 shapes take the routing kernels plus register-dequantising
 * tensor-core expert kernels (slower, about 2x at the pages' shape); T > 8
 * takes the tcgen05 prefill kernels.  The fused kernel is launched with
 * programmatic dependent launch: while an earlier fused launch on the same
 * stream finishes, it may already load its router rows and prefetch the
 * shared expert (weights, which no launch of this library writes); it reads
 * x and the workspace only after that launch has completed, and every other
 * earlier work on the stream completes before it starts. */
typedef struct {
  int32_t hidden;    /* H: model width (router and expert input/output size) */
  int32_t inter;     /* I: expert intermediate size (gate/up rows, down columns) */
  int32_t n_experts; /* E: routed experts (the shared expert is separate) */
  int32_t top_k;     /* k: routed experts per token */
} moe_dims;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,         /* a size or pointer is invalid */
  MOE_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than moe_workspace_bytes() */
  MOE_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
  MOE_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  MOE_ERR_DEVICE = 6,      /* a kernel found an inconsistent index */
  MOE_ERR_UNSUPPORTED = 7  /* not supported on this device (needs sm_100) */
} moe_status;

/* Router: w [n_experts, hidden] fp32; bias [n_experts] fp32 or NULL (no bias). */
typedef struct {
  const float *w;
  const float *bias;
} moe_router;

/* Routed experts: n_experts packed experts back to back, stride moe_packed_expert_bytes(). */
typedef struct {
  const void *packed;
} moe_experts;

/* The shared expert: one packed expert, applied to every token with weight 1. */
typedef struct {
  const void *packed;
} moe_shared;

/* ---- Q2 weights ------------------------------------------------------------
 * Canonical (input) format.  A block is 10 bytes: the fp16 scale d
 * (little-endian), then 8 code bytes; element j (0..31) is the 2-bit code
 * q = (code[j >> 2] >> (2*(j & 3))) & 3 and the weight is d * (q - 1)
 * ("affine, bias = -1" codebook, devlabs page, section 4).  One expert is three
 * row-major matrices back to back, blocks running along the contraction
 * dimension: gate [inter x hidden/32 blocks], up [inter x hidden/32],
 * down [hidden x inter/32].  moe_canonical_expert_bytes() gives its size.
 *
 * Packed format: the kernel layout written by moe_pack_q2; opaque to callers,
 * same number of bytes as the canonical format, padded to 256 bytes per expert. */

/* Host.  Bytes of one canonical expert (0 if dims are invalid). */
size_t moe_canonical_expert_bytes(const moe_dims *dims);
/* Host.  Bytes of one packed expert, the stride of moe_experts.packed (0 if invalid). */
size_t moe_packed_expert_bytes(const moe_dims *dims);

/* Repack n_experts canonical experts (device, back to back, stride
 * moe_canonical_expert_bytes) into the kernel layout (device, stride
 * moe_packed_expert_bytes).  packed_bytes is the size of the output buffer.
 * Untimed set-up step; canonical and packed must not overlap. */
moe_status moe_pack_q2(const moe_dims *dims, const void *canonical, int32_t n_experts, void *packed,
                       size_t packed_bytes, moe_stream_t stream);

/* ---- workspace --------------------------------------------------------------
 * Host.  Bytes of scratch memory moe_route / moe_layer_forward /
 * moe_experts_forward need for up to max_T tokens (0 if invalid).  Its first
 * 256 bytes hold the sticky device status word (offset 0) and the decode
 * kernel's grid-barrier arrival counter (offset 64): zero the workspace (or at
 * least those 256 bytes) once after allocating it, and again after a call reported
 * MOE_ERR_TIMEOUT.  One workspace must not be used by two calls that can run
 * at the same time.  A workspace of moe_workspace_bytes(dims, max_T) serves
 * every T <= max_T.  For T > 8 it also holds the router weights split into
 * three bf16 planes (3 * n_experts * hidden * 2 bytes) and the router's K-split
 * partial sums (at most 4.85 MB). */
size_t moe_workspace_bytes(const moe_dims *dims, int32_t max_T);

/* ---- routing ------------------------------------------------------------------
 * Every token goes to top_k of the n_experts routed experts (devlabs page,
 * section 1, "MoE 专家分流": 10 of 512; Strata tuning page, section 2 model
 * table).  The pages give no formula; this call computes, for each of T
 * tokens: logits[e] = sum_h x[h] Wr[e][h] + bias[e] (fp32 accumulation); the
 * top_k experts by logit, ties to the lower index, in descending-logit order;
 * weights = softmax over the selected logits (fp32), which is the full softmax
 * renormalised over the selected set.
 * x [T, hidden] bf16; topk_idx [T, top_k] int32 and topk_w [T, top_k] fp32 are
 * outputs.  T = 0 is a no-op. */
moe_status moe_route(const moe_dims *dims, const uint16_t *x, const moe_router *router, int32_t T,
                     int32_t *topk_idx, float *topk_w, void *workspace, size_t ws_bytes, moe_stream_t stream);

/* ---- routing without a workspace --------------------------------------------------
 * The paper has no counterpart to this entry point; it exists for callers of
 * this library that cannot allocate device memory: engines whose device
 * memory is reserved up front by their own pool, with nothing left to hand
 * out; plug-ins running inside a host framework that owns every device
 * allocation; and latency-bound loops that cannot afford an allocation's
 * implicit device synchronisation.
 * It computes what moe_route computes.  For T <= 8 it runs the same kernels
 * and returns identical results.  For more tokens moe_route's tcgen05 router
 * needs the split router weights in its workspace, so this entry point uses
 * the legacy-MMA router on the same exact weight split instead.  Its fp32
 * sums run in a different order, so near-tied logits may select or order
 * differently.  The scratch these kernels need -- the [T, n_experts] fp32
 * router logits -- lives in a file-scope device array of
 * MOE_NOALLOC_MAX_LOGITS floats (1 MiB) inside this library, which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * nothing.
 *  - T * n_experts > MOE_NOALLOC_MAX_LOGITS returns MOE_ERR_WORKSPACE.
 *  - The first call on each device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is kept together with the id of the CUDA context it was
 *    looked up in; after a device reset the first call in the new context
 *    looks it up again (so that call, too, should come before any capture).
 *  - All calls share the one array: calls that overlap on the GPU (different
 *    streams, or different host threads) race and may return each other's
 *    routing.  Nothing in the array needs to start at zero: every call
 *    rewrites the logits it reads.
 * Arguments as moe_route, minus the workspace. */
#define MOE_NOALLOC_MAX_LOGITS 262144
moe_status moe_route_noalloc(const moe_dims *dims, const uint16_t *x, const moe_router *router, int32_t T,
                             int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/* ---- the layer ------------------------------------------------------------------
 * The routed MoE FFN of the pages' model: top_k routed experts plus one shared
 * expert per token (Strata tuning page, section 2 model table: 512 routed,
 * top-10 + 1 shared), the experts computed straight from their 2-bit blocks
 * (strata-mlx page, "它是什么", first bullet):
 * out[t] = shared(x[t]) + sum_j w[t,j] * expert_{idx[t,j]}(x[t]), with
 * expert(v) = Wd (silu(Wg v) * (Wu v)) and silu(z) = z / (1 + exp(-z)).
 * Rounding points: x is bf16; every dot product accumulates in fp32; the
 * SwiGLU output h is rounded to bf16 before the down projection; the weighted
 * sum is fp32 and out is rounded to bf16 (nearest even).
 * x [T, hidden] bf16 in; out [T, hidden] bf16 out (must not overlap x).
 * topk_idx_out [T, top_k] / topk_w_out [T, top_k]: optional copies of the
 * routing decision (NULL to skip).  T = 0 is a no-op. */
moe_status moe_layer_forward(const moe_dims *dims, const uint16_t *x, const moe_router *router,
                             const moe_experts *experts, const moe_shared *shared, uint16_t *out, int32_t T,
                             int32_t *topk_idx_out, float *topk_w_out, void *workspace, size_t ws_bytes,
                             moe_stream_t stream);

/* ---- layer forward, token rows in host memory ----------------------------------
 * Host.  The layer of moe_layer_forward for a decode window (1 <= T <= 8)
 * whose token rows live in page-locked host memory, as in a serving loop that
 * hands the layer one window at a time: x_host [T, hidden] bf16 is read and
 * out_host [T, hidden] bf16 written by the library's own kernels over the
 * host link (zero-copy), in stream order with the layer, so that no copy call
 * of the caller's sits between them.  Both must be page-locked host memory
 * mapped into the device's address space (cudaHostAlloc / cudaMallocHost, or
 * cudaHostRegister with the mapped flag, on a unified-address system), each
 * range within one allocation, 16-byte aligned and not overlapping; anything
 * else returns MOE_ERR_ARG (MOE_ERR_ALIGN for alignment) before any launch,
 * as does T > 8.  The rows are staged in the workspace (moe_workspace_bytes
 * covers them).  out_host holds the result once the stream has passed this
 * call (e.g. after cudaStreamSynchronize).  Other arguments, the routing
 * copies and the errors are those of moe_layer_forward, whose output this
 * equals bit for bit. */
moe_status moe_layer_forward_host(const moe_dims *dims, const uint16_t *x_host, const moe_router *router,
                                  const moe_experts *experts, const moe_shared *shared, uint16_t *out_host,
                                  int32_t T, int32_t *topk_idx_out, float *topk_w_out, void *workspace,
                                  size_t ws_bytes, moe_stream_t stream);

/* One layer of a stack of layers (the pages' model stacks 48 of them, Strata
 * tuning page, section 2 model table), with the residual stream and the next
 * layer's normalisation done by the layer's own last kernel:
 *   y = the layer of moe_layer_forward applied to x_norm_in;
 *   resid += y                    (fp32; y is not rounded to bf16 on the way)
 *   x_norm_out = bf16(resid / sqrt(mean(resid^2) + eps))   (unit gain, nearest even)
 * resid [T, hidden] fp32 (in/out); x_norm_in / x_norm_out [T, hidden] bf16,
 * which must not overlap each other or resid.  A stack is
 *   moe_rmsnorm_residual(resid = x, NULL, x_norm);  then per layer
 *   moe_layer_forward_residual(layer, x_norm, resid, x_norm') with x_norm and
 *   x_norm' swapped between layers.
 * It equals moe_layer_forward followed by moe_rmsnorm_residual except that
 * the layer output reaches the residual unrounded, one launch fewer per
 * layer for T > 8 and one bf16 [T, hidden] round trip less.  eps >= 0.
 * Other arguments and errors as moe_layer_forward. */
moe_status moe_layer_forward_residual(const moe_dims *dims, const uint16_t *x_norm_in, const moe_router *router,
                                      const moe_experts *experts, const moe_shared *shared, float *resid,
                                      uint16_t *x_norm_out, float eps, int32_t T, int32_t *topk_idx_out,
                                      float *topk_w_out, void *workspace, size_t ws_bytes, moe_stream_t stream);

/* The expert half of the layer (the same model table: routed experts plus one
 * shared expert, computed from their 2-bit blocks) for a routing decision made
 * elsewhere:
 * dispatch (per-expert counts, offsets, stable token permutation), the routed
 * and shared SwiGLU experts and the weighted combine, with the rounding points
 * of moe_layer_forward.  topk_idx [T, top_k] int32 (each in [0, n_experts),
 * distinct per token) and topk_w [T, top_k] fp32 are inputs; an index out of
 * range sets MOE_ERR_DEVICE in the workspace status and that slot is skipped.
 * moe_layer_forward == moe_route followed by this call. */
moe_status moe_experts_forward(const moe_dims *dims, const uint16_t *x, const int32_t *topk_idx,
                               const float *topk_w, const moe_experts *experts, const moe_shared *shared,
                               uint16_t *out, int32_t T, void *workspace, size_t ws_bytes, moe_stream_t stream);

/* The dispatch step on its own, for a routing made elsewhere (the step the
 * expert half of the layer starts with): the token-to-expert histogram, its
 * exclusive scan and the stable permutation that groups the routed slots by
 * expert.  Each token is routed to top_k experts (Strata tuning page, section
 * 2 model table: 10 of 512 per token), so there are T * top_k slots; slot
 * s = t * top_k + j holds topk_idx[t][j].  Outputs (device, int32):
 *   counts [n_experts]      slots routed to each expert;
 *   offsets [n_experts + 1] exclusive prefix sum of counts, offsets[n_experts] = T * top_k;
 *   perm [T * top_k]        the slot at each sorted position: experts in ascending order, and within an
 *                           expert the slots in ascending order (a stable sort of the slots by expert);
 *   inv [T * top_k]         the sorted position of each slot (perm[inv[s]] == s).
 * Indices must lie in [0, n_experts) and be distinct within a token; a slot
 * with an index out of range sets MOE_ERR_DEVICE in the workspace status, is
 * left out of the counts and gets inv = -1.  The workspace is the one
 * moe_layer_forward takes (moe_workspace_bytes(dims, T) bytes). */
moe_status moe_dispatch(const moe_dims *dims, const int32_t *topk_idx, int32_t T, int32_t *counts,
                        int32_t *offsets, int32_t *perm, int32_t *inv, void *workspace, size_t ws_bytes,
                        moe_stream_t stream);

/* ---- between layers (a stack of layers) -------------------------------------------
 * resid [T, hidden] fp32 (in/out), y [T, hidden] bf16 (may be NULL),
 * x_norm [T, hidden] bf16 (out):
 *   if y: resid += y;  then  x_norm = bf16(resid / sqrt(mean(resid^2) + eps)).
 * Unit gain.  Used as x_{l+1} = x_l + MoE_l(RMSNorm(x_l)). */
moe_status moe_rmsnorm_residual(float *resid, const uint16_t *y, uint16_t *x_norm, int32_t T, int32_t hidden,
                                float eps, moe_stream_t stream);

/* ---- profiling aid ------------------------------------------------------------------
 * While kernel_id >= 0, every later call made by this host thread records the
 * CUDA event `before` (a cudaEvent_t created by the caller) on its stream just
 * before it launches kernel `kernel_id`, and `after` just after.  While the
 * stream is being captured into a CUDA graph the records are external event
 * records, so they become nodes of the graph; otherwise they are ordinary
 * records.  kernel_id < 0 turns this off.  The setting is per host thread.  The kernel
 * ids below name the library's kernels and may change between versions. */
enum {
  MOE_KERNEL_ROUTER_LOGITS = 0,
  MOE_KERNEL_TOPK = 1,
  MOE_KERNEL_DISPATCH_BITS = 2,
  MOE_KERNEL_DISPATCH_SCAN = 3,
  MOE_KERNEL_DISPATCH_PLACE = 4,
  MOE_KERNEL_GATE_UP = 5,
  MOE_KERNEL_DOWN = 6,
  MOE_KERNEL_COMBINE = 7,
  MOE_KERNEL_DECODE_FUSED = 8,
  MOE_KERNEL_GATHER = 9
};
moe_status moe_trace_kernel(int32_t kernel_id, void *before, void *after);

/* ---- per-expert kernel choice in a prefill chunk ---------------------------------------
 * Verify windows hold a few tokens (devlabs page, section 1; Strata tuning
 * page, sections 5 and 8: --spec 4/6/8), and in a prefill chunk with a skewed
 * router many experts get only a few tokens.  In a chunk of T > 8 tokens,
 * experts routed at most max_tokens tokens run on the register-dequant expert
 * kernels (8-token items) and the others, with the shared expert, on the
 * tcgen05 kernels.  The setting is per host thread; 0 (the default) sends
 * every expert to the tcgen05 kernels.  Measured on B200 (hidden 2048, 512
 * experts, Zipf router): any max_tokens > 0 was slower at every T from 16 to
 * 1024, because one tcgen05 work item costs less than one register-dequant
 * item even for a one-token expert; keep 0 unless measurement on another shape
 * says otherwise.  0 <= max_tokens <= 64, else MOE_ERR_ARG. */
moe_status moe_set_cold_expert_tokens(int32_t max_tokens);

/* ---- status ----------------------------------------------------------------------
 * Blocking host call: waits for `stream`, reads and clears the sticky device
 * status word in `workspace`; MOE_OK, MOE_ERR_DEVICE or MOE_ERR_TIMEOUT. */
moe_status moe_check_status(void *workspace, moe_stream_t stream);

/* Host.  Static string for a status code. */
const char *moe_status_str(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_Q2_H */
