// Internal launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include "common.cuh"

namespace moe {

// Workspace regions for one moe_layer_forward / moe_route call (device pointers).
struct Workspace {
  uint32_t *status;        // sticky status word
  uint32_t *zero_begin;    // [zero_begin, zero_begin + zero_words) is cleared by the router kernel
  size_t zero_words;
  uint32_t *n_items;
  uint32_t *bitmap;        // [E][words] token-membership bits per expert (inside the zeroed range)
  uint32_t *wprefix;       // [E][words] exclusive popcount prefix per word
  int32_t *counts;         // [E]
  int32_t *offsets;        // [E + 1]
  float *logits;           // [T][E]
  int32_t *idx;            // [T][k]
  float *w;                // [T][k]
  int32_t *slot_pos;       // [T*k]: sorted position of slot (t, j)
  int32_t *perm;           // optional [T*k]: slot t*k + j at each sorted position (moe_dispatch only)
  int32_t *sorted_tok;     // [T*k + T]: token of each sorted position (shared slots last)
  float *sorted_w;         // [T*k + T]
  int4 *items;             // [max_items]: (expert, first position, tokens <= 8, 0)
  int4 *tc_items;          // [max_tc_items]: (expert, first position, tokens <= tc_item_tokens, 0)
  uint32_t *n_tc_items;
  uint16_t *xs;            // [T*k + T][H] bf16 token rows in sorted-position order
  uint16_t *h;             // [T*k + T][I] bf16 SwiGLU outputs by sorted position
  float *y;                // [T*k + T][H] fp32 expert outputs by sorted position
  uint64_t *gbar;          // grid barrier of the fused decode kernel: monotonic arrival counter
  uint32_t *ready;         // fused decode: per-entry ready counters (finished gate/up units)
  float *partial;          // fused decode: per (expert, tile) partial outputs
  uint16_t *wsplit;        // tcgen05 router: [3][E][H] bf16 planes of the router weights (null: legacy router)
  float *rpart;            // tcgen05 router: [ksplit][T][E] K-split partial logits (ksplit > 1)
  uint16_t *host_x;        // moe_layer_forward_host: [min(T, 8)][H] bf16 token rows staged from host memory
  uint16_t *host_y;        // moe_layer_forward_host: [min(T, 8)][H] bf16 layer output staged for host memory
  int words;               // ceil(T / 32)
  int max_items;
  int max_tc_items;
  int tc_item_tokens;       // 64 or 128 (tc_item_tokens())
};

// Profiling hook (moe_trace_kernel): records the caller's events around kernel `id`.
void trace_mark(int id, bool after, cudaStream_t s);

size_t workspace_layout(const moe_dims &d, int T, void *base, Workspace *ws);

cudaError_t launch_pack(const uint8_t *canon, uint8_t *packed, int n_experts, const PackedGeom &G,
                        size_t canon_stride, cudaStream_t s);
cudaError_t launch_route(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias, int T,
                         const Workspace &ws, bool with_dispatch_bits, cudaStream_t s);
cudaError_t launch_dispatch_bits(const moe_dims &d, int T, const Workspace &ws, cudaStream_t s);
cudaError_t launch_dispatch(const moe_dims &d, int T, const Workspace &ws, cudaStream_t s);
cudaError_t launch_experts(const moe_dims &d, const PackedGeom &G, const uint8_t *experts, const uint8_t *shared,
                           const uint16_t *x, int T, const Workspace &ws, cudaStream_t s);
// Tokens per tcgen05 prefill work item for T tokens (64, or 128 once an expert averages 64 tokens).
int tc_item_tokens(const moe_dims &d, int T);
// In a prefill chunk (T > 8), experts with at most this many tokens run on the register-dequant expert
// kernels instead of the tcgen05 ones (0: none).
int cold_expert_tokens(const moe_dims &d, int T);
void set_cold_expert_tokens(int n);
cudaError_t launch_tc_experts(const moe_dims &d, const PackedGeom &G, const uint8_t *experts, const uint8_t *shared,
                              const uint16_t *x, int T, const Workspace &ws, cudaStream_t s);
cudaError_t launch_combine(const moe_dims &d, int T, const Workspace &ws, uint16_t *out, cudaStream_t s);
bool decode_fused_supported(const moe_dims &d, int T);
size_t decode_partial_floats(const moe_dims &d, int T);
size_t decode_counter_words(const moe_dims &d);
cudaError_t launch_decode_fused(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias,
                                const uint8_t *experts, const uint8_t *shared, int T, const Workspace &ws,
                                int32_t *idx_out, float *w_out, uint16_t *out, float *out_f32, cudaStream_t s);
bool router_tc_supported(const moe_dims &d, int T);
int router_tc_ksplit(const moe_dims &d, int T);
size_t router_tc_partial_bytes_max();
cudaError_t launch_router_tc(const moe_dims &d, const uint16_t *x, const float *Wr, const float *bias, int T,
                             const Workspace &ws, cudaStream_t s);
cudaError_t launch_rmsnorm_residual(float *resid, const uint16_t *y, uint16_t *x_norm, int T, int H, float eps,
                                    cudaStream_t s);
cudaError_t launch_rmsnorm_residual_f32(float *resid, const float *y, uint16_t *x_norm, int T, int H, float eps,
                                        cudaStream_t s);
cudaError_t launch_combine_rmsnorm(const moe_dims &d, int T, const Workspace &ws, float *resid, uint16_t *x_norm,
                                   float eps, cudaStream_t s);
// Host-memory token rows (hostio.cu): a one-kernel 16-byte copy in stream order (programmatic dependent launch,
// nothing touched before the wait), and the device address of a page-locked, device-mapped host range.
constexpr int kHostIoMaxTokens = 8;
cudaError_t launch_stream_copy16(const void *src, void *dst, size_t bytes, cudaStream_t s);
void *mapped_host_range(const void *p, size_t bytes);

}  // namespace moe
