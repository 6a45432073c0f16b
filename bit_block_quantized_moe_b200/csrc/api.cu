// C ABI entry points: host-side argument checks, workspace layout, launch order.
#include <stdio.h>

#include "kernels.cuh"

namespace moe {

// The limits the header states: hidden and inter multiples of 128 (the packed layout's 128-wide block groups
// along K) up to 4096; 1 <= top_k <= min(n_experts, 32) (one warp lane per selected expert); n_experts up to
// 65535.
static bool dims_ok(const moe_dims *d) {
  if (!d) return false;
  if (d->hidden < 128 || d->hidden > 4096 || d->hidden % 128) return false;
  if (d->inter < 128 || d->inter > 4096 || d->inter % 128) return false;
  if (d->n_experts < 1 || d->n_experts > 65535) return false;
  if (d->top_k < 1 || d->top_k > d->n_experts || d->top_k > 32) return false;
  return true;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static int max_items_for(const moe_dims &d, int T, int tile) {
  const long long routed = (long long)T * d.top_k;
  const long long touched = routed < d.n_experts ? routed : d.n_experts;
  return (int)(touched + (routed + tile - 1) / tile + (T + tile - 1) / tile);
}

// Lays out the workspace for T tokens; returns the bytes needed.  With base ==
// nullptr only the size is computed.
size_t workspace_layout(const moe_dims &d, int T, void *base, Workspace *ws) {
  const int E = d.n_experts, k = d.top_k, H = d.hidden, I = d.inter;
  const size_t words = (size_t)((T + 31) / 32);
  const size_t slots = (size_t)T * k + T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_hdr = take(256);                          // status, counters
  const size_t o_bitmap = take((size_t)E * words * 4);    // cleared each call, together with the counters below
  const size_t o_zero_tail = take(256);                    // end of the range the router clears
  const size_t o_wprefix = take((size_t)E * words * 4);
  const size_t o_counts = take((size_t)E * 4);
  const size_t o_offsets = take((size_t)(E + 1) * 4);
  const size_t o_logits = take((size_t)T * E * 4);
  const size_t o_idx = take((size_t)T * k * 4);
  const size_t o_w = take((size_t)T * k * 4);
  const size_t o_slot = take((size_t)T * k * 4);
  const size_t o_stok = take(slots * 4);
  const size_t o_sw = take(slots * 4);
  const int max_items = max_items_for(d, T, 8);
  const size_t o_items = take((size_t)max_items * 16);
  const int tc_n = tc_item_tokens(d, T);
  const int max_tc_items = max_items_for(d, T, tc_n);
  const size_t o_tc_items = take((size_t)max_tc_items * 16);
  const size_t o_xs = take(T > 8 ? slots * H * 2 : 0);
  const size_t o_h = take(slots * I * 2);
  const size_t o_y = take(slots * H * 4);
  const bool fused = decode_fused_supported(d, T);
  const size_t o_ready = take(fused ? decode_counter_words(d) * 4 : 0);
  const size_t o_part = take(fused ? decode_partial_floats(d, T) * 4 : 0);
  const bool rtc = router_tc_supported(d, T);
  const size_t o_wsplit = take(rtc ? (size_t)3 * E * H * 2 : 0);
  // sized by the bound on every T (the split count falls as T grows), so that a workspace sized for max_T fits
  const size_t o_rpart = take(rtc ? router_tc_partial_bytes_max() : 0);
  const size_t host_rows = (size_t)(T < kHostIoMaxTokens ? T : kHostIoMaxTokens) * H * 2;
  const size_t o_hx = take(host_rows), o_hy = take(host_rows);
  if (base && ws) {
    uint8_t *b = static_cast<uint8_t *>(base);
    ws->status = reinterpret_cast<uint32_t *>(b + o_hdr);
    ws->n_items = reinterpret_cast<uint32_t *>(b + o_hdr + 4);
    ws->bitmap = reinterpret_cast<uint32_t *>(b + o_bitmap);
    ws->zero_begin = ws->bitmap;
    ws->zero_words = (o_zero_tail + 4 - o_bitmap) / 4;
    ws->wprefix = reinterpret_cast<uint32_t *>(b + o_wprefix);
    ws->counts = reinterpret_cast<int32_t *>(b + o_counts);
    ws->offsets = reinterpret_cast<int32_t *>(b + o_offsets);
    ws->logits = reinterpret_cast<float *>(b + o_logits);
    ws->idx = reinterpret_cast<int32_t *>(b + o_idx);
    ws->w = reinterpret_cast<float *>(b + o_w);
    ws->slot_pos = reinterpret_cast<int32_t *>(b + o_slot);
    ws->perm = nullptr;
    ws->sorted_tok = reinterpret_cast<int32_t *>(b + o_stok);
    ws->sorted_w = reinterpret_cast<float *>(b + o_sw);
    ws->items = reinterpret_cast<int4 *>(b + o_items);
    ws->tc_items = reinterpret_cast<int4 *>(b + o_tc_items);
    ws->n_tc_items = reinterpret_cast<uint32_t *>(b + o_hdr + 8);
    ws->xs = reinterpret_cast<uint16_t *>(b + o_xs);
    ws->max_tc_items = max_tc_items;
    ws->tc_item_tokens = tc_n;
    ws->h = reinterpret_cast<uint16_t *>(b + o_h);
    ws->y = reinterpret_cast<float *>(b + o_y);
    ws->gbar = reinterpret_cast<uint64_t *>(b + o_hdr + 64);
    ws->ready = reinterpret_cast<uint32_t *>(b + o_ready);
    ws->partial = reinterpret_cast<float *>(b + o_part);
    ws->wsplit = rtc ? reinterpret_cast<uint16_t *>(b + o_wsplit) : nullptr;
    ws->rpart = reinterpret_cast<float *>(b + o_rpart);
    ws->host_x = reinterpret_cast<uint16_t *>(b + o_hx);
    ws->host_y = reinterpret_cast<uint16_t *>(b + o_hy);
    ws->words = (int)words;
    ws->max_items = max_items;
  }
  return off;
}

static thread_local int g_trace_id = -1;
static thread_local cudaEvent_t g_trace_ev[2] = {nullptr, nullptr};

// Inside stream capture the event becomes an external event node of the graph;
// outside it is an ordinary record (the external flag is only valid while capturing).
void trace_mark(int id, bool after, cudaStream_t s) {
  if (id != g_trace_id || !g_trace_ev[after ? 1 : 0]) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return;
  cudaEventRecordWithFlags(g_trace_ev[after ? 1 : 0], s,
                           cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault);
}

static moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

static moe_status device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MOE_ERR_CUDA;
  return major == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_canonical_expert_bytes(const moe_dims *dims) {
  if (!dims_ok(dims)) return 0;
  return (size_t)3 * dims->hidden * dims->inter / kQBlock * kCanonBlockBytes;
}

size_t moe_packed_expert_bytes(const moe_dims *dims) {
  if (!dims_ok(dims)) return 0;
  return packed_geom(dims->hidden, dims->inter).expert_bytes;
}

size_t moe_workspace_bytes(const moe_dims *dims, int32_t max_T) {
  if (!dims_ok(dims) || max_T < 0) return 0;
  // enough for every T <= max_T (the small-T layout carries the fused-decode regions)
  size_t need = workspace_layout(*dims, max_T, nullptr, nullptr);
  for (int t = 1; t <= 8 && t <= max_T; ++t) {
    const size_t n = workspace_layout(*dims, t, nullptr, nullptr);
    need = n > need ? n : need;
  }
  return need;
}

moe_status moe_pack_q2(const moe_dims *dims, const void *canonical, int32_t n_experts, void *packed,
                       size_t packed_bytes, moe_stream_t stream) {
  if (!dims_ok(dims) || n_experts < 0) return MOE_ERR_ARG;
  if (n_experts == 0) return MOE_OK;
  if (!canonical || !packed) return MOE_ERR_ARG;
  if (!aligned16(packed)) return MOE_ERR_ALIGN;
  const PackedGeom G = packed_geom(dims->hidden, dims->inter);
  if (packed_bytes < (size_t)n_experts * G.expert_bytes) return MOE_ERR_ARG;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  return cuda_status(launch_pack(static_cast<const uint8_t *>(canonical), static_cast<uint8_t *>(packed), n_experts,
                                 G, moe_canonical_expert_bytes(dims), reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_route(const moe_dims *dims, const uint16_t *x, const moe_router *router, int32_t T,
                     int32_t *topk_idx, float *topk_w, void *workspace, size_t ws_bytes, moe_stream_t stream) {
  if (!dims_ok(dims) || T < 0 || !router) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !router->w || !topk_idx || !topk_w || !workspace) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(router->w) || !aligned16(workspace)) return MOE_ERR_ALIGN;
  if (ws_bytes < workspace_layout(*dims, T, nullptr, nullptr)) return MOE_ERR_WORKSPACE;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  ws.idx = topk_idx;
  ws.w = topk_w;
  return cuda_status(launch_route(*dims, x, router->w, router->bias, T, ws, false,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

static moe_status check_layer_args(const moe_dims *dims, const uint16_t *x, const moe_experts *experts,
                                   const moe_shared *shared, const uint16_t *out, int32_t T, void *workspace,
                                   size_t ws_bytes) {
  if (!dims_ok(dims) || T < 0 || !experts || !shared) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !out || !experts->packed || !shared->packed || !workspace) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned16(experts->packed) || !aligned16(shared->packed) ||
      !aligned16(workspace))
    return MOE_ERR_ALIGN;
  const size_t xb = (size_t)T * dims->hidden * 2;
  const uintptr_t xo = (uintptr_t)x, oo = (uintptr_t)out;
  if (xo < oo + xb && oo < xo + xb) return MOE_ERR_ARG;  // out overlaps x
  if (ws_bytes < workspace_layout(*dims, T, nullptr, nullptr)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Where the layer output goes: bf16 rows `out`, or (resid set) added in fp32 to the residual, whose RMSNorm
// becomes the next layer's bf16 input x_norm.
struct LayerOut {
  uint16_t *out = nullptr;
  float *resid = nullptr;
  uint16_t *x_norm = nullptr;
  float eps = 0.f;
};

// Dispatch, experts and combine for a routing already in ws.idx / ws.w.
static cudaError_t run_experts(const moe_dims &d, const uint16_t *x, const moe_experts *experts,
                               const moe_shared *shared, const LayerOut &lo, int T, Workspace &ws, cudaStream_t s,
                               bool bits_ready) {
  const PackedGeom G = packed_geom(d.hidden, d.inter);
  cudaError_t err = cudaSuccess;
  if (!bits_ready) err = launch_dispatch_bits(d, T, ws, s);
  if (err == cudaSuccess) err = launch_dispatch(d, T, ws, s);
  if (err == cudaSuccess) {
    const uint8_t *ex = static_cast<const uint8_t *>(experts->packed);
    const uint8_t *sh = static_cast<const uint8_t *>(shared->packed);
    // few tokens: register-dequant tensor-core tiles of 8 tokens; otherwise the tcgen05 grouped GEMM
    err = T <= 8 ? launch_experts(d, G, ex, sh, x, T, ws, s) : launch_tc_experts(d, G, ex, sh, x, T, ws, s);
  }
  if (err == cudaSuccess)
    err = lo.resid ? launch_combine_rmsnorm(d, T, ws, lo.resid, lo.x_norm, lo.eps, s) : launch_combine(d, T, ws, lo.out, s);
  return err;
}

// The layer for x (routing, experts, combine) into `lo`.
static cudaError_t run_layer(const moe_dims &d, const uint16_t *x, const moe_router *router,
                             const moe_experts *experts, const moe_shared *shared, const LayerOut &lo, int T,
                             int32_t *topk_idx_out, float *topk_w_out, Workspace &ws, cudaStream_t s) {
  if (topk_idx_out) ws.idx = topk_idx_out;
  if (topk_w_out) ws.w = topk_w_out;
  if (decode_fused_supported(d, T)) {
    // The fused kernel writes the routing copies as a pair (both pointers or neither): when only one is
    // requested, the other goes to the workspace's own [T, top_k] buffer.
    const bool copies = topk_idx_out || topk_w_out;
    // with a residual the fused kernel leaves the fp32 layer output in the workspace's expert-output rows
    cudaError_t err = launch_decode_fused(d, x, router->w, router->bias, static_cast<const uint8_t *>(experts->packed),
                                          static_cast<const uint8_t *>(shared->packed), T, ws,
                                          copies ? ws.idx : nullptr, copies ? ws.w : nullptr,
                                          lo.resid ? nullptr : lo.out, lo.resid ? ws.y : nullptr, s);
    if (err == cudaSuccess && lo.resid) err = launch_rmsnorm_residual_f32(lo.resid, ws.y, lo.x_norm, T, d.hidden, lo.eps, s);
    return err;
  }
  cudaError_t err = launch_route(d, x, router->w, router->bias, T, ws, true, s);
  if (err == cudaSuccess) err = run_experts(d, x, experts, shared, lo, T, ws, s, true);
  return err;
}

moe_status moe_layer_forward(const moe_dims *dims, const uint16_t *x, const moe_router *router,
                             const moe_experts *experts, const moe_shared *shared, uint16_t *out, int32_t T,
                             int32_t *topk_idx_out, float *topk_w_out, void *workspace, size_t ws_bytes,
                             moe_stream_t stream) {
  if (!router) return MOE_ERR_ARG;
  moe_status st = check_layer_args(dims, x, experts, shared, out, T, workspace, ws_bytes);
  if (st != MOE_OK || T == 0) return st;
  if (!router->w) return MOE_ERR_ARG;
  if (!aligned16(router->w)) return MOE_ERR_ALIGN;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  LayerOut lo;
  lo.out = out;
  return cuda_status(run_layer(*dims, x, router, experts, shared, lo, T, topk_idx_out, topk_w_out, ws, s));
}

moe_status moe_layer_forward_host(const moe_dims *dims, const uint16_t *x_host, const moe_router *router,
                                  const moe_experts *experts, const moe_shared *shared, uint16_t *out_host,
                                  int32_t T, int32_t *topk_idx_out, float *topk_w_out, void *workspace,
                                  size_t ws_bytes, moe_stream_t stream) {
  if (!router) return MOE_ERR_ARG;
  moe_status st = check_layer_args(dims, x_host, experts, shared, out_host, T, workspace, ws_bytes);
  if (st != MOE_OK || T == 0) return st;
  if (T > kHostIoMaxTokens || !router->w) return MOE_ERR_ARG;
  if (!aligned16(router->w)) return MOE_ERR_ALIGN;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  const size_t rows = (size_t)T * dims->hidden * 2;
  void *xd = mapped_host_range(x_host, rows), *od = mapped_host_range(out_host, rows);
  if (!xd || !od) return MOE_ERR_ARG;  // not page-locked, device-mapped host memory: nothing launched
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  LayerOut lo;
  lo.out = ws.host_y;
  cudaError_t err = launch_stream_copy16(xd, ws.host_x, rows, s);
  if (err == cudaSuccess)
    err = run_layer(*dims, ws.host_x, router, experts, shared, lo, T, topk_idx_out, topk_w_out, ws, s);
  if (err == cudaSuccess) err = launch_stream_copy16(ws.host_y, od, rows, s);
  return cuda_status(err);
}

static bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

moe_status moe_layer_forward_residual(const moe_dims *dims, const uint16_t *x_norm_in, const moe_router *router,
                                      const moe_experts *experts, const moe_shared *shared, float *resid,
                                      uint16_t *x_norm_out, float eps, int32_t T, int32_t *topk_idx_out,
                                      float *topk_w_out, void *workspace, size_t ws_bytes, moe_stream_t stream) {
  if (!router || !(eps >= 0.f)) return MOE_ERR_ARG;
  moe_status st = check_layer_args(dims, x_norm_in, experts, shared, x_norm_out, T, workspace, ws_bytes);
  if (st != MOE_OK || T == 0) return st;
  if (!router->w || !resid) return MOE_ERR_ARG;
  if (!aligned16(router->w) || !aligned16(resid)) return MOE_ERR_ALIGN;
  const size_t xb = (size_t)T * dims->hidden * 2, rb = (size_t)T * dims->hidden * 4;
  if (overlaps(resid, rb, x_norm_in, xb) || overlaps(resid, rb, x_norm_out, xb)) return MOE_ERR_ARG;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  LayerOut lo;
  lo.resid = resid;
  lo.x_norm = x_norm_out;
  lo.eps = eps;
  return cuda_status(run_layer(*dims, x_norm_in, router, experts, shared, lo, T, topk_idx_out, topk_w_out, ws, s));
}

moe_status moe_experts_forward(const moe_dims *dims, const uint16_t *x, const int32_t *topk_idx,
                               const float *topk_w, const moe_experts *experts, const moe_shared *shared,
                               uint16_t *out, int32_t T, void *workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_layer_args(dims, x, experts, shared, out, T, workspace, ws_bytes);
  if (st != MOE_OK || T == 0) return st;
  if (!topk_idx || !topk_w) return MOE_ERR_ARG;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  ws.idx = const_cast<int32_t *>(topk_idx);
  ws.w = const_cast<float *>(topk_w);
  LayerOut lo;
  lo.out = out;
  return cuda_status(run_experts(*dims, x, experts, shared, lo, T, ws, s, false));
}

moe_status moe_dispatch(const moe_dims *dims, const int32_t *topk_idx, int32_t T, int32_t *counts,
                        int32_t *offsets, int32_t *perm, int32_t *inv, void *workspace, size_t ws_bytes,
                        moe_stream_t stream) {
  if (!dims_ok(dims) || T < 0) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !counts || !offsets || !perm || !inv || !workspace) return MOE_ERR_ARG;
  if (!aligned16(workspace)) return MOE_ERR_ALIGN;
  if (ws_bytes < workspace_layout(*dims, T, nullptr, nullptr)) return MOE_ERR_WORKSPACE;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace ws;
  workspace_layout(*dims, T, workspace, &ws);
  ws.idx = const_cast<int32_t *>(topk_idx);
  ws.counts = counts;
  ws.offsets = offsets;
  ws.slot_pos = inv;
  ws.perm = perm;
  cudaError_t err = launch_dispatch_bits(*dims, T, ws, s);
  if (err == cudaSuccess) err = launch_dispatch(*dims, T, ws, s);
  return cuda_status(err);
}

moe_status moe_rmsnorm_residual(float *resid, const uint16_t *y, uint16_t *x_norm, int32_t T, int32_t hidden,
                                float eps, moe_stream_t stream) {
  if (T < 0 || hidden < 1 || !(eps >= 0.f)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!resid || !x_norm) return MOE_ERR_ARG;
  const moe_status dev = device_ok();
  if (dev != MOE_OK) return dev;
  return cuda_status(
      launch_rmsnorm_residual(resid, y, x_norm, T, hidden, eps, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_trace_kernel(int32_t kernel_id, void *before, void *after) {
  if (kernel_id >= 0 && (!before || !after)) return MOE_ERR_ARG;
  g_trace_id = kernel_id < 0 ? -1 : kernel_id;
  g_trace_ev[0] = static_cast<cudaEvent_t>(before);
  g_trace_ev[1] = static_cast<cudaEvent_t>(after);
  return MOE_OK;
}

moe_status moe_set_cold_expert_tokens(int32_t max_tokens) {
  if (max_tokens < 0 || max_tokens > 64) return MOE_ERR_ARG;
  set_cold_expert_tokens(max_tokens);
  return MOE_OK;
}

moe_status moe_check_status(void *workspace, moe_stream_t stream) {
  if (!workspace) return MOE_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (word && cudaMemsetAsync(workspace, 0, sizeof word, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (word & kStatusBadIndex) return MOE_ERR_DEVICE;
  return MOE_OK;
}

const char *moe_status_str(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument";
    case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE: return "device found an inconsistent index";
    case MOE_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.x)";
  }
  return "unknown status";
}

}  // extern "C"
