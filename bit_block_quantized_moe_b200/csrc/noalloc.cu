// moe_route_noalloc: routing for callers that cannot allocate device memory.
//
// The router and top-k kernels of moe_route (for more than 8 tokens the
// legacy-MMA router, since the tcgen05 one keeps its split weights in the
// workspace), but the scratch they need (the [T, n_experts] fp32 router
// logits) is a file-scope device array of this library instead of a
// caller-provided workspace.  Every GPU that loads the library holds the
// array until the process exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr size_t kNoAllocLogits = MOE_NOALLOC_MAX_LOGITS;  // 1 MiB of fp32 logits
static __device__ __align__(256) float g_noalloc_logits[kNoAllocLogits];

constexpr int kMaxDevices = 64;

// Device address of the array, looked up with the device current and kept per
// device together with the id of the CUDA context it belongs to: a device
// reset ends that context (and the module image holding the array), so a call
// made in a new context looks the address up again.
struct ScratchAddr {
  unsigned long long ctx_id = 0;
  float *ptr = nullptr;
};
std::mutex g_lookup_mutex;
ScratchAddr g_scratch[kMaxDevices];

// Driver entry points for the current context's id (through the runtime, so
// the library needs no link against the driver library).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
  bool ok = false;
};
const CtxFns &ctx_fns() {
  static CtxFns f = [] {
    CtxFns r;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      r.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      r.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    r.ok = r.get_current && r.get_id;
    return r;
  }();
  return f;
}

cudaError_t current_ctx_id(unsigned long long *id) {
  const CtxFns &f = ctx_fns();
  if (!f.ok) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
  return f.get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// The array's name is only a host-side stand-in in host code; the kernels get
// its device address, looked up once per device and context with that device
// current.
cudaError_t scratch_for_current_device(float **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_lookup_mutex);
  unsigned long long id = 0;
  // With no context current yet, the lookup below creates the device's primary context.
  const bool have_ctx = current_ctx_id(&id) == cudaSuccess;
  ScratchAddr &s = g_scratch[dev];
  if (!have_ctx || !s.ptr || s.ctx_id != id) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_logits);
    if (err != cudaSuccess) return err;
    err = current_ctx_id(&id);
    if (err != cudaSuccess) return err;
    s.ptr = static_cast<float *>(p);
    s.ctx_id = id;
  }
  *out = s.ptr;
  return cudaSuccess;
}

bool noalloc_dims_ok(const moe_dims *d) {
  if (!d) return false;
  if (d->hidden < 128 || d->hidden > 4096 || d->hidden % 128) return false;
  if (d->inter < 128 || d->inter > 4096 || d->inter % 128) return false;
  if (d->n_experts < 1 || d->n_experts > 65535) return false;
  if (d->top_k < 1 || d->top_k > d->n_experts || d->top_k > 32) return false;
  return true;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_noalloc(const moe_dims *dims, const uint16_t *x, const moe_router *router,
                                        int32_t T, int32_t *topk_idx, float *topk_w, moe_stream_t stream) {
  if (!noalloc_dims_ok(dims) || T < 0 || !router) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !router->w || !topk_idx || !topk_w) return MOE_ERR_ARG;
  if (((uintptr_t)x & 15u) || ((uintptr_t)router->w & 15u)) return MOE_ERR_ALIGN;
  if ((size_t)T * (size_t)dims->n_experts > kNoAllocLogits) return MOE_ERR_WORKSPACE;  // beyond the static scratch
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  float *logits = nullptr;
  if (scratch_for_current_device(&logits) != cudaSuccess) return MOE_ERR_CUDA;
  // The logits are rewritten in full by every call: nothing needs clearing.
  Workspace ws{};
  ws.logits = logits;
  ws.idx = topk_idx;
  ws.w = topk_w;
  ws.zero_begin = nullptr;
  ws.zero_words = 0;
  ws.bitmap = nullptr;
  ws.words = 0;
  return launch_route(*dims, x, router->w, router->bias, T, ws, false, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
