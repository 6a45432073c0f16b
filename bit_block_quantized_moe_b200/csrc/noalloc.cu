// moe_route_noalloc: routing for callers that cannot allocate device memory.
//
// The router and top-k kernels of moe_route (for more than 8 tokens the
// legacy-MMA router, since the tcgen05 one keeps its split weights in the
// workspace), but the scratch they need (the [T, n_experts] fp32 router
// logits) is a file-scope device array of this library instead of a
// caller-provided workspace.  Every GPU that loads the library holds the
// array until the process exits.
#include <mutex>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr size_t kNoAllocLogits = MOE_NOALLOC_MAX_LOGITS;  // 1 MiB of fp32 logits
static __device__ __align__(256) float g_noalloc_logits[kNoAllocLogits];

constexpr int kMaxDevices = 64;
std::mutex g_lookup_mutex;
float *g_scratch[kMaxDevices];  // device address of the array, looked up once per device

// The array's name is only a host-side stand-in in host code; the kernels get
// its device address, looked up once per device with that device current.
cudaError_t scratch_for_current_device(float **out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_lookup_mutex);
  if (!g_scratch[dev]) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_logits);
    if (err != cudaSuccess) return err;
    g_scratch[dev] = static_cast<float *>(p);
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

bool noalloc_dims_ok(const moe_dims *d) {
  if (!d) return false;
  if (d->hidden < 128 || d->hidden > 4096 || d->hidden % 128) return false;
  if (d->inter < 128 || d->inter > 4096 || d->inter % 128) return false;
  if (d->n_experts < 1 || d->n_experts > 4096) return false;
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
