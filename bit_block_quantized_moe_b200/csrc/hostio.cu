// Token rows in and layer output out through page-locked host memory, for
// moe_layer_forward_host: two one-CTA copy kernels that read and write the
// host buffers over the host link (device-mapped pinned memory, zero-copy) in
// stream order with the layer's own kernels.
//
// Both are launched as programmatic dependents of whatever precedes them on
// the stream, and release their own dependents at once: the copy-in's launch
// and the fused decode kernel's set-up (router rows, shared-expert prefetch)
// overlap the previous work, the copy-out is resident and waiting when the
// layer ends.  Neither touches memory before griddepcontrol.wait, so the
// stream's order holds for every byte (the preceding work has completed and
// its writes are visible when the wait returns).
#include <algorithm>

#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kCopyThreads = 256;

// dst[i] = src[i] for n 16-byte pieces; either side may be device-mapped host memory.
__global__ void __launch_bounds__(kCopyThreads) stream_copy16_kernel(const uint4 *__restrict__ src,
                                                                     uint4 *__restrict__ dst, int n) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x + blockIdx.x * blockDim.x; i < n; i += blockDim.x * gridDim.x) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_stream_copy16(const void *src, void *dst, size_t bytes, cudaStream_t s) {
  if (bytes % 16 || ((uintptr_t)src & 15u) || ((uintptr_t)dst & 15u)) return cudaErrorInvalidValue;
  const int n = (int)(bytes / 16);
  if (n == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)std::min(8, (n + kCopyThreads - 1) / kCopyThreads));
  cfg.blockDim = dim3(kCopyThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stream_copy16_kernel, static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n);
}

// The device address of `bytes` bytes of page-locked host memory at p, or nullptr when p is not such memory
// (pageable, device memory, unmapped) or the two ends of the range do not lie in one mapping.
void *mapped_host_range(const void *p, size_t bytes) {
  if (!p || bytes == 0) return nullptr;
  cudaPointerAttributes a0{}, a1{};
  const void *last = static_cast<const uint8_t *>(p) + (bytes - 1);
  if (cudaPointerGetAttributes(&a0, p) != cudaSuccess || cudaPointerGetAttributes(&a1, last) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of a failed lookup
    return nullptr;
  }
  if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer || !a1.devicePointer)
    return nullptr;
  if (static_cast<const uint8_t *>(a1.devicePointer) - static_cast<const uint8_t *>(a0.devicePointer) !=
      (ptrdiff_t)(bytes - 1))
    return nullptr;
  return a0.devicePointer;
}

}  // namespace moe
