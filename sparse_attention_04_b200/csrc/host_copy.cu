// host_copy.cu -- copies between page-locked host memory and device memory
// done by a kernel instead of a copy engine.
//
// A decode step that takes its inputs from the host and hands its output back
// is a chain of short kernels.  A copy-engine transfer in that chain ends the
// programmatic launch overlap between neighbouring kernels, and each switch
// between the copy engine and the SMs costs several microseconds of
// dependency latency.  These kernels read (or write) the host buffer through
// its device mapping over PCIe instead, so the whole step stays one chain of
// kernel launches.  The bytes crossing the bus are the same.
#include <algorithm>

#include "dsa_internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyInFlight = 4;  // 16-byte chunks a thread has in flight

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// dst[i] = src[i] for i < n (16-byte chunks).  Host memory is read with
// ld.global.cv, so no cache line from an earlier step can be returned, and
// written with write-through stores.
template <bool kToHost>
__global__ void __launch_bounds__(kCopyThreads)
    host_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n) {
  grid_dependency_wait();  // the source may come from (or the target be read by) the previous kernel
  allow_dependents_launch();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + (kCopyInFlight - 1) * stride < n; i += kCopyInFlight * stride) {
    uint4 v[kCopyInFlight];
#pragma unroll
    for (int j = 0; j < kCopyInFlight; ++j) v[j] = kToHost ? src[i + j * stride] : __ldcv(src + i + j * stride);
#pragma unroll
    for (int j = 0; j < kCopyInFlight; ++j) {
      if (kToHost)
        __stwt(dst + i + j * stride, v[j]);
      else
        dst[i + j * stride] = v[j];
    }
  }
  for (; i < n; i += stride) {
    const uint4 v = kToHost ? src[i] : __ldcv(src + i);
    if (kToHost)
      __stwt(dst + i, v);
    else
      dst[i] = v;
  }
}

// The device address of [host, host + bytes) if the whole range is
// page-locked host memory mapped into the device's address space as one
// contiguous mapping, else nullptr.
void* mapped_host_range(const void* host, size_t bytes) {
  cudaPointerAttributes first{}, last{};
  if (cudaPointerGetAttributes(&first, host) != cudaSuccess ||
      cudaPointerGetAttributes(&last, static_cast<const uint8_t*>(host) + bytes - 1) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (first.type != cudaMemoryTypeHost || last.type != cudaMemoryTypeHost || !first.devicePointer ||
      static_cast<uint8_t*>(last.devicePointer) != static_cast<uint8_t*>(first.devicePointer) + bytes - 1)
    return nullptr;
  return first.devicePointer;
}

template <bool kToHost>
int launch_host_copy(const void* src, void* dst, size_t bytes, void* stream) {
  const int64_t n = (int64_t)(bytes / 16);
  const int64_t grid = std::min<int64_t>((n + kCopyThreads - 1) / kCopyThreads,
                                         (int64_t)device_info().sm_count * kCopyInFlight);
  const cudaError_t e = launch_pdl(host_copy_kernel<kToHost>, dim3((unsigned)grid), dim3(kCopyThreads), 0,
                                   reinterpret_cast<cudaStream_t>(stream), static_cast<const uint4*>(src),
                                   static_cast<uint4*>(dst), n);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

int dsa_copy_host_to_device(void* dst, const void* src_host, size_t bytes, void* stream) {
  if (bytes == 0) return DSA_OK;
  if (!dst || !src_host || bytes % 16 || !aligned16(dst) || !aligned16(src_host)) return DSA_ERR_INVALID_ARG;
  const void* src = mapped_host_range(src_host, bytes);
  if (!src) return DSA_ERR_INVALID_ARG;
  return launch_host_copy<false>(src, dst, bytes, stream);
}

int dsa_copy_device_to_host(void* dst_host, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return DSA_OK;
  if (!dst_host || !src || bytes % 16 || !aligned16(dst_host) || !aligned16(src)) return DSA_ERR_INVALID_ARG;
  void* dst = mapped_host_range(dst_host, bytes);
  if (!dst) return DSA_ERR_INVALID_ARG;
  return launch_host_copy<true>(src, dst, bytes, stream);
}

}  // extern "C"
