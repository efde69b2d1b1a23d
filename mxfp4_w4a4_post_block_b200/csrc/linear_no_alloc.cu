// batq_linear_no_alloc: the W4A4 linear for callers that cannot allocate device memory.
//
// batq_linear needs a scratch workspace for the quantised activations (codes
// and tcgen05-layout scales) between its two kernels, and expects the caller
// to allocate it.  Some callers cannot: code running inside a host process
// whose device memory is entirely reserved up front by another allocator,
// plugins that are handed tensors but no allocator, and latency-critical paths
// where cudaMalloc / cudaFree (which may synchronise the device) are not
// allowed.  This entry point takes its scratch from a fixed array that lives
// in the library's own device memory instead.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "../../include/batq.h"

namespace {

// The scratch array.  Every device that loads this library's module holds it
// until the process exits.  With CUDA's default lazy module loading the array
// is created on a device when the module is first used there (at the latest by
// the address lookup below), so it needs 16 MiB of free device memory at that
// moment.  In host code its name is only a host-side handle, never a device
// address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_linear_scratch[BATQ_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device, looked up once
// per device with that device current.  Host threads may make their first
// call on a device at the same time: the cache slots are atomics, and two
// threads that both look the address up store the same value.
batq_status scratch_address(void** out) {
  static std::atomic<void*> cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BATQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BATQ_ERR_INVALID_ARG;
  void* p = cached[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr) return BATQ_ERR_CUDA;
    cached[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return BATQ_OK;
}

}  // namespace

extern "C" BATQ_API batq_status batq_linear_no_alloc(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                                     const float* A_host, const float* B_dev,
                                                     const float* ratios_dev, const uint8_t* w_codes,
                                                     const uint8_t* w_scales, int M, batq_dtype out_dtype,
                                                     void* out, int ldo, void* stream) {
  size_t need = 0;
  batq_status st = batq_linear_workspace_size(S, N, &need);
  if (st != BATQ_OK) return st;
  if (need > (size_t)BATQ_NO_ALLOC_SCRATCH_BYTES) return BATQ_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != BATQ_OK) return st;
  // The quantiser writes every scratch byte the GEMM reads (codes, scales and
  // their padding), so nothing left over from an earlier call is ever used.
  return batq_linear(X, x_dtype, S, N, ldx, A_host, B_dev, ratios_dev, w_codes, w_scales, M, scratch,
                     (size_t)BATQ_NO_ALLOC_SCRATCH_BYTES, out_dtype, out, ldo, stream);
}
