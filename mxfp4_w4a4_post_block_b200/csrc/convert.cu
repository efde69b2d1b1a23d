// k_e2m1_to_e4m3: the W4A8 variant's weight containers.
//
// The MXFP4 weights keep their E2M1 values and E8M0 scales; for the
// E4M3 x E4M3 block-scaled MMA each 4-bit code is widened to the one-byte
// E4M3 code of the same value (every E2M1 value is an E4M3 value: 0, 0.5, 1,
// 1.5, 2, 3, 4, 6 are E4M3 bytes 0x00, 0x30, 0x38, 0x3C, 0x40, 0x44, 0x48,
// 0x4C; the sign moves from bit 3 to bit 7).  Offline, off the timed path.
#include <cstdint>

#include "host_util.h"
#include "kernels.h"
#include "ptx.cuh"

namespace batq {
namespace {

__device__ __forceinline__ uint32_t widen_nibble(uint32_t c) {
  const uint32_t mag = __byte_perm(0x3C383000u, 0x4C484440u, c & 7u) & 0xFFu;
  return mag | ((c & 8u) << 4);
}

// Four packed bytes (eight codes, element 2j in the low nibble) -> eight E4M3 bytes.
__device__ __forceinline__ uint2 widen_word(uint32_t w) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t e = widen_nibble(w >> (8 * i)) | (widen_nibble(w >> (8 * i + 4)) << 8);
    if (i < 2)
      lo |= e << (16 * i);
    else
      hi |= e << (16 * (i - 2));
  }
  return make_uint2(lo, hi);
}

__global__ void k_e2m1_to_e4m3(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    const uint2 a = widen_word(v.x), b = widen_word(v.y), c = widen_word(v.z), d = widen_word(v.w);
    dst[2 * i] = make_uint4(a.x, a.y, b.x, b.y);
    dst[2 * i + 1] = make_uint4(c.x, c.y, d.x, d.y);
  }
}

}  // namespace

cudaError_t launch_e2m1_to_e4m3(const uint8_t* packed, uint8_t* out, size_t packed_bytes, cudaStream_t stream) {
  const size_t n16 = packed_bytes / 16;
  if (n16 == 0) return cudaSuccess;
  const int threads = 256;
  const size_t want = (n16 + threads - 1) / threads;
  const int grid = (int)(want < (size_t)(sm_count() * 8) ? want : (size_t)(sm_count() * 8));
  k_e2m1_to_e4m3<<<grid, threads, 0, stream>>>(reinterpret_cast<const uint4*>(packed), reinterpret_cast<uint4*>(out),
                                              n16);
  return cudaGetLastError();
}

}  // namespace batq
