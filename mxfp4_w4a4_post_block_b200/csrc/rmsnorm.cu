// k_row_rms: the RMSNorm factor r = 1 / sqrt(mean over the token of x^2 + eps)
// of every token, for the fused RMSNorm -> transform -> clip -> MXFP4 path.
//
// The norm ahead of each linear is z = x r gamma (the ARCQuant reading notes,
// section "融合核函数设计", fuse it with the quantisation; BATQuant applies its
// transform online before every linear, thelatestinai.com page, Figure 3
// caption).  z never leaves the quantiser: gamma is folded into the transform
// (P_i rows scaled by gamma, or x multiplied by gamma before the CUDA-core
// transform) and r multiplies the transformed values, y = r ((x gamma) P_i).
// Only r must be known before any block of a token can be scaled, and it needs
// the whole row, so this kernel computes it first; the quantiser that follows
// re-reads X, which the L2 (126 MB) still holds for activations of that size.
//
// One warp per token: 16-byte loads along the row, the sum of squares in fp64
// (bf16 and fp32 squares are exact in fp64; the sum of N of them is within
// about N 2^-53 relative, far below fp32 resolution for any row this library
// accepts), 1 / sqrt(sum / N + eps) in fp64, rounded to fp32 once.
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace batq {
namespace {

constexpr int kWarpsPerCta = 8;

template <bool kBF16>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    k_row_rms(const uint8_t* __restrict__ X, int S, int N, int ldx, float eps, float* __restrict__ r_out) {
  // X may be written by the preceding grid.  The dependent quantiser waits for
  // this whole grid to complete before it reads r, so it may start its set-up.
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S) return;
  constexpr int kPerChunk = kBF16 ? 8 : 4;  // elements per 16-byte chunk
  const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)row * (size_t)ldx * (kBF16 ? 2 : 4));
  const int chunks = N / kPerChunk;
  double acc0 = 0.0, acc1 = 0.0;
#pragma unroll 4
  for (int c = lane; c < chunks; c += 32) {
    const uint4 v = __ldg(src + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (kBF16) {
        const double lo = (double)__uint_as_float(w[i] << 16);
        const double hi = (double)__uint_as_float(w[i] & 0xFFFF0000u);
        acc0 = fma(lo, lo, acc0);
        acc1 = fma(hi, hi, acc1);
      } else {
        const double x = (double)__uint_as_float(w[i]);
        if (i & 1) acc1 = fma(x, x, acc1); else acc0 = fma(x, x, acc0);
      }
    }
  }
  double acc = acc0 + acc1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) r_out[row] = (float)(1.0 / sqrt(acc / (double)N + (double)eps));
}

}  // namespace

cudaError_t launch_row_rms(const void* X, bool bf16, int S, int N, int ldx, float eps, float* r_out,
                           cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((S + kWarpsPerCta - 1) / kWarpsPerCta));
  cfg.blockDim = dim3(kWarpsPerCta * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* x = static_cast<const uint8_t*>(X);
  return bf16 ? cudaLaunchKernelEx(&cfg, k_row_rms<true>, x, S, N, ldx, eps, r_out)
              : cudaLaunchKernelEx(&cfg, k_row_rms<false>, x, S, N, ldx, eps, r_out);
}

}  // namespace batq
