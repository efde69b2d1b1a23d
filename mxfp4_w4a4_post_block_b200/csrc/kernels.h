// Launchers of the device kernels (internal to libbatq).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace batq {

struct QuantLaunch {
  const void* X;
  bool bf16;
  int S, N, ldx;
  float A[64];          // 8x8 row-major, passed by value into the launch
  const float* B;       // device, k x 16
  const float* ratios;  // device, 2k, or nullptr (no clip)
  uint8_t* codes;       // device, S x N/2
  uint8_t* scales;      // device
  bool mma_layout;
  float* y_debug;       // device S x N or nullptr
  unsigned* err;        // device error word
  cudaStream_t stream;
};

// Returns cudaErrorInvalidValue when the tensor map cannot be encoded.
// All kernels are launched as programmatic dependents of the preceding grid in
// the stream: each waits for that grid before touching memory it may write
// (the GEMM's weights excepted when GemmLaunch::weights_ready is set), and
// lets its own dependents start early.
cudaError_t launch_quant_act(const QuantLaunch& L);

struct GemmLaunch {
  const uint8_t* a_codes;
  const uint8_t* a_scales;  // MMA layout, S rows
  const uint8_t* w_codes;
  const uint8_t* w_scales;  // MMA layout, M rows
  int S, M, N;
  bool out_bf16;
  void* out;
  int ldo;
  unsigned* err;
  cudaStream_t stream;
  // The grid launched just before this one in the stream does not write the
  // weights, so they may be read before waiting for it (set by the linear
  // layer, whose preceding grid is its own quantiser).
  bool weights_ready;
};

cudaError_t launch_gemm_mxfp4(const GemmLaunch& L);

// Prefill-shape GEMM on CTA pairs (tcgen05 cta_group::2); used for S > 128.
cudaError_t launch_gemm_pair(const GemmLaunch& L);

// One-thread kernel whose barrier wait always expires after limit_ns.
cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned* err, cudaStream_t stream);

}  // namespace batq
