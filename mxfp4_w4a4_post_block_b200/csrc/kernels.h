// Launchers of the device kernels (internal to libbatq).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace batq {

// Element / scale format of a quantised operand.
enum Fmt : int {
  kFmtMxfp4 = 0,  // packed E2M1, one E8M0 scale per 32 elements
  kFmtMxfp8 = 1,  // E4M3 bytes, one E8M0 scale per 32 elements (the W4A8 variant's activations)
  kFmtNvfp4 = 2,  // packed E2M1, one E4M3 scale per 16 elements, per-tensor fp32 encode scale
};

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
  int fmt;              // Fmt
  // NVFP4 only.  The per-tensor encode scale gs comes from gs_amax (device word
  // holding the fp32 bits of a tensor amax: gs = 448 * 6 / amax) if set, else
  // from gs (device float), else is 1.  gs_out (device, nullable) receives the
  // gs used.  With amax_out set the launch only measures: the largest clipped
  // |y| of every finite block is folded into *amax_out (fp32 bits, atomic max)
  // and nothing else is written.
  const float* gs = nullptr;
  const unsigned* gs_amax = nullptr;
  float* gs_out = nullptr;
  unsigned* amax_out = nullptr;
  // Output row of token r: row_map[r] (device int32[S]; rows < 0 or >= num_slots
  // are skipped), e.g. the slot of a paged KV cache.  Linear scale layout only.
  const int* row_map = nullptr;
  int num_slots = 0;
  // Naive Kronecker decomposition: one 8x8 A_i per block (device, k x 64
  // floats, 16-byte aligned) replaces A; MXFP4 output only.
  const float* A_blocks = nullptr;
  // RMSNorm ahead of the transform (both set or both null): gamma (device, N
  // floats, 16-byte aligned) scales element j of every token before the
  // transform, row_scale (device, S floats: 1 / rms of each token, from
  // launch_row_rms) scales the transformed values of the token.
  const float* gamma = nullptr;
  const float* row_scale = nullptr;
};

// Returns cudaErrorInvalidValue when the tensor map cannot be encoded.
// All kernels are launched as programmatic dependents of the preceding grid in
// the stream: each waits for that grid before touching memory it may write
// (the GEMM's weights excepted when GemmLaunch::weights_ready is set), and
// lets its own dependents start early.
cudaError_t launch_quant_act(const QuantLaunch& L);

// Up to kMaxQuantGroup independent activations (MXFP4, MMA or linear scale
// layout, no RMSNorm, naive Kronecker or row map) on Ls[0]'s stream with
// Ls[0]'s error word: each takes the kernel launch_quant_act would give it,
// and those of one kernel and input type share a launch (at most three:
// tensor-core, CUDA-core bf16, CUDA-core fp32).  Refuses
// (cudaErrorInvalidValue) what it does not cover.
constexpr int kMaxQuantGroup = 8;
cudaError_t launch_quant_act_group(const QuantLaunch* Ls, int count);

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
  // kFmtMxfp8: both operands are E4M3 bytes (the W4A8 variant: MXFP8
  // activations, MXFP4 weights in E4M3 containers); kFmtNvfp4: packed E2M1
  // with E4M3 scales per 16 K, and the epilogue multiplies by
  // fp32(1 / fp32(gs_a * gs_w)) read from the device (each nullable: 1).
  int fmt;
  const float* gs_a;
  const float* gs_w;
};

cudaError_t launch_gemm_mxfp4(const GemmLaunch& L);

// Prefill-shape GEMM on CTA pairs (tcgen05 cta_group::2); used for S > 128.
cudaError_t launch_gemm_pair(const GemmLaunch& L);

// Up to kMaxGemmGroup independent prefill GEMMs (MXFP4, S > 128 each, one
// output type, one stream: Ls[0]'s) in one launch of the pair kernel over all
// of their tiles; Ls[0] also gives the error word and weights_ready.
constexpr int kMaxGemmGroup = 8;
cudaError_t launch_gemm_pair_group(const GemmLaunch* Ls, int count);

// Up to kMaxGemmGroup independent small-S GEMMs (MXFP4, all S in the same one
// of the tile configurations S <= 16 / 32 / 64 / 128, one output type, Ls[0]'s
// stream) in one launch of the single-CTA kernel, one CTA per output tile.
cudaError_t launch_gemm_mxfp4_small_group(const GemmLaunch* Ls, int count);

// Widen packed E2M1 codes (element 2j in the low nibble) to one E4M3 byte per
// element holding the same value; packed_bytes must be a multiple of 16 and
// both pointers 16-byte aligned.
cudaError_t launch_e2m1_to_e4m3(const uint8_t* packed, uint8_t* out, size_t packed_bytes, cudaStream_t stream);

// r_out[s] = fp32(1 / sqrt(sum_j x_sj^2 / N + eps)) for every token s (sum in
// fp64); X as for the quantisers (16-byte aligned rows).
cudaError_t launch_row_rms(const void* X, bool bf16, int S, int N, int ldx, float eps, float* r_out,
                           cudaStream_t stream);

// One-thread kernel whose barrier wait always expires after limit_ns.
cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned* err, cudaStream_t stream);

}  // namespace batq
