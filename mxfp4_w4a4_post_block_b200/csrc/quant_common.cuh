// Pieces shared by the two quantiser kernels (CUDA-core transform in
// quant_act.cu, tensor-core transform in quant_act_tc.cu): launch arguments,
// the scale-layout address, and the clip / scale / encode / store of one
// token's 32-element block from its transformed values, so both kernels take
// every rounding decision with the same instructions.
#pragma once

#include <cfloat>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace batq {

constexpr uint8_t kPadScale = 0x7F;        // E8M0 1.0 in padding rows and columns
constexpr uint32_t kPadScaleNv = 0x3838u;  // two E4M3 1.0 scales in NVFP4 padding rows
constexpr float kNvGlobalNumerator = 2688.0f;  // 448 (largest E4M3) x 6 (largest E2M1)

struct QuantArgs {
  float A[64];
  const float* B;
  const float* ratios;
  uint8_t* codes;
  uint8_t* scales;
  float* y_debug;
  unsigned* err;
  int S, N, k, kpad;
  int rows_out;  // rows whose scales are written (S, or S rounded up to 128 in MMA layout)
  int mma_layout;
  // Tiling of the CUDA-core kernel (32 tokens x 8 blocks); the tensor-core kernel tiles itself.
  int tiles_r, tiles_c;
  unsigned long long tiles_c_magic;  // ceil(2^40 / tiles_c): t / tiles_c = (t * magic) >> 40 for t < 2^24
  // NVFP4 per-tensor scale sources and outputs (see QuantLaunch)
  const float* gs;
  const unsigned* gs_amax;
  float* gs_out;
  unsigned* amax_out;
  // Output row of token r: row_map[r] (skipped when < 0 or >= rows_cap), or r
  // itself when row_map is null (then rows_cap = S).  Linear scale layout only.
  const int* row_map;
  int rows_cap;
  // Naive Kronecker: one 8x8 A_i per block (device, k x 64 floats) instead of A.
  const float* A_blocks;
  // RMSNorm ahead of the transform (both null without it): per-element gamma
  // (N floats) and per-token 1 / rms (S floats).
  const float* gamma;
  const float* row_scale;
};

__device__ __forceinline__ int tile_row(int t, const QuantArgs& p) {
  return (int)(((unsigned long long)(unsigned)t * p.tiles_c_magic) >> 40);
}

__device__ __forceinline__ uint32_t mma_scale_offset(int row, int kb, int kpad) {
  return (uint32_t)(((row >> 7) * (kpad >> 2) + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// The GPK block transform of one token's block on CUDA cores (daily-arxiv
// summary, "GPK 分解": y = x (B_i (x) A), computed as Y = B_i^T X A with X the
// row-major 4 x 8 view of x).  T = X A produces column pairs (T[r][2j],
// T[r][2j+1]) from a duplicated x value and an A row pair, then Y = B^T T
// reuses those column pairs with a duplicated B entry: 192 packed fp32x2 FMAs
// per block, accumulated in the order a = 0..7, then r = 0..3.  a_pair(a, j)
// returns (A[a][2j], A[a][2j + 1]); Bm is B_i row-major.  y2[4 c + j] holds
// (Y[c][2j], Y[c][2j + 1]).
template <typename APair>
__device__ __forceinline__ void gpk_transform(const float (&x)[32], APair a_pair, const float (&Bm)[16],
                                              float2 (&y2)[16]) {
  float2 tm[16];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float xv = x[8 * r + a];
        acc = __ffma2_rn(make_float2(xv, xv), a_pair(a, j), acc);
      }
      tm[4 * r + j] = acc;
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float bv = Bm[4 * r + c];
        acc = __ffma2_rn(make_float2(bv, bv), tm[4 * r + j], acc);
      }
      y2[4 * c + j] = acc;
    }
  }
}

// NVFP4 per-tensor encode scale: 448 * 6 / amax from the measured amax word if
// given, else the device float, else 1.  Read only after the preceding grid
// has completed (griddepcontrol.wait).
__device__ __forceinline__ float nv_encode_scale(const QuantArgs& p) {
  float gs = 1.0f;
  if (p.gs_amax != nullptr) {
    const float a = __uint_as_float(*p.gs_amax);
    if (a > 0.0f) {
      gs = __fdiv_rn(kNvGlobalNumerator, a);
      if (!(gs <= FLT_MAX)) gs = 1.0f;
    }
  } else if (p.gs != nullptr) {
    gs = *p.gs;
  }
  return gs;
}

// The fields of QuantArgs that encode_block and pad_scales read, held as
// values, for a launch serving several problems (launch_quant_act_tc_group):
// it copies its tile's problem into these once per tile instead of indexing
// the parameter table inside the encode.  Such launches never have a row map,
// y_debug or a measuring pass, so those are compile-time null.
struct BlockOut {
  uint8_t* codes;
  uint8_t* scales;
  int S, N, k, kpad, rows_out, rows_cap, mma_layout;
  static constexpr float* y_debug = nullptr;
  static constexpr const int* row_map = nullptr;
  static constexpr unsigned* amax_out = nullptr;
};
__device__ __forceinline__ BlockOut block_out(const QuantArgs& p) {
  BlockOut o;
  o.codes = p.codes;
  o.scales = p.scales;
  o.S = p.S;
  o.N = p.N;
  o.k = p.k;
  o.kpad = p.kpad;
  o.rows_out = p.rows_out;
  o.rows_cap = p.rows_cap;
  o.mma_layout = p.mma_layout;
  return o;
}

// Clip, scale, encode and store one token's 32-element block b (y: its
// transformed values; gs: the NVFP4 encode scale, unused otherwise).  Rows
// past S only get padding scales (MMA layout).  All 32 lanes of the warp call
// it together (the measuring pass reduces across the warp).  Args: QuantArgs
// or BlockOut.
template <int kFmt, class Args>
__device__ __forceinline__ void encode_block(const float (&y)[32], float r_min, float r_max, float gs, int row, int b,
                                             int lane, const Args& p) {
  constexpr bool kFp8 = (kFmt == kFmtMxfp8);
  constexpr bool kNv = (kFmt == kFmtNvfp4);
  // Extrema (NaN-propagating) of each 16-element half, and of the block.
  float mn0 = fmin3_nan(y[0], y[1], y[2]), mx0 = fmax3_nan(y[0], y[1], y[2]);
  float mn1 = fmin3_nan(y[16], y[17], y[18]), mx1 = fmax3_nan(y[16], y[17], y[18]);
#pragma unroll
  for (int j = 3; j < 15; j += 2) {
    mn0 = fmin3_nan(mn0, y[j], y[j + 1]);
    mx0 = fmax3_nan(mx0, y[j], y[j + 1]);
    mn1 = fmin3_nan(mn1, y[16 + j], y[17 + j]);
    mx1 = fmax3_nan(mx1, y[16 + j], y[17 + j]);
  }
  mn0 = fmin_nan(mn0, y[15]);
  mx0 = fmax_nan(mx0, y[15]);
  mn1 = fmin_nan(mn1, y[31]);
  mx1 = fmax_nan(mx1, y[31]);
  const float mn = fmin_nan(mn0, mn1), mx = fmax_nan(mx0, mx1);
  const bool finite = (fabsf(mn) <= FLT_MAX) && (fabsf(mx) <= FLT_MAX);
  // Clip bounds from the whole block; clipped amax = max(|clamp(min)|, |clamp(max)|).
  const float lo = r_min * mn;
  const float hi = r_max * mx;
  auto clampf = [&](float v) { return fminf(fmaxf(v, lo), hi); };

  if (kNv && p.amax_out != nullptr) {
    // Measuring pass: fold this warp's largest clipped |y| into the tensor amax.
    const float a = finite ? fmaxf(fmaxf(fabsf(clampf(mn0)), fabsf(clampf(mx0))),
                                   fmaxf(fabsf(clampf(mn1)), fabsf(clampf(mx1))))
                           : 0.0f;
    const unsigned v = __reduce_max_sync(0xffffffffu, row < p.S ? __float_as_uint(a) : 0u);
    if (lane == 0 && v != 0u) atomicMax(p.amax_out, v);
  } else {
    uint32_t sbits;  // scale byte (MX) or two scale bytes (NVFP4, half 0 in the low byte)
    float2 mult;     // multiplier of the elements of each half
    if constexpr (kNv) {
      // Group scale E4M3(fp32(amax * gs) / 6) per half; multiplier fp32(gs / scale).
      const float a0 = fmaxf(fabsf(clampf(mn0)), fabsf(clampf(mx0)));
      const float a1 = fmaxf(fabsf(clampf(mn1)), fabsf(clampf(mx1)));
      sbits = e4m3x2_bits(__fdiv_rn(__fmul_rn(a0, gs), 6.0f), __fdiv_rn(__fmul_rn(a1, gs), 6.0f));
      const float2 sv = e4m3x2_values(sbits);
      mult.x = sv.x == 0.0f ? 0.0f : __fdiv_rn(gs, sv.x);
      mult.y = sv.y == 0.0f ? 0.0f : __fdiv_rn(gs, sv.y);
    } else {
      // Shared scale: floor(log2 amax) = biased exponent - 127, so the scale
      // byte e + 127 = biased exponent - emax (emax = 2 for E2M1, 8 for E4M3;
      // clamped at 0, which also covers amax == 0 and subnormal amax).  2^-e
      // is built from exponent bits.
      const float amax = fmaxf(fabsf(clampf(mn)), fabsf(clampf(mx)));
      constexpr uint32_t kEmax = kFp8 ? 8u : 2u;
      const uint32_t ebits = __float_as_uint(amax) >> 23;
      sbits = ebits > kEmax ? ebits - kEmax : 0u;
      const float inv_scale = __uint_as_float((254u - sbits) << 23);
      mult = make_float2(inv_scale, inv_scale);
    }

    // Clip, then divide by the scale (an exact power-of-two multiply for MX,
    // the fp32 multiplier for NVFP4; two elements per packed multiply), then
    // round to E2M1 or E4M3.
    constexpr int kWords = kFp8 ? 8 : 4;  // 32 codes of 4 or 8 bits
    uint32_t words[kWords];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float m = w < 2 ? mult.x : mult.y;
      const float2 inv2 = make_float2(m, m);
      float2 q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 c2 = make_float2(clampf(y[8 * w + 2 * j]), clampf(y[8 * w + 2 * j + 1]));
        q[j] = __fmul2_rn(c2, inv2);
      }
      if constexpr (kFp8) {
        words[2 * w] = e4m3x4(q[0].x, q[0].y, q[1].x, q[1].y);
        words[2 * w + 1] = e4m3x4(q[2].x, q[2].y, q[3].x, q[3].y);
      } else {
        words[w] = e2m1x8(q[0].x, q[0].y, q[1].x, q[1].y, q[2].x, q[2].y, q[3].x, q[3].y);
      }
    }
    if (!finite) {
      sbits = kNv ? 0x7F7Fu : 0xFFu;
#pragma unroll
      for (int w = 0; w < kWords; ++w) words[w] = 0u;
    }

    const int orow = (row < p.S && p.row_map != nullptr) ? p.row_map[row] : row;
    if (row < p.S && orow >= 0 && orow < p.rows_cap) {
      constexpr int kBlockCodeBytes = kWords * 4;
      uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)orow * (size_t)(kFp8 ? p.N : p.N >> 1) +
                                            (size_t)b * kBlockCodeBytes);
      dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
      if constexpr (kFp8) dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
      if constexpr (kNv) {
        // scale columns 2b and 2b + 1 are adjacent in both layouts
        uint8_t* sp = p.mma_layout ? p.scales + mma_scale_offset(orow, 2 * b, p.kpad)
                                   : p.scales + (size_t)orow * (size_t)(2 * p.k) + 2 * b;
        *reinterpret_cast<uint16_t*>(sp) = (uint16_t)sbits;
      } else if (p.mma_layout) {
        p.scales[mma_scale_offset(orow, b, p.kpad)] = (uint8_t)sbits;
      } else {
        p.scales[(size_t)orow * p.k + b] = (uint8_t)sbits;
      }
      if (p.y_debug != nullptr) {
        float4* yd = reinterpret_cast<float4*>(p.y_debug + (size_t)row * p.N + (size_t)b * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) yd[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
      }
    } else if (row >= p.S && p.mma_layout && row < p.rows_out) {
      if constexpr (kNv)
        *reinterpret_cast<uint16_t*>(p.scales + mma_scale_offset(row, 2 * b, p.kpad)) = (uint16_t)kPadScaleNv;
      else
        p.scales[mma_scale_offset(row, b, p.kpad)] = kPadScale;
    }
  }
}

// Padding scales for (row, block b) when the block holds no data: rows past S
// (all formats) and block columns past k (MX only; the NVFP4 column count 2k is
// already a multiple of 4).
template <int kFmt, class Args>
__device__ __forceinline__ void pad_scales(int row, int b, const Args& p) {
  if (!p.mma_layout || row >= p.rows_out) return;
  if constexpr (kFmt == kFmtNvfp4) {
    if (b < p.k)
      *reinterpret_cast<uint16_t*>(p.scales + mma_scale_offset(row, 2 * b, p.kpad)) = (uint16_t)kPadScaleNv;
  } else if (b < p.kpad) {
    p.scales[mma_scale_offset(row, b, p.kpad)] = kPadScale;
  }
}

// The tensor-core quantiser for bf16 activations (quant_act_tc.cu).
cudaError_t launch_quant_act_tc(const QuantLaunch& L, const QuantArgs& a);
// The same kernel over 1 .. kMaxQuantGroup activations in one launch (MXFP4,
// bf16, plain GPK: no RMSNorm, naive Kronecker or row map), Ls[0]'s stream.
cudaError_t launch_quant_act_tc_group(const QuantLaunch* Ls, const QuantArgs* as, int count);

}  // namespace batq
