// k_quant_act_tc: the online activation path for bf16 activations with the
// block transform on the tensor cores.
//
// Y = X P_i for every token and 32-element block is a dense 32 x 32 product
// per block column (BATQuant daily-arxiv summary, "GPK 分解": P_i = B_i (x) A;
// thelatestinai.com page, Table 1: the "XP" product).  bf16 activations are
// exact operands of a kind::f16 MMA; each entry of P_i, the product
// B_i[r][c] A[a][b] formed exactly in fp64, is split into three bf16 parts
// hi + mid + lo that carry its leading 24 bits, so Y = X hi + X mid + X lo is
// accumulated in fp32 in tensor memory (the parts' truncation error is below
// 2^-24 of sum_j |x_j| |P_ji|).  The clip, scale and encode that follow are the
// CUDA-core kernel's own code (quant_common.cuh), so every rounding decision
// is taken with the same instructions.
//
// Layout of the work: a strip is 4 block columns (128 elements of every
// token), a tile 128 tokens of a strip; tiles are ordered strip by strip (one
// launch may cover up to eight independent activations, problem after
// problem, each with its own tensor map and arguments) and
// each CTA (one per SM) takes an equal contiguous share, so it meets at most
// a few strips and builds each strip's P_i parts once in shared memory (24 KB,
// 64-byte swizzled K-major rows, as the MMA reads them).  The three parts of
// one P_i are 96 consecutive rows: per tile, block column and K step one MMA
// with N = 64 (M = 128 tokens, K = 16) writes X hi and X mid side by side in
// TMEM and one with N = 32 adds X lo onto the mid columns, so the encoders
// read two 32-column results and add them in fp32 (hi + (mid + lo)).  That
// is 16 MMAs per tile where three separate N = 32 accumulations took 24, each
// of which re-read the 4 KB activation slice from shared memory.
//   warp 0      TMA producer: one 3-D box per tile (128 tokens x 4 blocks of
//               bf16, 32 KB, 64-byte swizzle = the MMA's K-major operand
//               layout) into a 4-stage ring;
//   warp 1      TMEM allocation (512 columns: one 64-column accumulator per
//               block column, 128 columns apart) and the MMAs, issued by one
//               elected lane while the whole warp runs the loop: per tile and
//               block column four MMAs, then a commit to that column's
//               accumulator barrier;
//   warps 2-17  encoders: warp w reads TMEM lane quadrant w % 4 (its 32
//               tokens) and block column (w - 2) / 4 of the tile with two
//               tcgen05.ld of 32 columns, releases the accumulator, sums the
//               parts, then clips, scales, encodes and stores; they also build
//               the P_i parts of their block column at the start of every strip.
// Every barrier wait is bounded; on expiry a bit is set in the device error
// word and the loop ends.
#include <cuda_bf16.h>

#include <cstdint>

#include "host_util.h"
#include "kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace batq {
namespace {

constexpr int kTok = 128;                        // tokens per tile (MMA M, TMEM lanes)
constexpr int kCB = 4;                           // block columns per strip and tile
constexpr int kStages = 4;                       // activation tile ring
constexpr int kParts = 3;                        // bf16 parts of P_i
constexpr int kSlab = kTok * 64;                 // one block column of a tile: 128 rows x 64 bytes
constexpr int kXBytes = kCB * kSlab;             // 32 KB
constexpr int kPPart = 32 * 64;                  // one part of one P_i: 32 output rows x 32 bf16
constexpr int kPBytes = kCB * kParts * kPPart;   // 24 KB
constexpr int kAccStride = 128;                  // TMEM columns between block columns' accumulators
constexpr int kTmemCols = kCB * kAccStride;      // 512 (the 154 KB of shared memory keeps one CTA per SM)
constexpr int kEncWarps = 4 * kCB;               // one per (TMEM lane quadrant, block column)
constexpr int kThreads = (2 + kEncWarps) * 32;   // 576
constexpr int kPOffset = kStages * kXBytes;
constexpr int kBarOffset = kPOffset + kPBytes;
constexpr int kSmemBytes = kBarOffset + 256 + 1024;
static_assert(kEncWarps * 32 == kCB * 32 * 4, "one encoder thread per (block, output row, 8-element chunk) of P");

__device__ __forceinline__ uint32_t bf16_bits(float v) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ double bf16_value(uint32_t bits) {
  return (double)__uint_as_float(bits << 16);
}

// Encoder thread tid (0..511) writes the three parts of 8 entries of P_i for
// block column cb = tid / 128 of strip s: output element n, input elements
// 8 jc .. 8 jc + 7, i.e. P[8 jc + a][n] = B_i[jc][n / 8] A[a][n % 8] for a = 0..7
// (A_i[a][n % 8] with the naive Kronecker decomposition), as one 16-byte chunk
// per part at its 64-byte-swizzle position.  With the RMSNorm ahead of the
// transform (kNorm) row 8 jc + a of P_i is scaled by gamma of that input
// element, so the MMA computes (x gamma) P_i.
template <bool kNorm>
__device__ __forceinline__ void build_p_chunk(uint8_t* sp, int tid, int s, const QuantArgs& p) {
  const int cb = tid >> 7;
  const int n = (tid >> 2) & 31;
  const int jc = tid & 3;
  const int b = s * kCB + cb;
  const double bv = b < p.k ? (double)p.B[(size_t)b * 16 + jc * 4 + (n >> 3)] : 0.0;
  uint32_t w[kParts][4];
#pragma unroll
  for (int a = 0; a < 8; a += 2) {
    uint32_t pr[kParts][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ai = (a + h) * 8 + (n & 7);
      const float av = p.A_blocks == nullptr ? p.A[ai] : (b < p.k ? p.A_blocks[(size_t)b * 64 + ai] : 0.0f);
      double v = bv * (double)av;  // exact in fp64
      if constexpr (kNorm) v *= b < p.k ? (double)p.gamma[(size_t)b * 32 + jc * 8 + a + h] : 0.0;
      const uint32_t hi = bf16_bits((float)v);
      const double r1 = v - bf16_value(hi);
      const uint32_t mid = bf16_bits((float)r1);
      const double r2 = r1 - bf16_value(mid);
      pr[0][h] = hi;
      pr[1][h] = mid;
      pr[2][h] = bf16_bits((float)r2);
    }
#pragma unroll
    for (int q = 0; q < kParts; ++q) w[q][a >> 1] = pr[q][0] | (pr[q][1] << 16);
  }
  const int chunk = jc ^ ((n >> 1) & 3);
#pragma unroll
  for (int q = 0; q < kParts; ++q)
    *reinterpret_cast<uint4*>(sp + (cb * kParts + q) * kPPart + n * 64 + chunk * 16) =
        make_uint4(w[q][0], w[q][1], w[q][2], w[q][3]);
}

// One launch: 1 .. kG independent activations (same format), each with its
// tensor map and arguments.  The tiles of all of them form one list, problem
// by problem, each strip-major; CTAs take contiguous shares of it.
template <int kG>
struct TcLaunch {
  CUtensorMap tmx[kG];
  QuantArgs args[kG];
  int tile_begin[kG];  // first tile of each problem in the list
  int count;           // problems in use
  int num_tiles;       // tiles of all problems
};

// Problem of list tile i (tiles are in problem order).
template <int kG>
__device__ __forceinline__ int tc_problem_of(const TcLaunch<kG>& L, int i) {
  int q = 0;
#pragma unroll
  for (int r = 1; r < kG; ++r)
    if (r < L.count && i >= L.tile_begin[r]) q = r;
  return q;
}

// kNorm: RMSNorm ahead of the transform (gamma folded into P_i, the token's
// 1 / rms from p.row_scale applied to the transformed values).
template <int kFmt, bool kNorm, int kG>
__global__ void __launch_bounds__(kThreads, 1)
    k_quant_act_tc(const __grid_constant__ TcLaunch<kG> L) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;   // per block column: its MMAs of the tile completed
  uint64_t* acc_empty = acc_full + kCB;   // per block column: its four encoder warps read TMEM
  uint64_t* p_ready = acc_empty + kCB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(p_ready + 1);
  if (threadIdx.x == 0)
    for (int q = 0; q < L.count; ++q) tma_prefetch_map(&L.tmx[q]);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
#pragma unroll
    for (int b = 0; b < kCB; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(p_ready, kEncWarps);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  // This CTA's share of the list.  Within problem q, tile li = i -
  // tile_begin[q] is token tile li % tiles_r of strip li / tiles_r (tiles_r =
  // the problem's 128-token tiles); a new strip starts at li % tiles_r == 0.
  const long long ntiles = L.num_tiles;
  const int i0 = (int)((long long)blockIdx.x * ntiles / gridDim.x);
  const int total = (int)((long long)(blockIdx.x + 1) * ntiles / gridDim.x) - i0;
  struct TileAt {
    int q, s, t;  // problem, strip, token tile
  };
  auto tile_at = [&](int g) {
    TileAt a;
    a.q = tc_problem_of(L, i0 + g);
    const int tiles_r = (L.args[a.q].S + kTok - 1) / kTok;
    const int li = i0 + g - L.tile_begin[a.q];
    a.s = li / tiles_r;
    a.t = li - a.s * tiles_r;
    return a;
  };
  unsigned* const err_word = L.args[0].err;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      // X may come from the preceding grid, which may also still read the
      // outputs: touch nothing before it has finished, then let the dependent
      // grid start its set-up.
      griddep_wait();
      griddep_launch_dependents();
      for (int g = 0; g < total; ++g) {
        const int st = g % kStages;
        if (!mbar_wait(&empty[st], ((g / kStages) & 1) ^ 1)) {
          set_error(err_word, kErrReleaseTimeout);
          break;
        }
        const TileAt a = tile_at(g);
        mbar_arrive_expect_tx(&full[st], (uint32_t)kXBytes);  // the box always delivers all of it (zero fill)
        tma_load_3d(smem + st * kXBytes, &L.tmx[a.q], &full[st], 0, a.t * kTok, a.s * kCB);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA warp ------------------------------
    // The whole warp runs the loop (its state stays warp-uniform) and one
    // elected lane issues the MMAs and their commits.
    constexpr uint32_t kIdesc64 = idesc_bf16(kTok, 64);  // hi and mid side by side
    constexpr uint32_t kIdesc32 = idesc_bf16(kTok, 32);  // lo, accumulated onto mid
    const uint64_t db = sdesc_kmajor_sw64(smem_u32(smem + kPOffset));
    const bool leader = elect_one();
    uint32_t strip_count = 0;
    bool ok = true;
    for (int g = 0; g < total && ok; ++g) {
      if (g == 0 || tile_at(g).t == 0) {
        // The new strip's P_i parts are in shared memory.
        if (!mbar_wait_warp(p_ready, strip_count & 1)) {
          if (leader) set_error(err_word, kErrDataTimeout);
          break;
        }
        ++strip_count;
      }
      const int st = g % kStages;
      if (!mbar_wait_warp(&full[st], (g / kStages) & 1)) {
        if (leader) set_error(err_word, kErrDataTimeout);
        break;
      }
      tc_fence_after_sync();
      // Shared addresses stay below 2^18, so a descriptor's 14-bit address
      // field never carries: the descriptor of base + off is the base
      // descriptor + off / 16, one add per operand and MMA.
      const uint64_t da = sdesc_kmajor_sw64(smem_u32(smem + st * kXBytes));
#pragma unroll
      for (int cb = 0; cb < kCB; ++cb) {
        // The block column's accumulator must have been read by its encoders.
        if (!mbar_wait_warp(&acc_empty[cb], (g & 1) ^ 1)) {
          if (leader) set_error(err_word, kErrDrainTimeout);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // K step kk = bytes 32 kk .. 32 kk + 31 of each 64-byte row; B = the
            // 96 rows of the three parts of this block column's P_i.
            tc_mma_bf16(tmem + (uint32_t)(cb * kAccStride), da + (uint64_t)((cb * kSlab + kk * 32) >> 4),
                        db + (uint64_t)((cb * kParts * kPPart + kk * 32) >> 4), kIdesc64, kk ? 1u : 0u);
            tc_mma_bf16(tmem + (uint32_t)(cb * kAccStride + 32), da + (uint64_t)((cb * kSlab + kk * 32) >> 4),
                        db + (uint64_t)(((cb * kParts + 2) * kPPart + kk * 32) >> 4), kIdesc32, 1u);
          }
          tc_commit(&acc_full[cb]);  // the encoders may read this block column's results
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) tc_commit(&empty[st]);  // the stage may be refilled once these MMAs have read it
      __syncwarp();
    }
  } else {
    // ------------------------------ encoders ------------------------------
    const int e = warp - 2;
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31
    const int cb = e >> 2;      // block column of the strip
    griddep_wait();             // parameters and the NVFP4 scale may come from the preceding grid
    float gs = 1.0f;
    if constexpr (kFmt == kFmtNvfp4) {
      gs = nv_encode_scale(L.args[0]);
      if (L.args[0].gs_out != nullptr && blockIdx.x == 0 && e == 0 && lane == 0) *L.args[0].gs_out = gs;
    }
    uint8_t* sp = smem + kPOffset;
    float r_min = 1.0f, r_max = 1.0f;
    int b = 0;
    for (int g = 0; g < total; ++g) {
      const TileAt at = tile_at(g);
      const int s = at.s, t = at.t;
      const QuantArgs& p = L.args[at.q];
      // With several problems per launch, the tile's problem as register
      // values, fetched before the waits below (its table entry is indexed at
      // run time); a single-problem launch reads its parameters directly.
      [[maybe_unused]] const BlockOut o = kG > 1 ? block_out(p) : BlockOut{};
      if (g == 0 || t == 0) {
        // Every MMA of the previous strip has completed (this warp saw its
        // last accumulator), so the parts may be overwritten.
        build_p_chunk<kNorm>(sp, e * 32 + lane, s, p);
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);
        b = s * kCB + cb;
        r_min = r_max = 1.0f;
        if (p.ratios != nullptr && b < p.k) {
          r_min = p.ratios[2 * b];
          r_max = p.ratios[2 * b + 1];
        }
      }
      if (!mbar_wait_warp(&acc_full[cb], g & 1)) {
        if (lane == 0) set_error(p.err, kErrMmaTimeout);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      // X hi and X mid + X lo (added in TMEM) of this block column, summed in fp32.
      const uint32_t tacc = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(cb * kAccStride);
      uint32_t ra[32], rb[32];
      tmem_ld_32cols(tacc, ra);
      tmem_ld_32cols(tacc + 32, rb);
      tmem_ld_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[cb]);
      float y[32];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 sv = __fadd2_rn(make_float2(__uint_as_float(ra[j]), __uint_as_float(ra[j + 1])),
                                     make_float2(__uint_as_float(rb[j]), __uint_as_float(rb[j + 1])));
        y[j] = sv.x;
        y[j + 1] = sv.y;
      }
      const int row = t * kTok + 32 * quad + lane;
      if constexpr (kNorm) {
        const float rs = row < p.S ? p.row_scale[row] : 0.0f;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 sv = __fmul2_rn(make_float2(y[j], y[j + 1]), make_float2(rs, rs));
          y[j] = sv.x;
          y[j + 1] = sv.y;
        }
      }
      if constexpr (kG == 1) {
        if (b < p.k) {
          encode_block<kFmt>(y, r_min, r_max, gs, row, b, lane, p);
        } else {
          pad_scales<kFmt>(row, b, p);
        }
      } else {
        if (b < o.k) {
          encode_block<kFmt>(y, r_min, r_max, gs, row, b, lane, o);
        } else {
          pad_scales<kFmt>(row, b, o);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Ls / as [0 .. count-1]: one format, bf16 activations, one stream (Ls[0]'s).
template <int kFmt, bool kNorm, int kG>
cudaError_t launch_tc_impl(const QuantLaunch* Ls, const QuantArgs* as, int count) {
  if (count < 1 || count > kG) return cudaErrorInvalidValue;
  TcLaunch<kG> T = {};
  long long tiles = 0;
  for (int q = 0; q < count; ++q) {
    const QuantLaunch& L = Ls[q];
    // X viewed as {32 elements of a block, S tokens, k blocks}; one box = one tile.
    if (!make_map_3d_swizzled(&T.tmx[q], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L.X, 32, (uint64_t)L.S,
                              (uint64_t)(L.N / 32), (uint64_t)L.ldx * 2u, 64, 32, kTok, kCB,
                              CU_TENSOR_MAP_SWIZZLE_64B)) {
      return cudaErrorInvalidValue;
    }
    T.args[q] = as[q];
    T.tile_begin[q] = (int)tiles;
    tiles += (long long)((as[q].k + kCB - 1) / kCB) * ((as[q].S + kTok - 1) / kTok);
  }
  if (tiles >= (1LL << 31)) return cudaErrorInvalidValue;
  T.count = count;
  T.num_tiles = (int)tiles;
  auto kern = k_quant_act_tc<kFmt, kNorm, kG>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int grid = tiles < sm_count() ? (int)tiles : sm_count();  // one CTA per SM
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = Ls[0].stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, T);
}

}  // namespace

cudaError_t launch_quant_act_tc(const QuantLaunch& L, const QuantArgs& a) {
  if (L.gamma != nullptr) {  // RMSNorm ahead of the transform: MXFP4 output, shared A
    if (L.fmt != kFmtMxfp4 || L.A_blocks != nullptr || L.row_scale == nullptr) return cudaErrorInvalidValue;
    return launch_tc_impl<kFmtMxfp4, true, 1>(&L, &a, 1);
  }
  switch (L.fmt) {
    case kFmtMxfp4: return launch_tc_impl<kFmtMxfp4, false, 1>(&L, &a, 1);
    case kFmtMxfp8: return launch_tc_impl<kFmtMxfp8, false, 1>(&L, &a, 1);
    case kFmtNvfp4: return launch_tc_impl<kFmtNvfp4, false, 1>(&L, &a, 1);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quant_act_tc_group(const QuantLaunch* Ls, const QuantArgs* as, int count) {
  return launch_tc_impl<kFmtMxfp4, false, kMaxQuantGroup>(Ls, as, count);
}

}  // namespace batq
