// k_quant_act: BATQuant online activation path on sm_100a.
//
// For every token and 32-element block: Y = B_i^T X A (GPK block-wise affine
// transform), per-block clip to [r_min * min Y, r_max * max Y], E8M0 shared
// scale and E2M1 codes (BATQuant daily-arxiv summary, sections "块仿射变换",
// "GPK 分解", "块级可学习裁剪"; thelatestinai.com page, Figure 2 caption for
// the divide-then-round order; OCP MX v1.0 for the scale rule).
//
// Memory-bound design:
//   * one CTA per SM, each owning a contiguous, equal share of the tiles (so
//     no SM is left with more work than another); one producer warp streams
//     tiles of 32 tokens x 8 blocks into a shared-memory ring with one 3-D TMA
//     box per tile ({32 elements, 32 tokens, 8 blocks}: each block column lands
//     as a 32-row slab, swizzled so the per-lane row reads below are
//     bank-conflict free);
//   * the producer also stages the tile's eight B_i and clip ratios with
//     1-D bulk copies, so consumers read them from shared memory (broadcast);
//   * consumer groups of eight warps take the CTA's tiles in turn (three
//     groups for bf16 input); in a group, warp w owns block column c0 + w of
//     the tile and lane l owns token r0 + l, so B_i and the clip ratios are
//     warp-uniform and A is read from the kernel's parameter (constant) bank;
//   * the transform runs on packed fp32x2 FMAs: T = X A produces column
//     pairs (T[r][2j], T[r][2j+1]) from a duplicated x value and an A row
//     pair, then Y = B^T T reuses those column pairs with a duplicated B
//     entry, so 384 scalar FMAs per block become 192 packed ones;
//   * the block extrema are in-thread (the whole block lives in one thread),
//     the clipped amax is max(|clamp(min)|, |clamp(max)|) (clamp is
//     monotone), and the scale comes from the exponent bits of amax;
//   * one launch may cover up to eight independent activations (a table of
//     tensor maps and arguments; their tiles form one list): A then comes from
//     a 2 KB shared-memory copy of every problem's A instead of the parameter
//     bank, with the same values in the same FMA order.
//
// Output formats: MXFP4 (E2M1 + E8M0 per 32), MXFP8 (E4M3 + E8M0 per 32, the
// W4A8 variant) and NVFP4 (E2M1 + E4M3 per 16 elements with a per-tensor fp32
// encode scale gs; ARCQuant page, "背景" section, for the 16-element E4M3
// grouping).  For NVFP4 the transform and the clip still work on the 32-block;
// each half then gets scale E4M3(fp32(amax_half * gs) / 6) and the elements
// are multiplied by fp32(gs / scale) before the E2M1 rounding, every step an
// IEEE fp32 operation.
#include <cfloat>
#include <cstdint>

#include "host_util.h"
#include "kernels.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace batq {
namespace {

constexpr int kRows = 32;         // tokens per tile (one per lane)
constexpr int kCols = 8;          // 32-blocks per tile (one per warp of a consumer group)

// kNaive: one A_i per block column, staged with the tile (naive Kronecker);
// kNorm: the RMSNorm gamma of the tile's block columns staged too.
template <bool kBF16, bool kNaive = false, bool kNorm = false>
struct Tile {
  static constexpr int kGroups = kBF16 ? 3 : 1;          // consumer groups per CTA
  static constexpr int kStages = kGroups * (kBF16 ? 3 : 4);  // ring depth (a multiple of kGroups)
  static constexpr int kConsumerWarps = kGroups * kCols;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  static constexpr int kBlockBytes = kBF16 ? 64 : 128;      // one 32-element block row
  static constexpr int kBoxBytes = kRows * kBlockBytes;     // one TMA box (32 tokens x 1 block)
  static constexpr int kXBytes = kCols * kBoxBytes;         // activations of one tile
  static constexpr int kBOffset = kXBytes;                  // kCols x 16 fp32 B_i
  static constexpr int kROffset = kXBytes + kCols * 64;     // kCols x 2 fp32 clip ratios
  static constexpr int kAOffset = kROffset + kCols * 8;     // kCols x 64 fp32 A_i (naive Kronecker)
  static constexpr int kGOffset = kAOffset + (kNaive ? kCols * 256 : 0);  // kCols x 32 fp32 RMSNorm gamma
  static constexpr int kStageBytes = (kGOffset + (kNorm ? kCols * 128 : 0) + 1023) / 1024 * 1024;
  static constexpr int kSmemBytes = kStages * kStageBytes + 2 * kStages * 8 + 16 + 1024;
};

// One token's 32-element block from the swizzled tile (box = shared address of its slab).  bf16 boxes use the
// 64-byte swizzle (16-byte chunk c of row t stored at chunk c ^ ((t >> 1) & 3)),
// fp32 boxes the 128-byte swizzle (chunk c ^ (t & 7)).
template <bool kBF16>
__device__ __forceinline__ void load_block(uint32_t box, int lane, float x[32]) {
  if constexpr (kBF16) {
    const uint32_t row = box + lane * 64;
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = lds128(row + ((c ^ sw) << 4));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[c * 8 + 2 * j] = __uint_as_float(w[j] << 16);
        x[c * 8 + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  } else {
    const uint32_t row = box + lane * 128;
    const int sw = lane & 7;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = lds128(row + ((c ^ sw) << 4));
      x[c * 4 + 0] = __uint_as_float(v.x);
      x[c * 4 + 1] = __uint_as_float(v.y);
      x[c * 4 + 2] = __uint_as_float(v.z);
      x[c * 4 + 3] = __uint_as_float(v.w);
    }
  }
}

// One launch: 1 .. kG independent activations (one format and input type),
// each with its tensor map and arguments; their tiles (32 tokens x 8 blocks,
// row-major within each) form one list, problem after problem.
template <int kG>
struct CcLaunch {
  CUtensorMap tmx[kG];
  QuantArgs args[kG];
  int tile_begin[kG];  // first tile of each problem in the list
  int count;           // problems in use
  int num_tiles;       // tiles of all problems
};

// kFmt: output format (Fmt); kNaive: per-block A_i from p.A_blocks; kNorm:
// RMSNorm ahead of the transform (p.gamma and p.row_scale); kG: problems per
// launch (with more than one, each problem's A is staged in shared memory at
// the start and the transform reads it from there, as for kNaive).
template <bool kBF16, int kFmt, bool kNaive, bool kNorm, int kG>
__global__ void __launch_bounds__(Tile<kBF16, kNaive, kNorm>::kThreads, 1)
    k_quant_act(const __grid_constant__ CcLaunch<kG> L) {
  using T = Tile<kBF16, kNaive, kNorm>;
  constexpr bool kNv = (kFmt == kFmtNvfp4);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::kStages * T::kStageBytes);
  uint64_t* empty = full + T::kStages;
  float* gs_smem = reinterpret_cast<float*>(empty + T::kStages);  // NVFP4 per-tensor encode scale
  // kG > 1: every problem's A (64 floats each) right after the scale word
  // (16-byte aligned: the stages are 1 KB multiples, the barriers 144 or 192 bytes).
  float* a_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(gs_smem) + 16);
  // Fetch the TMA descriptors while the barriers and TMEM are set up.
  if (threadIdx.x == 0)
    for (int q = 0; q < L.count; ++q) tma_prefetch_map(&L.tmx[q]);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const QuantArgs& p0 = L.args[0];  // launch-wide fields: error word, NVFP4 scale sources

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < T::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCols);  // the eight warps of the group that consumed it
    }
    fence_barrier_init();
  }
  if constexpr (kG > 1)
    for (int i = threadIdx.x; i < L.count * 64; i += blockDim.x) a_tab[i] = L.args[i >> 6].A[i & 63];
  __syncthreads();

  // This CTA's contiguous share of the tiles (one CTA per SM, shares differ by
  // at most one tile).  Local tile i sits in stage i % kStages; consumer group
  // i % kGroups processes it (kStages is a multiple of kGroups, so each stage
  // always serves the same group).
  const long long ntiles = L.num_tiles;
  const int t_begin = (int)((long long)blockIdx.x * ntiles / gridDim.x);
  const int nloc = (int)((long long)(blockIdx.x + 1) * ntiles / gridDim.x) - t_begin;
  // Problem of list tile t, and t's tile row and first block column within it.
  struct TileAt {
    int q, r0, c0;
  };
  auto tile_at = [&](int t) {
    TileAt a;
    a.q = 0;
#pragma unroll
    for (int r = 1; r < kG; ++r)
      if (r < L.count && t >= L.tile_begin[r]) a.q = r;
    const QuantArgs& pq = L.args[a.q];
    const int lt = t - L.tile_begin[a.q];
    const int tr = tile_row(lt, pq);
    a.r0 = tr * kRows;
    a.c0 = (lt - tr * pq.tiles_c) * kCols;
    return a;
  };

  if (warp == T::kConsumerWarps) {
    // ---------------- producer: one thread issues the TMA boxes ----------------
    if (lane == 0) {
      // Launched as a programmatic dependent: X (and the outputs, which the
      // preceding grid may still read) are touched only after that grid has
      // finished.  Consumers access memory only after this thread's loads.
      griddep_wait();
      // Every grid before this one is complete from here on, so the dependent
      // GEMM may start (and fetch weights) while the codes are produced.
      griddep_launch_dependents();
      if constexpr (kNv) {
        // Per-tensor encode scale, published to the consumers through the
        // release of this thread's first arrivals on the stage barriers.
        const float gs = nv_encode_scale(p0);
        *gs_smem = gs;
        if (p0.gs_out != nullptr && blockIdx.x == 0) *p0.gs_out = gs;
      }
      for (int i = 0; i < nloc; ++i) {
        const int s = i % T::kStages;
        if (!mbar_wait(&empty[s], ((i / T::kStages) & 1) ^ 1)) {
          set_error(p0.err, kErrReleaseTimeout);
          break;
        }
        const TileAt at = tile_at(t_begin + i);
        const QuantArgs& p = L.args[at.q];
        const int r0 = at.r0, c0 = at.c0;
        if (r0 < p.S) {
          const int nb = min(kCols, p.k - c0);  // even: k is even and c0 a multiple of 8
          uint8_t* dst = smem + s * T::kStageBytes;
          const uint32_t pbytes = (uint32_t)nb * 64u + (p.ratios != nullptr ? (uint32_t)nb * 8u : 0u) +
                                  (kNaive ? (uint32_t)nb * 256u : 0u) + (kNorm ? (uint32_t)nb * 128u : 0u);
          // the box always delivers all 8 block columns (zero-filled past k)
          mbar_arrive_expect_tx(&full[s], (uint32_t)T::kXBytes + pbytes);
          tma_load_3d(dst, &L.tmx[at.q], &full[s], 0, r0, c0);
          bulk_load(dst + T::kBOffset, p.B + (size_t)c0 * 16, (uint32_t)nb * 64u, &full[s]);
          if (p.ratios != nullptr) bulk_load(dst + T::kROffset, p.ratios + (size_t)c0 * 2, (uint32_t)nb * 8u, &full[s]);
          if constexpr (kNaive) bulk_load(dst + T::kAOffset, p.A_blocks + (size_t)c0 * 64, (uint32_t)nb * 256u, &full[s]);
          if constexpr (kNorm) bulk_load(dst + T::kGOffset, p.gamma + (size_t)c0 * 32, (uint32_t)nb * 128u, &full[s]);
        } else {
          mbar_arrive(&full[s]);  // padding rows only: nothing to load
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  // The RMSNorm factors come from the preceding grid (launch_row_rms); the
  // consumers read them directly, so they too wait for that grid.
  if constexpr (kNorm) griddep_wait();
  const int grp = warp / kCols;
  const int wc = warp % kCols;  // block column of the tile owned by this warp
  for (int i = grp; i < nloc; i += T::kGroups) {
    const int s = i % T::kStages;
    const TileAt at = tile_at(t_begin + i);
    const QuantArgs& p = L.args[at.q];
    const int r0 = at.r0, c0 = at.c0;
    const int b = c0 + wc;
    const int row = r0 + lane;
    if (!mbar_wait_warp(&full[s], (i / T::kStages) & 1)) {
      if (lane == 0) set_error(p.err, kErrDataTimeout);
      break;
    }
    if (r0 < p.S && b < p.k) {
      const uint32_t st = smem_u32(smem) + s * T::kStageBytes;
      float x[32];
      load_block<kBF16>(st + wc * T::kBoxBytes, lane, x);
      if constexpr (kNorm) {
        // RMSNorm: x gamma (the block's 32 gamma values are the same for the whole warp)
        const uint32_t gp = st + T::kGOffset + wc * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 gv = lds128(gp + c * 16);
          const float2 g01 = __fmul2_rn(make_float2(x[4 * c], x[4 * c + 1]),
                                        make_float2(__uint_as_float(gv.x), __uint_as_float(gv.y)));
          const float2 g23 = __fmul2_rn(make_float2(x[4 * c + 2], x[4 * c + 3]),
                                        make_float2(__uint_as_float(gv.z), __uint_as_float(gv.w)));
          x[4 * c] = g01.x;
          x[4 * c + 1] = g01.y;
          x[4 * c + 2] = g23.x;
          x[4 * c + 3] = g23.y;
        }
      }

      // B_i (row-major 4x4) and the clip ratios: the same for the whole warp.
      const uint32_t bp = st + T::kBOffset + wc * 64;
      const uint4 b0 = lds128(bp), b1 = lds128(bp + 16), b2 = lds128(bp + 32), b3 = lds128(bp + 48);
      const float Bm[16] = {__uint_as_float(b0.x), __uint_as_float(b0.y), __uint_as_float(b0.z), __uint_as_float(b0.w),
                            __uint_as_float(b1.x), __uint_as_float(b1.y), __uint_as_float(b1.z), __uint_as_float(b1.w),
                            __uint_as_float(b2.x), __uint_as_float(b2.y), __uint_as_float(b2.z), __uint_as_float(b2.w),
                            __uint_as_float(b3.x), __uint_as_float(b3.y), __uint_as_float(b3.z), __uint_as_float(b3.w)};
      float r_min = 1.0f, r_max = 1.0f;
      if (p.ratios != nullptr) {
        const float2 r = lds64f(st + T::kROffset + wc * 8);
        r_min = r.x;
        r_max = r.y;
      }

      // Y = B^T X A (X is the row-major 4x8 view of the block), from A (the
      // parameter bank) or the staged A_i (naive Kronecker).
      float2 y2[16];
      if constexpr (kNaive) {
        const uint32_t ap = st + T::kAOffset + wc * 256;
        gpk_transform(x, [&](int a, int j) { return lds64f(ap + (8 * a + 2 * j) * 4); }, Bm, y2);
      } else if constexpr (kG > 1) {
        const uint32_t ap = smem_u32(a_tab) + at.q * 256;
        gpk_transform(x, [&](int a, int j) { return lds64f(ap + (8 * a + 2 * j) * 4); }, Bm, y2);
      } else {
        gpk_transform(x, [&](int a, int j) { return make_float2(p.A[8 * a + 2 * j], p.A[8 * a + 2 * j + 1]); }, Bm,
                      y2);
      }
      if constexpr (kNorm) {
        // RMSNorm: the token's 1 / rms times the transformed values
        const float rs = p.row_scale[row];
#pragma unroll
        for (int i = 0; i < 16; ++i) y2[i] = __fmul2_rn(y2[i], make_float2(rs, rs));
      }
      float y[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        y[2 * i] = y2[i].x;
        y[2 * i + 1] = y2[i].y;
      }

      encode_block<kFmt>(y, r_min, r_max, kNv ? *gs_smem : 1.0f, row, b, lane, p);
    } else {
      pad_scales<kFmt>(row, b, p);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

QuantArgs make_args(const QuantLaunch& L) {
  QuantArgs a;
  for (int i = 0; i < 64; ++i) a.A[i] = L.A[i];
  a.B = L.B;
  a.ratios = L.ratios;
  a.codes = L.codes;
  a.scales = L.scales;
  a.y_debug = L.y_debug;
  a.err = L.err;
  a.S = L.S;
  a.N = L.N;
  a.k = L.N / 32;
  // scale columns of the MMA layout: k rounded up to 4 (MX), 2k (NVFP4, already a multiple of 4)
  a.kpad = L.fmt == kFmtNvfp4 ? 2 * a.k : (a.k + 3) / 4 * 4;
  a.mma_layout = (L.mma_layout && L.amax_out == nullptr) ? 1 : 0;
  a.gs = L.gs;
  a.gs_amax = L.gs_amax;
  a.gs_out = L.gs_out;
  a.amax_out = L.fmt == kFmtNvfp4 ? L.amax_out : nullptr;
  a.row_map = L.row_map;
  a.rows_cap = L.row_map != nullptr ? L.num_slots : L.S;
  a.A_blocks = L.A_blocks;
  a.gamma = L.gamma;
  a.row_scale = L.row_scale;
  a.rows_out = a.mma_layout ? (L.S + 127) / 128 * 128 : L.S;
  a.tiles_r = (a.rows_out + kRows - 1) / kRows;
  a.tiles_c = (a.k + kCols - 1) / kCols;
  a.tiles_c_magic = ((1ull << 40) + (unsigned long long)a.tiles_c - 1) / (unsigned long long)a.tiles_c;
  return a;
}

// Ls / as [0 .. count-1]: one format and input type on Ls[0]'s stream.
template <bool kBF16, int kFmt, bool kNaive = false, bool kNorm = false, int kG = 1>
cudaError_t launch_impl(const QuantLaunch* Ls, const QuantArgs* as, int count) {
  using T = Tile<kBF16, kNaive, kNorm>;
  if (count < 1 || count > kG) return cudaErrorInvalidValue;
  CcLaunch<kG> C = {};
  long long tiles = 0;
  for (int q = 0; q < count; ++q) {
    const QuantLaunch& L = Ls[q];
    // X viewed as {32 elements of a block, S tokens, k blocks}; one box = one tile.
    const uint64_t esz = kBF16 ? 2u : 4u;
    if (!make_map_3d_swizzled(&C.tmx[q], kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                              L.X, 32, (uint64_t)L.S, (uint64_t)(L.N / 32), (uint64_t)L.ldx * esz, 32 * esz, 32,
                              kRows, kCols, kBF16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B)) {
      return cudaErrorInvalidValue;
    }
    C.args[q] = as[q];
    C.tile_begin[q] = (int)tiles;
    tiles += (long long)as[q].tiles_r * as[q].tiles_c;
  }
  if (tiles >= (1LL << 31)) return cudaErrorInvalidValue;
  C.count = count;
  C.num_tiles = (int)tiles;
  auto kern = k_quant_act<kBF16, kFmt, kNaive, kNorm, kG>;
  const int smem_bytes = T::kSmemBytes + (kG > 1 ? kG * 256 : 0);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int grid = tiles < sm_count() ? (int)tiles : sm_count();  // one CTA per SM
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(T::kThreads);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = Ls[0].stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, C);
}

}  // namespace

cudaError_t launch_quant_act(const QuantLaunch& L) {
  const QuantArgs a = make_args(L);
  // bf16 activations are exact tensor-core operands.  When every SM gets at
  // least six of its 128-token x 128-element tiles, the tensor-core kernel
  // (quant_act_tc.cu) is faster: its per-tile cost is lower but its pipeline
  // takes longer to fill.  Smaller bf16 problems and fp32 activations take the
  // CUDA-core kernel above.
  const long long tc_tiles = (long long)((a.k + 3) / 4) * ((L.S + 127) / 128);
  if (L.bf16 && tc_tiles >= 6LL * sm_count()) return launch_quant_act_tc(L, a);
  if (L.gamma != nullptr) {  // RMSNorm ahead of the transform: MXFP4 output, shared A
    if (L.fmt != kFmtMxfp4 || L.A_blocks != nullptr || L.row_scale == nullptr) return cudaErrorInvalidValue;
    return L.bf16 ? launch_impl<true, kFmtMxfp4, false, true>(&L, &a, 1) : launch_impl<false, kFmtMxfp4, false, true>(&L, &a, 1);
  }
  if (L.A_blocks != nullptr) {  // naive Kronecker: MXFP4 output
    if (L.fmt != kFmtMxfp4) return cudaErrorInvalidValue;
    return L.bf16 ? launch_impl<true, kFmtMxfp4, true>(&L, &a, 1) : launch_impl<false, kFmtMxfp4, true>(&L, &a, 1);
  }
  switch (L.fmt) {
    case kFmtMxfp4: return L.bf16 ? launch_impl<true, kFmtMxfp4>(&L, &a, 1) : launch_impl<false, kFmtMxfp4>(&L, &a, 1);
    case kFmtMxfp8: return L.bf16 ? launch_impl<true, kFmtMxfp8>(&L, &a, 1) : launch_impl<false, kFmtMxfp8>(&L, &a, 1);
    case kFmtNvfp4: return L.bf16 ? launch_impl<true, kFmtNvfp4>(&L, &a, 1) : launch_impl<false, kFmtNvfp4>(&L, &a, 1);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quant_act_group(const QuantLaunch* Ls, int count) {
  if (count < 1 || count > kMaxQuantGroup) return cudaErrorInvalidValue;
  // Each activation takes the kernel its own launch_quant_act would take, so
  // the codes are the same: one launch for those of the tensor-core kernel,
  // one for the bf16 and one for the fp32 ones of the CUDA-core kernel.
  QuantLaunch part[3][kMaxQuantGroup];
  QuantArgs args[3][kMaxQuantGroup];
  int n[3] = {0, 0, 0};
  for (int q = 0; q < count; ++q) {
    const QuantLaunch& L = Ls[q];
    if (L.fmt != kFmtMxfp4 || L.gamma != nullptr || L.row_scale != nullptr || L.A_blocks != nullptr ||
        L.row_map != nullptr || L.amax_out != nullptr)
      return cudaErrorInvalidValue;
    const long long tc_tiles = (long long)((L.N / 32 + 3) / 4) * ((L.S + 127) / 128);
    const int k = (L.bf16 && tc_tiles >= 6LL * sm_count()) ? 0 : (L.bf16 ? 1 : 2);
    part[k][n[k]] = L;
    part[k][n[k]].stream = Ls[0].stream;
    args[k][n[k]] = make_args(L);
    args[k][n[k]].err = Ls[0].err;
    ++n[k];
  }
  cudaError_t e = cudaSuccess;
  if (n[0] > 0) e = launch_quant_act_tc_group(part[0], args[0], n[0]);
  if (e == cudaSuccess && n[1] > 0) e = launch_impl<true, kFmtMxfp4, false, false, kMaxQuantGroup>(part[1], args[1], n[1]);
  if (e == cudaSuccess && n[2] > 0) e = launch_impl<false, kFmtMxfp4, false, false, kMaxQuantGroup>(part[2], args[2], n[2]);
  return e;
}

}  // namespace batq
