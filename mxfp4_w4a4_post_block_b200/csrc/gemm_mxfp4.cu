// k_gemm_mxfp4: W4A4 MXFP4 x MXFP4 block-scaled GEMM on the sm_100a tensor cores.
//
// D[i][j] = sum_k P[i][k] Q[j][k] with P, Q packed E2M1 (K-major, two codes per
// byte) and one E8M0 scale per 32 K elements, fp32 accumulation in tensor
// memory (TMEM).  The W4A4 linear of BATQuant (daily-arxiv summary: weight-side
// transform fused into the weights offline, activation side online; MXFP4 =
// 32 elements sharing one E8M0 scale, thelatestinai.com page, DuQuant++
// abstract) maps onto it as
//   * prefill: P = activations (S rows), Q = fused weights (M rows),
//     out[i][j] = D[i][j], tiles of 128 x 256;
//   * decode (S <= 64): P = weights, Q = activations ("swap"), out[j][i] =
//     D[i][j], tiles of 128 x {16, 32, 64}, so the weight stream fills the
//     128-row MMA and the narrow activation side sits in N.
//
// One CTA computes one output tile; one launch may cover up to eight
// independent products of one tile configuration (a table of tensor maps and
// arguments, each problem's CTAs a contiguous range of the grid), which is
// how a decode step's linears share one launch:
//   warp 0     TMA producer: per stage a 128 x 256-element P tile, a BN x 256
//              Q tile (both 128-byte swizzled) and their scale atoms (1-D bulk
//              copies of the 512-byte 128x4 scale tiles);
//   warp 1     TMEM allocator and MMA issuer: four tcgen05.mma
//              kind::mxf4.block_scale (K = 64 each) per stage, then commits
//              the stage back to the producer;
//   warp 6     copies each stage's scales into TMEM (tcgen05.cp 32x128b.warpx4)
//              and signals the MMA thread (copies issued by the MMA thread
//              itself would serialise with its MMAs);
//   (warps 1 and 6 run their stage loops warp-wide, one elected lane issuing)
//   warps 2-5  epilogue: tcgen05.ld of the accumulator quadrant of each warp,
//              staged through shared memory and written with TMA stores
//              (prefill) or stored directly, coalesced along i (decode).
//
// The same kernel serves the W4A8 variant (E4M3 bytes, kind::mxf8f6f4, K = 32
// per MMA) and NVFP4 operands (packed E2M1 with an E4M3 scale per 16 K,
// kind::mxf4nvf4 block16, four scales per MMA; the epilogue multiplies by
// fp32(1 / (gs_a gs_w)), the per-tensor encode scales of both operands).
#include <cstdint>

#include "host_util.h"
#include "kernels.h"
#include "ptx.cuh"

namespace batq {
namespace {

constexpr int kBM = 128;          // MMA M (rows of P per tile, TMEM lanes)
constexpr int kBKBytes = 128;     // bytes of K per stage and row (256 E2M1 or 128 E4M3 codes)
constexpr int kMmasPerStage = 4;  // an MMA consumes 32 bytes of K per row
constexpr int kThreads = 224;     // 7 warps: producer, MMA, 4 epilogue, scale copies
constexpr int kSfWarp = 6;
constexpr int kSfAtom = 512;      // bytes of one 128-row x 4-scale tile

// kFmt: operand format (Fmt).
template <int BN, bool kSwap, int kStages, int kFmt>
struct GemmCfg {
  static constexpr bool kFp8 = (kFmt == kFmtMxfp8);
  static constexpr bool kNv = (kFmt == kFmtNvfp4);
  static constexpr int kBK = kFp8 ? kBKBytes : 2 * kBKBytes;     // K elements per stage
  static constexpr int kKPerMma = kFp8 ? 32 : 64;                // K elements per MMA
  static constexpr int kSfBlock = kNv ? 16 : 32;                 // K elements per scale
  static constexpr int kSfPerMma = kKPerMma / kSfBlock;          // scales per row and MMA
  static constexpr int kAtoms = kBK / (4 * kSfBlock);            // 4-scale atoms per row and stage
  static constexpr int kPBytes = kBM * kBKBytes;
  static constexpr int kQBytes = BN * kBKBytes;
  static constexpr int kQRowAtoms = BN > 128 ? 2 : 1;           // 128-row scale atoms covering Q rows
  static constexpr int kSfPBytes = kAtoms * kSfAtom;
  static constexpr int kSfQBytes = kAtoms * kQRowAtoms * kSfAtom;
  static constexpr int kStageBytes = (kPBytes + kQBytes + kSfPBytes + kSfQBytes + 1023) / 1024 * 1024;
  // TMEM columns: accumulator, then per stage 4 columns per K atom of P
  // scales and 4 * kQRowAtoms per K atom of Q scales.
  static constexpr int kSfPCols = 4 * kAtoms;
  static constexpr int kSfQCols = 4 * kAtoms * kQRowAtoms;
  static constexpr int kTmemUsed = BN + kStages * (kSfPCols + kSfQCols);
  static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                 : kTmemUsed <= 256 ? 256 : 512;
  static_assert(kTmemUsed <= 512, "TMEM budget");
  static constexpr int kBarBytes = 64 * 8;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
};

struct GemmArgs {
  const uint8_t* p_scales;  // MMA layout of P rows
  const uint8_t* q_scales;  // MMA layout of Q rows
  void* out;
  unsigned* err;
  int rows_p, rows_q;       // valid rows of P and Q
  int rows_p_pad, rows_q_pad;
  int N;                    // K elements
  int kpad;                 // scale columns per row (k rounded up to 4)
  int ldo;
  int tiles_q;              // tiles along Q
  int num_kstages;          // ceil(N / 256)
  const uint8_t* w_codes;   // the weight operand (P when swapped, else Q), for the L2 prefetch
  int w_rows;               // its valid rows
  int early_w;              // the preceding grid does not write the weights: prefetch them before waiting
  const float* gs_a;        // NVFP4 per-tensor encode scales (device, nullable: 1)
  const float* gs_w;
};

// One product of a launch: its tensor maps and arguments.  A launch runs one
// to kG of them (same tile configuration), one CTA per output tile; problem
// p's CTAs are blocks block_begin .. block_begin + its tile count - 1.
struct MxProblem {
  CUtensorMap tm_p, tm_q, tm_out;
  GemmArgs g;
  int block_begin;
};

template <int kG>
struct MxLaunch {
  MxProblem prob[kG];
  int count;
};

template <int BN, bool kSwap, int kStages, bool kOutBF16, int kFmt, int kG>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_mxfp4(const __grid_constant__ MxLaunch<kG> L) {
  using C = GemmCfg<BN, kSwap, kStages, kFmt>;
  int pi = 0;  // this CTA's problem
#pragma unroll
  for (int r = 1; r < kG; ++r)
    if (r < L.count && (int)blockIdx.x >= L.prob[r].block_begin) pi = r;
  const MxProblem& P = L.prob[pi];
  const GemmArgs& g = P.g;
  const int bid = (int)blockIdx.x - P.block_begin;  // this CTA's tile within its problem
  constexpr bool kFp8 = C::kFp8;
  constexpr int kBK = C::kBK, kKPerMma = C::kKPerMma;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* sf_ready = acc_full + 1;  // [kStages] scales of the stage are in TMEM
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sf_ready + kStages);

  // Fetch the TMA descriptors while the barriers and TMEM are set up.
  if (threadIdx.x == 0) {
    tma_prefetch_map(&P.tm_p);
    tma_prefetch_map(&P.tm_q);
    tma_prefetch_map(&P.tm_out);
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_p = bid / g.tiles_q;
  const int tile_q = bid % g.tiles_q;
  const int p0 = tile_p * kBM;
  const int q0 = tile_q * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    for (int s = 0; s < kStages; ++s) mbar_init(&sf_ready[s], 1);
    fence_barrier_init();
    // The next grid in the stream may start its set-up now; it waits for this
    // grid to finish before it touches memory.
    griddep_launch_dependents();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_acc = tmem;
  const uint32_t t_sfp = tmem + BN;
  const uint32_t t_sfq = tmem + BN + kStages * C::kSfPCols;

  const int nks = g.num_kstages;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      if (g.early_w) {
        // This CTA's weight rows (contiguous) and their scale tiles go to L2 while
        // the preceding grid (the linear layer's quantiser) still runs.
        const int w0 = kSwap ? p0 : q0;
        const int wn = min(kSwap ? kBM : BN, g.w_rows - w0);
        const size_t row_bytes = (size_t)(kFp8 ? g.N : g.N >> 1);
        const uint8_t* wbase = g.w_codes + (size_t)w0 * row_bytes;
        const size_t wbytes = (size_t)wn * row_bytes;
        for (size_t off = 0; off < wbytes; off += 65536)
          bulk_prefetch_l2(wbase + off, (uint32_t)(wbytes - off < 65536 ? wbytes - off : 65536));
        const size_t sf_tile = (size_t)(g.kpad >> 2) * kSfAtom;  // one 128-row scale tile
        const uint8_t* wsf = kSwap ? g.p_scales : g.q_scales;
        for (int a = 0; a < (wn + 127) / 128; ++a) bulk_prefetch_l2(wsf + (size_t)((w0 >> 7) + a) * sf_tile, (uint32_t)sf_tile);
      }
      griddep_wait();  // operands may come from the grid just before this one
      const int p_tile_atom = p0 >> 7;  // 128-row scale tile of P
      const int q_tile_atom = q0 >> 7;
      const int q_atoms_valid = min(C::kQRowAtoms, (g.rows_q_pad >> 7) - q_tile_atom);
      int s = 0;
      uint32_t ph = 0;
      for (int ks = 0; ks < nks; ++ks) {
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          set_error(g.err, kErrReleaseTimeout);
          break;
        }
        uint8_t* st = smem + s * C::kStageBytes;
        const int katom0 = ks * C::kAtoms;  // first 4-scale atom of this stage
        const int katoms = min(C::kAtoms, (g.kpad >> 2) - katom0);
        const uint32_t sf_bytes = (uint32_t)katoms * kSfAtom;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(C::kPBytes + C::kQBytes) + sf_bytes * (1 + q_atoms_valid));
        tma_load_2d(st, &P.tm_p, &full[s], ks * kBKBytes, p0);
        tma_load_2d(st + C::kPBytes, &P.tm_q, &full[s], ks * kBKBytes, q0);
        const size_t row_stride = (size_t)(g.kpad >> 2) * kSfAtom;
        bulk_load(st + C::kPBytes + C::kQBytes, g.p_scales + (size_t)p_tile_atom * row_stride + katom0 * kSfAtom,
                  sf_bytes, &full[s]);
        for (int a = 0; a < q_atoms_valid; ++a) {
          bulk_load(st + C::kPBytes + C::kQBytes + C::kSfPBytes + a * C::kAtoms * kSfAtom,
                    g.q_scales + (size_t)(q_tile_atom + a) * row_stride + katom0 * kSfAtom, sf_bytes, &full[s]);
        }
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp runs the loop (warp-uniform state: a loop run by one lane
    // spends many more instructions per MMA); one elected lane issues.
    const bool issuer = elect_one();
    int s = 0;
    uint32_t ph = 0;
    for (int ks = 0; ks < nks; ++ks) {
      if (!mbar_wait_warp(&sf_ready[s], ph)) {
        if (issuer) set_error(g.err, kErrDataTimeout);
        break;
      }
      tc_fence_after_sync();
      const uint64_t dp = sdesc_kmajor_sw128(smem_u32(smem + s * C::kStageBytes));
      const uint64_t dq = dp + (uint64_t)(C::kPBytes >> 4);  // addresses < 2^18: no carry out of the field
      const uint32_t tsfp = t_sfp + s * C::kSfPCols, tsfq = t_sfq + s * C::kSfQCols;
      const int kleft = g.N - ks * kBK;
      const int nmma = kleft >= kBK ? kMmasPerStage : kleft / kKPerMma;
      if (issuer) {
        for (int j = 0; j < nmma; ++j) {
          // MMA j covers scale blocks kb.. of the stage: atom kb / 4, byte
          // kb % 4 of each 4-scale TMEM column (NVFP4: four scales, byte 0).
          const int kb = j * C::kSfPerMma;
          const int a = kb >> 2;
          const int sf_id = kb & 3;
          const uint32_t acc = (ks > 0 || j > 0) ? 1u : 0u;
          // Advance K by 32 bytes inside the 128-byte swizzle atom.
          if constexpr (kFp8)
            tc_mma_mxf8(t_acc, dp + (uint64_t)(j * 2), dq + (uint64_t)(j * 2), idesc_mxf8(kBM, BN, sf_id, sf_id),
                        tsfp + a * 4, tsfq + a * 4 * C::kQRowAtoms, acc);
          else if constexpr (C::kNv)
            tc_mma_nvf4(t_acc, dp + (uint64_t)(j * 2), dq + (uint64_t)(j * 2), idesc_nvf4(kBM, BN), tsfp + a * 4,
                        tsfq + a * 4 * C::kQRowAtoms, acc);
          else
            tc_mma_mxf4(t_acc, dp + (uint64_t)(j * 2), dq + (uint64_t)(j * 2), idesc_mxf4(BN, sf_id, sf_id),
                        tsfp + a * 4, tsfq + a * 4 * C::kQRowAtoms, acc);
        }
        tc_commit(&empty[s]);
      }
      __syncwarp();
      if (++s == kStages) {
        s = 0;
        ph ^= 1;
      }
    }
    // Signal the epilogue once every issued MMA has completed (also on error).
    if (issuer) tc_commit(acc_full);
    __syncwarp();
  } else if (warp == kSfWarp) {
    // ------------------------------ scale copies ------------------------------
    // Warp-wide loop, one elected issuer (as the MMA warp).
    const bool issuer = elect_one();
    int s = 0;
    uint32_t ph = 0;
    for (int ks = 0; ks < nks; ++ks) {
      if (!mbar_wait_warp(&full[s], ph)) {
        if (issuer) set_error(g.err, kErrDataTimeout);
        break;
      }
      tc_fence_after_sync();
      const uint64_t dsfp = sdesc_sf_atom(smem_u32(smem + s * C::kStageBytes) + C::kPBytes + C::kQBytes);
      const uint64_t dsfq = dsfp + (uint64_t)(C::kSfPBytes >> 4);
      const uint32_t tsfp = t_sfp + s * C::kSfPCols, tsfq = t_sfq + s * C::kSfQCols;
      const int kleft = g.N - ks * kBK;
      const int nmma = kleft >= kBK ? kMmasPerStage : kleft / kKPerMma;
      const int atoms = ((nmma - 1) * C::kSfPerMma) / 4 + 1;  // atoms the stage's MMAs read
      if (issuer) {
        for (int a = 0; a < atoms; ++a) {
          tc_cp_32x128b_warpx4(tsfp + a * 4, dsfp + (uint64_t)(a * (kSfAtom >> 4)));
#pragma unroll
          for (int r = 0; r < C::kQRowAtoms; ++r) {
            tc_cp_32x128b_warpx4(tsfq + a * 4 * C::kQRowAtoms + r * 4,
                                 dsfq + (uint64_t)((r * C::kAtoms + a) * (kSfAtom >> 4)));
          }
        }
        tc_commit(&sf_ready[s]);
      }
      __syncwarp();
      if (++s == kStages) {
        s = 0;
        ph ^= 1;
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31 are this warp's
    float alpha = 1.0f;
    if constexpr (C::kNv) {
      // The scales may come from the preceding grid (the weight preparation).
      griddep_wait();
      alpha = __frcp_rn(__fmul_rn(g.gs_a != nullptr ? *g.gs_a : 1.0f, g.gs_w != nullptr ? *g.gs_w : 1.0f));
    }
    auto scaled = [&](uint32_t bits) {
      if constexpr (C::kNv) return __fmul_rn(__uint_as_float(bits), alpha);
      return __uint_as_float(bits);
    };
    if (!mbar_wait(acc_full, 0)) set_error(g.err, kErrMmaTimeout);
    tc_fence_after_sync();
    const uint32_t t_row = t_acc + ((uint32_t)(32 * quad) << 16);
    if constexpr (kSwap) {
      // D[i][j]: i = weight row (this lane), j = token.  out[j][i]: lanes write consecutive i.
      const int i = p0 + 32 * quad + lane;
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld_16cols(t_row + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int tok = q0 + c0 + j;
          if (tok < g.rows_q && i < g.rows_p) {
            if constexpr (kOutBF16) {
              const uint32_t pk = pack_bf16x2(scaled(r[j]), 0.0f);
              reinterpret_cast<uint16_t*>(g.out)[(size_t)tok * g.ldo + i] = (uint16_t)(pk & 0xFFFFu);
            } else {
              reinterpret_cast<float*>(g.out)[(size_t)tok * g.ldo + i] = scaled(r[j]);
            }
          }
        }
      }
    } else {
      // Stage the warp's 32 rows through shared memory (pipeline buffers are
      // idle once the accumulator is complete) and write 32-row boxes with TMA.
      constexpr int kColsPerBox = kOutBF16 ? 64 : 32;  // 128 bytes per box row
      constexpr int kBoxes = BN / kColsPerBox;
      uint8_t* stage_out = smem + (size_t)quad * kBoxes * 4096;
#pragma unroll 1
      for (int bx = 0; bx < kBoxes; ++bx) {
        uint8_t* box = stage_out + bx * 4096;
        uint8_t* rowp = box + lane * 128;
        if constexpr (kOutBF16) {
          uint32_t r0[32], r1[32];
          tmem_ld_32cols(t_row + bx * 64, r0);
          tmem_ld_32cols(t_row + bx * 64 + 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* r = c < 4 ? r0 : r1;
            const int o = (c & 3) * 8;
            uint4 v = make_uint4(pack_bf16x2(scaled(r[o + 0]), scaled(r[o + 1])),
                                 pack_bf16x2(scaled(r[o + 2]), scaled(r[o + 3])),
                                 pack_bf16x2(scaled(r[o + 4]), scaled(r[o + 5])),
                                 pack_bf16x2(scaled(r[o + 6]), scaled(r[o + 7])));
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) = v;
          }
        } else {
          uint32_t r[32];
          tmem_ld_32cols(t_row + bx * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                make_uint4(__float_as_uint(scaled(r[4 * c])), __float_as_uint(scaled(r[4 * c + 1])),
                           __float_as_uint(scaled(r[4 * c + 2])), __float_as_uint(scaled(r[4 * c + 3])));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int bx = 0; bx < kBoxes; ++bx) {
          tma_store_2d(&P.tm_out, stage_out + bx * 4096, q0 + bx * kColsPerBox, p0 + 32 * quad);
        }
        tma_store_commit();
        tma_store_wait_read_all();
      }
      __syncwarp();
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Tensor maps and arguments of one product; its CTA count, or -1 when a map
// cannot be encoded.
template <int BN, bool kSwap, int kStages, bool kOutBF16, int kFmt>
int fill_problem(const GemmLaunch& L, int block_begin, MxProblem* P) {
  using C = GemmCfg<BN, kSwap, kStages, kFmt>;
  constexpr bool kFp8 = C::kFp8;
  const int rows_p = kSwap ? L.M : L.S;
  const int rows_q = kSwap ? L.S : L.M;
  const uint8_t* codes_p = kSwap ? L.w_codes : L.a_codes;
  const uint8_t* codes_q = kSwap ? L.a_codes : L.w_codes;
  const uint64_t row_bytes = (uint64_t)(kFp8 ? L.N : L.N / 2);
  if (!make_map_2d(&P->tm_p, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_p, row_bytes, (uint64_t)rows_p, row_bytes, kBKBytes,
                   kBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return -1;
  if (!make_map_2d(&P->tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_q, row_bytes, (uint64_t)rows_q, row_bytes, kBKBytes,
                   BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return -1;
  if (!kSwap) {
    const uint32_t esz = kOutBF16 ? 2 : 4;
    if (!make_map_2d(&P->tm_out, kOutBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, L.out,
                     (uint64_t)L.M, (uint64_t)L.S, (uint64_t)L.ldo * esz, 128 / esz, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return -1;
  } else {
    P->tm_out = P->tm_q;  // unused in the decode epilogue
  }
  GemmArgs& g = P->g;
  g.p_scales = kSwap ? L.w_scales : L.a_scales;
  g.q_scales = kSwap ? L.a_scales : L.w_scales;
  g.out = L.out;
  g.err = L.err;
  g.rows_p = rows_p;
  g.rows_q = rows_q;
  g.rows_p_pad = (rows_p + 127) / 128 * 128;
  g.rows_q_pad = (rows_q + 127) / 128 * 128;
  g.N = L.N;
  g.kpad = C::kNv ? L.N / 16 : (L.N / 32 + 3) / 4 * 4;  // scale columns (NVFP4: N / 16, a multiple of 4)
  g.ldo = L.ldo;
  g.tiles_q = (rows_q + BN - 1) / BN;
  g.num_kstages = (L.N + C::kBK - 1) / C::kBK;
  g.w_codes = L.w_codes;
  g.w_rows = L.M;
  g.early_w = L.weights_ready ? 1 : 0;
  g.gs_a = L.gs_a;
  g.gs_w = L.gs_w;
  P->block_begin = block_begin;
  return ((rows_p + kBM - 1) / kBM) * g.tiles_q;
}

// Ls[0 .. count-1]: products of one tile configuration, format and output
// type on Ls[0]'s stream.
template <int BN, bool kSwap, int kStages, bool kOutBF16, int kFmt, int kG>
cudaError_t launch_cfg(const GemmLaunch* Ls, int count) {
  using C = GemmCfg<BN, kSwap, kStages, kFmt>;
  if (count < 1 || count > kG) return cudaErrorInvalidValue;
  MxLaunch<kG> T = {};
  long long blocks = 0;
  for (int q = 0; q < count; ++q) {
    const int n = fill_problem<BN, kSwap, kStages, kOutBF16, kFmt>(Ls[q], (int)blocks, &T.prob[q]);
    if (n < 0) return cudaErrorInvalidValue;
    blocks += n;
  }
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  T.count = count;
  auto kern = k_gemm_mxfp4<BN, kSwap, kStages, kOutBF16, kFmt, kG>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = Ls[0].stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, T);
}

template <bool kOutBF16, int kFmt>
cudaError_t launch_dtype(const GemmLaunch& L) {
  if (L.S <= 16) return launch_cfg<16, true, 4, kOutBF16, kFmt, 1>(&L, 1);
  if (L.S <= 32) return launch_cfg<32, true, 4, kOutBF16, kFmt, 1>(&L, 1);
  if (L.S <= 64) return launch_cfg<64, true, 4, kOutBF16, kFmt, 1>(&L, 1);
  if (L.S <= 128) return launch_cfg<256, false, 4, kOutBF16, kFmt, 1>(&L, 1);
  return launch_gemm_pair(L);
}

// Tile configuration of a product with S tokens (0: S <= 16, 1: <= 32, 2: <= 64, 3: <= 128).
int small_s_bucket(int S) { return S <= 16 ? 0 : S <= 32 ? 1 : S <= 64 ? 2 : 3; }

template <bool kOutBF16>
cudaError_t launch_small_group(const GemmLaunch* Ls, int count) {
  switch (small_s_bucket(Ls[0].S)) {
    case 0: return launch_cfg<16, true, 4, kOutBF16, kFmtMxfp4, kMaxGemmGroup>(Ls, count);
    case 1: return launch_cfg<32, true, 4, kOutBF16, kFmtMxfp4, kMaxGemmGroup>(Ls, count);
    case 2: return launch_cfg<64, true, 4, kOutBF16, kFmtMxfp4, kMaxGemmGroup>(Ls, count);
    default: return launch_cfg<256, false, 4, kOutBF16, kFmtMxfp4, kMaxGemmGroup>(Ls, count);
  }
}

}  // namespace

cudaError_t launch_gemm_mxfp4_small_group(const GemmLaunch* Ls, int count) {
  if (count < 1 || count > kMaxGemmGroup) return cudaErrorInvalidValue;
  for (int q = 0; q < count; ++q)
    if (Ls[q].fmt != kFmtMxfp4 || Ls[q].out_bf16 != Ls[0].out_bf16 || Ls[q].S > 128 ||
        small_s_bucket(Ls[q].S) != small_s_bucket(Ls[0].S))
      return cudaErrorInvalidValue;
  return Ls[0].out_bf16 ? launch_small_group<true>(Ls, count) : launch_small_group<false>(Ls, count);
}

cudaError_t launch_gemm_mxfp4(const GemmLaunch& L) {
  switch (L.fmt) {
    case kFmtMxfp4: return L.out_bf16 ? launch_dtype<true, kFmtMxfp4>(L) : launch_dtype<false, kFmtMxfp4>(L);
    case kFmtMxfp8: return L.out_bf16 ? launch_dtype<true, kFmtMxfp8>(L) : launch_dtype<false, kFmtMxfp8>(L);
    case kFmtNvfp4: return L.out_bf16 ? launch_dtype<true, kFmtNvfp4>(L) : launch_dtype<false, kFmtNvfp4>(L);
  }
  return cudaErrorInvalidValue;
}

}  // namespace batq
