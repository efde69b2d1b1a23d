// k_gemm_pair: W4A4 MXFP4 GEMM for prefill shapes on CTA pairs (tcgen05 cta_group::2).
//
// Same product as k_gemm_mxfp4 (out[s][m] = sum_n deq(a)[s][n] deq(w)[m][n],
// fp32 accumulation in TMEM), computed by persistent clusters of two CTAs on
// neighbouring SMs.  One launch runs one to eight independent products (a
// table of tensor maps and shapes in the kernel parameters; their tiles form
// one list), so a batch of linears pays the pipeline fill and drain once.
// A pair owns a 256 (tokens) x 256 (out-features) tile (in a launch whose last
// round would fill at most half of the clusters, that round's tiles run as
// 256 x 128 halves on twice as many clusters):
//   * each CTA loads its own 128 token rows of activation codes and its own
//     128-row half of the weight tile, so one SM moves 64 bytes of operands per
//     tensor-core cycle instead of the 96 a single-CTA 128x256 tile needs;
//   * the leader CTA (rank 0) issues one M=256 x N=256 x K=64 block-scaled MMA
//     per K step for both SMs; its TMA loads and its peer's count on the
//     leader's stage barrier, and its commits arrive on both CTAs' barriers;
//   * each CTA keeps the activation scales of its own rows and the weight
//     scales of all 256 columns in its TMEM (128-row x 4-scale tiles copied
//     with tcgen05.cp 32x128b.warpx4); a dedicated warp issues those copies
//     and signals the MMA warp per stage, because copies issued by the MMA
//     thread itself serialise with its MMAs in the tensor pipe (a stage of
//     six copies and four MMAs takes ~990 cycles inline, ~700 when split);
//   * the MMA and scale-copy warps run their stage loops warp-wide (the loop
//     state stays warp-uniform) and one elected lane issues; a loop run by
//     lane 0 alone spent several more instructions per MMA or copy;
//   * eight epilogue warps per CTA read their 128 accumulator columns (64 of a
//     half tile) into registers, release TMEM for the next tile at once (the
//     arrive on the leader's barrier is a CTA-scope release: a cluster-scope
//     one waited for the SM's operand loads in flight), and write the output
//     through a small per-warp shared-memory box (32 rows x 32 bytes) with TMA
//     stores while the next tile's MMAs run;
//   * three 70 KB stages (two 128-byte swizzle tiles of K each, eight MMAs
//     per stage) keep ~210 KB of operand loads in flight per SM: under full
//     load the L2-to-SM latency is ~1.5 us, and this tile needs 64 bytes per
//     SM per tensor-core cycle.  NVFP4 operands (E4M3 scale per 16 K: twice
//     the scale bytes and TMEM columns per K) use five 38 KB stages of one
//     swizzle tile each, which fit the 512 TMEM columns;
//   * formats: MXFP4 (kind::mxf4, E8M0 per 32 K), MXFP8 x MXFP4-in-E4M3 (the
//     W4A8 variant, kind::mxf8f6f4) and NVFP4 (kind::mxf4nvf4 block16, with
//     the per-tensor factor fp32(1 / (gs_a gs_w)) applied in the epilogue).
// Every barrier wait is bounded; on expiry a bit is set in the device error
// word and the waiting loop ends (TMEM is released and both CTAs still meet
// at the closing cluster barrier).
#include <cstdint>

#include "host_util.h"
#include "kernels.h"
#include "ptx.cuh"

namespace batq {
namespace {

constexpr int kRowsPerCta = 128;       // token rows per CTA (TMEM lanes)
constexpr int kTileM = 256;            // token rows per pair
constexpr int kTileN = 256;            // out-features per pair (MMA N)
constexpr int kHalfN = kTileN / 2;     // weight rows loaded by each CTA
constexpr int kSwTile = 128 * 128;     // one 128-row x 128-byte swizzled operand tile
constexpr int kSfAtom = 512;           // 128 rows x 4 scales
constexpr int kEpiWarps = 8;
constexpr int kSfWarp = 2 + kEpiWarps;          // issues the scale-factor copies
constexpr int kThreads = (3 + kEpiWarps) * 32;

constexpr int kBoxBytes = 1024;                             // one epilogue store box: 32 rows x 32 bytes
constexpr int kStagingBytes = kEpiWarps * kBoxBytes;
constexpr int kTmemCols = 512;

// Per operand format (Fmt).  An MMA consumes 32 bytes of K per row.
template <int kFmt>
struct PairCfg {
  static constexpr bool kFp8 = (kFmt == kFmtMxfp8);
  static constexpr bool kNv = (kFmt == kFmtNvfp4);
  static constexpr int kSwAtoms = kNv ? 1 : 2;               // 128-byte swizzle atoms along K per stage
  static constexpr int kBKBytes = 128 * kSwAtoms;            // bytes of K per stage and row
  static constexpr int kStages = kNv ? 5 : 3;                // ~190-210 KB of operands in flight per SM
  static constexpr int kABytes = kRowsPerCta * kBKBytes;     // own activation rows
  static constexpr int kBBytes = kHalfN * kBKBytes;          // own half of the weight rows
  static constexpr int kBK = kFp8 ? kBKBytes : 2 * kBKBytes;  // K elements per stage
  static constexpr int kKPerMma = kFp8 ? 32 : 64;             // K elements per MMA
  static constexpr int kSfBlock = kNv ? 16 : 32;              // K elements per scale
  static constexpr int kAtoms = kBK / (4 * kSfBlock);         // 4-scale atoms per row and stage
  static constexpr int kSfaBytes = kAtoms * kSfAtom;          // K atoms of own rows
  static constexpr int kSfbBytes = 2 * kAtoms * kSfAtom;      // 2 row atoms x K atoms
  static constexpr int kStageTxBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // bytes one CTA's loads deliver
  static constexpr int kStageBytes = (kStageTxBytes + 1023) / 1024 * 1024;
  static constexpr int kBarOffset = kStages * kStageBytes + kStagingBytes;
  static constexpr int kSmemBytes = kBarOffset + 512 + 1024;
  // TMEM columns: accumulator [0, 256), then per stage 4 columns per atom of
  // activation scales and 8 per atom of weight scales (2 row atoms).
  static constexpr int kSfaCols = 4 * kAtoms;
  static constexpr int kSfbCols = 8 * kAtoms;
  static_assert(kTileN + kStages * (kSfaCols + kSfbCols) <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// One GEMM of a launch: its tensor maps and shape.  A launch runs one to kG
// of them (independent problems of one format and output type) over a single
// list of pair tiles: problem p's tiles are tile_begin .. tile_begin +
// tiles_m * tiles_n - 1, row-major over (token tile, out-feature tile).
struct PairProblem {
  CUtensorMap tm_a, tm_w, tm_w_half, tm_sfa, tm_sfw, tm_out, tm_out_wide;
  int S, M, N;
  int tiles_n;         // pair tiles along out-features
  int tile_begin;      // first tile of this problem in the launch's list
  int num_kstages;     // K stages per tile
  int sf_box_chunks;   // 256-byte scale chunks per row tile in one stage's box (<= 2 * kAtoms)
};

template <int kG>
struct PairLaunch {
  PairProblem prob[kG];
  int count;           // problems in use (1 .. kG)
  int num_tiles;       // tiles of all problems
  int split_begin;     // tiles from here on run as two 128-column halves (num_tiles: none)
  int num_units;       // work units: whole tiles before split_begin, then two halves per tile
  unsigned* err;
  int early_weights;   // weights may be read before waiting for the preceding grid
  const float* gs_a;   // NVFP4 per-tensor encode scales (device, nullable: 1); one problem only
  const float* gs_w;
};

// Problem of tile t (tiles are in problem order).
template <int kG>
__device__ __forceinline__ int problem_of(const PairLaunch<kG>& g, int t) {
  int p = 0;
#pragma unroll
  for (int q = 1; q < kG; ++q)
    if (q < g.count && t >= g.prob[q].tile_begin) p = q;
  return p;
}

// Work unit u: tile t whole (half < 0), or its out-feature columns
// [128 half, 128 half + 128) computed as one M=256 x N=128 accumulation.  A
// launch whose last round of whole tiles would fill at most half of the
// clusters runs those tiles as halves on twice as many clusters instead.
struct Unit {
  int t, half;
};
template <int kG>
__device__ __forceinline__ Unit unit_of(const PairLaunch<kG>& g, int u) {
  if (u < g.split_begin) return Unit{u, -1};
  const int v = u - g.split_begin;
  return Unit{g.split_begin + (v >> 1), v & 1};
}

template <bool kOutBF16, int kFmt, int kG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_gemm_pair(const __grid_constant__ PairLaunch<kG> g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using C = PairCfg<kFmt>;
  constexpr int kStageBytes = C::kStageBytes, kSfaBytes = C::kSfaBytes, kSfaCols = C::kSfaCols,
                kSfbCols = C::kSfbCols, kBK = C::kBK, kKPerMma = C::kKPerMma, kStages = C::kStages,
                kABytes = C::kABytes, kBBytes = C::kBBytes, kSwAtoms = C::kSwAtoms, kBKBytes = C::kBKBytes,
                kSfPerMma = C::kKPerMma / C::kSfBlock;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sf_ready = acc_empty + 1;  // [kStages], leader only: scales of the stage are in TMEM
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sf_ready + kStages);

  // Fetch the TMA descriptors while the barriers and TMEM are set up.
  if (threadIdx.x == 0) {
    for (int p = 0; p < g.count; ++p) {
      tma_prefetch_map(&g.prob[p].tm_a);
      tma_prefetch_map(&g.prob[p].tm_w);
      if (g.split_begin < g.num_tiles) tma_prefetch_map(&g.prob[p].tm_w_half);
      tma_prefetch_map(&g.prob[p].tm_sfa);
      tma_prefetch_map(&g.prob[p].tm_sfw);
      tma_prefetch_map(&g.prob[p].tm_out);
      tma_prefetch_map(&g.prob[p].tm_out_wide);
    }
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;
  const int num_units = g.num_units;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    for (int st = 0; st < kStages; ++st) mbar_init(&sf_ready[st], 1);
    fence_barrier_init();
    // The next grid in the stream may start its set-up now; it waits for this
    // grid to finish before it touches memory.
    griddep_launch_dependents();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncwarp();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_acc = tmem;
  const uint32_t t_sfa = tmem + kTileN;
  const uint32_t t_sfb = tmem + kTileN + kStages * kSfaCols;

  // Every role walks this cluster's work units (cluster_id, cluster_id +
  // num_clusters, ...) and each unit's K stages in the same order: one sequence
  // of stages whose ring slot and phase advance by one per stage.
  if (warp == 0) {
    // ------------------------------ producer (both CTAs) ------------------------------
    if (lane == 0) {
      // Cursor over the sequence: unit u (a tile of problem p or its half hf),
      // K step ks, its first rows.
      int u = cluster_id, ks = 0, p = 0, hf = -1, nks = 0, a_row = 0, w_row = 0;
      auto enter_unit = [&]() {
        if (u >= num_units) return;
        const Unit w = unit_of(g, u);
        p = problem_of(g, w.t);
        hf = w.half;
        const int lt = w.t - g.prob[p].tile_begin;
        a_row = (lt / g.prob[p].tiles_n) * kTileM + (int)rank * kRowsPerCta;
        w_row = (lt % g.prob[p].tiles_n) * kTileN + (hf > 0 ? kHalfN : 0);
        nks = g.prob[p].num_kstages;
      };
      auto advance = [&]() {
        if (++ks == nks) {
          ks = 0;
          u += num_clusters;
          enter_unit();
        }
      };
      // Bytes one CTA's loads deliver per stage: the code tiles (a half unit
      // loads 64 weight rows per CTA) and the scale boxes (one box of own
      // activation scales, one of two weight row tiles).
      auto stage_tx = [&](int q, int h) {
        return (uint32_t)(kABytes + (h < 0 ? kBBytes : kBBytes / 2)) + 3u * (uint32_t)g.prob[q].sf_box_chunks * 256u;
      };
      auto issue_weights = [&](int st_idx, int q, int h, int k_step, int wr) {
        uint8_t* st = smem + st_idx * kStageBytes;
        const uint32_t bar = mapa_shared(smem_u32(&full[st_idx]), 0);
        const CUtensorMap* map = h < 0 ? &g.prob[q].tm_w : &g.prob[q].tm_w_half;
        const int rows = h < 0 ? kHalfN : kHalfN / 2;
#pragma unroll
        for (int a = 0; a < kSwAtoms; ++a)
          tma_load_2d_pair(st + kABytes + a * kSwTile, map, bar, k_step * kBKBytes + a * 128, wr + (int)rank * rows);
        // {2 row tiles} x {sf_box_chunks}; a half unit uses the first row tile
        tma_load_3d_pair(st + kABytes + kBBytes + kSfaBytes, &g.prob[q].tm_sfw, bar, 0, k_step * 2 * C::kAtoms,
                         wr / kRowsPerCta);
      };
      auto issue_activations = [&](int st_idx, int q, int k_step, int ar) {
        uint8_t* st = smem + st_idx * kStageBytes;
        const uint32_t bar = mapa_shared(smem_u32(&full[st_idx]), 0);
#pragma unroll
        for (int a = 0; a < kSwAtoms; ++a)
          tma_load_2d_pair(st + a * kSwTile, &g.prob[q].tm_a, bar, k_step * kBKBytes + a * 128, ar);
        // scale tiles: {256-byte chunk, K chunk (2 per 4-scale atom), 128-row tile}
        tma_load_3d_pair(st + kABytes + kBBytes, &g.prob[q].tm_sfa, bar, 0, k_step * 2 * C::kAtoms,
                         ar / kRowsPerCta);
      };
      enter_unit();
      // When the preceding grid is known not to write the weights (the linear
      // layer's own quantiser), the first ring's weights are loaded before
      // waiting for that grid; the activations always come after the wait.
      // Otherwise both operands of each stage are requested together, so the
      // first stage does not queue behind the later stages' weights.
      int pro_p[kStages], pro_ks[kStages], pro_a[kStages];
      int npro = 0;
      if (!g.early_weights) griddep_wait();
      while (npro < kStages && u < num_units) {
        if (leader) mbar_arrive_expect_tx(&full[npro], 2u * stage_tx(p, hf));
        issue_weights(npro, p, hf, ks, w_row);
        if (!g.early_weights) issue_activations(npro, p, ks, a_row);
        pro_p[npro] = p;
        pro_ks[npro] = ks;
        pro_a[npro] = a_row;
        ++npro;
        advance();
      }
      if (g.early_weights) {
        griddep_wait();
        for (int i = 0; i < npro; ++i) issue_activations(i, pro_p[i], pro_ks[i], pro_a[i]);
      }
      int s = npro % kStages;
      uint32_t ph = npro == kStages ? 1u : 0u;
      while (u < num_units) {
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          set_error(g.err, kErrReleaseTimeout);
          break;
        }
        if (leader) mbar_arrive_expect_tx(&full[s], 2u * stage_tx(p, hf));
        issue_weights(s, p, hf, ks, w_row);
        issue_activations(s, p, ks, a_row);
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
        advance();
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader only) ------------------------------
    // Stage g's scales are already in TMEM slot g % kStages when sf_ready fires.
    // The whole warp runs the loop, so its state stays warp-uniform (a loop run
    // by one lane spends many more instructions per MMA), and one elected lane
    // issues the MMAs and commits.
    if (leader) {
      const bool issuer = elect_one();
      int st_idx = 0;
      uint32_t sph = 0, tile_iter = 0;
      bool ok = true;
      for (int u = cluster_id; u < num_units && ok; u += num_clusters, ++tile_iter) {
        const Unit w = unit_of(g, u);
        const int p = problem_of(g, w.t);
        const int nks = g.prob[p].num_kstages, N = g.prob[p].N;
        const int mma_n = w.half < 0 ? kTileN : kTileN / 2;
        for (int ks = 0; ks < nks; ++ks) {
          if (ks == 0) {
            // The accumulator must have been drained by both CTAs' epilogues.
            if (!mbar_wait_warp(acc_empty, (tile_iter & 1) ^ 1)) {
              if (issuer) set_error(g.err, kErrDrainTimeout);
              ok = false;
              break;
            }
            tc_fence_after_sync();
          }
          if (!mbar_wait_warp(&sf_ready[st_idx], sph)) {
            if (issuer) set_error(g.err, kErrDataTimeout);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          // Shared addresses stay below 2^18, so the descriptor of base + off is
          // the base descriptor + off / 16.
          const uint64_t da0 = sdesc_kmajor_sw128(smem_u32(smem + st_idx * kStageBytes));
          const uint64_t db0 = da0 + (uint64_t)(kABytes >> 4);
          const uint32_t tsfa = t_sfa + st_idx * kSfaCols, tsfb = t_sfb + st_idx * kSfbCols;
          const int kleft = N - ks * kBK;
          const int nmma = kleft >= kBK ? kBK / kKPerMma : kleft / kKPerMma;
          if (issuer) {
            for (int j = 0; j < nmma; ++j) {
              // MMA j covers scale blocks kb.. of the stage: atom kb / 4, byte
              // kb % 4 of each 4-scale TMEM column (NVFP4: four scales, byte 0).
              const int kb = j * kSfPerMma;
              const int a = kb >> 2;
              const int sf_id = kb & 3;
              // Bytes 32j.. of the stage's K: swizzle tile j / 4, then 32 bytes per
              // MMA inside its 128-byte swizzle atom.
              const uint64_t off = (uint64_t)((j >> 2) * (kSwTile >> 4) + (j & 3) * 2);
              const uint32_t acc = (ks > 0 || j > 0) ? 1u : 0u;
              if constexpr (C::kFp8)
                tc_mma_pair_mxf8(t_acc, da0 + off, db0 + off, idesc_mxf8(256, mma_n, sf_id, sf_id), tsfa + a * 4,
                                 tsfb + a * 8, acc);
              else if constexpr (C::kNv)
                tc_mma_pair_nvf4(t_acc, da0 + off, db0 + off, idesc_nvf4(256, mma_n), tsfa + a * 4, tsfb + a * 8,
                                 acc);
              else
                tc_mma_pair_mxf4(t_acc, da0 + off, db0 + off, idesc_mxf4_m256(mma_n, sf_id, sf_id), tsfa + a * 4,
                                 tsfb + a * 8, acc);
            }
            tc_commit_pair(&empty[st_idx], 0x3);
            // Both epilogues may read the accumulator once every MMA of the tile has completed.
            if (ks == nks - 1) tc_commit_pair(acc_full, 0x3);
          }
          __syncwarp();
          if (++st_idx == kStages) {
            st_idx = 0;
            sph ^= 1u;
          }
        }
      }
    }
  } else if (warp == kSfWarp) {
    // ---------------------- scale-factor copies (leader only) ----------------------
    // Stage g's data has landed (full) -> copy its scale tiles into TMEM slot
    // g % kStages in both CTAs -> sf_ready.  The slot's previous contents were
    // consumed by the MMAs of stage g - kStages, which completed before the
    // producer could refill the stage.  Warp-wide loop, one elected issuer.
    if (leader) {
      const bool issuer = elect_one();
      int st_idx = 0;
      uint32_t fph = 0;
      bool ok = true;
      for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
        const Unit w = unit_of(g, u);
        const int p = problem_of(g, w.t);
        const int nks = g.prob[p].num_kstages, N = g.prob[p].N, box_chunks = g.prob[p].sf_box_chunks;
        const bool whole = w.half < 0;  // a half unit's N = 128 columns need one weight row tile
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait_warp(&full[st_idx], fph)) {
            if (issuer) set_error(g.err, kErrDataTimeout);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const int kleft = N - ks * kBK;
          const int nmma = kleft >= kBK ? kBK / kKPerMma : kleft / kKPerMma;
          const uint64_t dsfa = sdesc_sf_atom(smem_u32(smem + st_idx * kStageBytes) + kABytes + kBBytes);
          const uint64_t dsfb = dsfa + (uint64_t)(kSfaBytes >> 4);
          const uint64_t dsfb1 = dsfb + (uint64_t)((box_chunks * 256) >> 4);
          const uint32_t tsfa = t_sfa + st_idx * kSfaCols, tsfb = t_sfb + st_idx * kSfbCols;
          const int atoms = ((nmma - 1) * kSfPerMma) / 4 + 1;  // atoms the stage's MMAs read
          if (issuer) {
            for (int a = 0; a < atoms; ++a) {
              const uint64_t off = (uint64_t)(a * (kSfAtom >> 4));
              tc_cp_pair_32x128b_warpx4(tsfa + a * 4, dsfa + off);
              // weight-scale box is {2 row tiles} x {sf_box_chunks}: row tile r, atom a at
              // r * sf_box_chunks * 256 + a * 512
              tc_cp_pair_32x128b_warpx4(tsfb + a * 8, dsfb + off);
              if (whole) tc_cp_pair_32x128b_warpx4(tsfb + a * 8 + 4, dsfb1 + off);
            }
            tc_commit_pair_local(&sf_ready[st_idx]);
          }
          __syncwarp();
          if (++st_idx == kStages) {
            st_idx = 0;
            fph ^= 1u;
          }
        }
      }
    }
  } else if (warp >= 2 && warp < 2 + kEpiWarps) {
    // ------------------------------ epilogue (both CTAs) ------------------------------
    const int ew = warp - 2;
    const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
    uint8_t* box = smem + kStages * kStageBytes + ew * kBoxBytes;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    uint32_t tile_iter = 0;
    bool store_pending = false;
    float alpha = 1.0f;
    if constexpr (C::kNv) {
      // The scales may come from the preceding grid (the weight preparation).
      griddep_wait();
      alpha = __frcp_rn(__fmul_rn(g.gs_a != nullptr ? *g.gs_a : 1.0f, g.gs_w != nullptr ? *g.gs_w : 1.0f));
    }
    // accumulator bits -> output value (NVFP4: times the per-tensor factor)
    auto scaled = [&](uint32_t bits) {
      if constexpr (C::kNv) return __fmul_rn(__uint_as_float(bits), alpha);
      return __uint_as_float(bits);
    };
    for (int u = cluster_id; u < num_units; u += num_clusters, ++tile_iter) {
      const Unit w = unit_of(g, u);
      const PairProblem& P = g.prob[problem_of(g, w.t)];
      const int lt = w.t - P.tile_begin;
      // This warp's accumulator columns: half of the unit's 256 (whole tile) or 128.
      const int wcols = w.half < 0 ? 128 : 64;
      const int col0 = (ew >> 2) * wcols;
      const int row0 = (lt / P.tiles_n) * kTileM + (int)rank * kRowsPerCta + 32 * quad;
      const int n0 = (lt % P.tiles_n) * kTileN + (w.half > 0 ? kHalfN : 0) + col0;
      if (!mbar_wait_warp(acc_full, tile_iter & 1)) {
        if (lane == 0) set_error(g.err, kErrMmaTimeout);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      uint32_t v[4][32];
      const uint32_t taddr = t_acc + ((uint32_t)(32 * quad) << 16) + col0;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (32 * c < wcols) tmem_ld_32cols(taddr + 32 * c, v[c]);
      tmem_ld_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);  // TMEM free for the next tile

      const bool last_unit = (u + num_clusters >= num_units);
      if (last_unit) {
        // Nothing is loaded after the last unit, and its MMAs have completed,
        // so the operand stages are idle: each warp stages its whole 32-row
        // block there (128-byte rows, 128-byte swizzle) and issues all of its
        // stores at once instead of one small box at a time.
        if (store_pending) {
          if (lane == 0) tma_store_wait_read_all();
          __syncwarp();
        }
        constexpr int kWideCols = kOutBF16 ? 64 : 32;   // 128-byte box rows
        constexpr int kWideBoxes = 128 / kWideCols;
        uint8_t* wide = smem + ew * (kWideBoxes * 4096);
#pragma unroll
        for (int bx = 0; bx < kWideBoxes; ++bx) {
          if (bx * kWideCols >= wcols) break;
          uint8_t* wrow = wide + bx * 4096 + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 q;
            if constexpr (kOutBF16) {
              const uint32_t* r = v[2 * bx + (c >> 2)] + (c & 3) * 8;
              q = make_uint4(pack_bf16x2(scaled(r[0]), scaled(r[1])), pack_bf16x2(scaled(r[2]), scaled(r[3])),
                             pack_bf16x2(scaled(r[4]), scaled(r[5])), pack_bf16x2(scaled(r[6]), scaled(r[7])));
            } else {
              const uint32_t* r = v[bx] + 4 * c;
              q = make_uint4(__float_as_uint(scaled(r[0])), __float_as_uint(scaled(r[1])),
                             __float_as_uint(scaled(r[2])), __float_as_uint(scaled(r[3])));
            }
            *reinterpret_cast<uint4*>(wrow + ((c ^ (lane & 7)) << 4)) = q;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < P.S) {
          for (int bx = 0; bx < kWideBoxes; ++bx) {
            const int x = n0 + bx * kWideCols;
            if (bx * kWideCols < wcols && x < P.M) tma_store_2d(&P.tm_out_wide, wide + bx * 4096, x, row0);
          }
          tma_store_commit();
        }
        store_pending = true;
        continue;
      }

      // 32-byte box rows: 8 fp32 or 16 bf16 columns; 32-byte swizzle (16-byte
      // chunk c of row r stored at chunk c ^ ((r >> 2) & 1)).
      constexpr int kColsPerBox = kOutBF16 ? 16 : 8;
      uint8_t* rowp = box + lane * 32;
      const int sw = (lane >> 2) & 1;
#pragma unroll
      for (int bx = 0; bx < 128 / kColsPerBox; ++bx) {
        if (bx * kColsPerBox >= wcols) break;
        if (store_pending) {
          if (lane == 0) tma_store_wait_read_all();
          __syncwarp();
        }
        if constexpr (kOutBF16) {
          const uint32_t* r = v[bx >> 1] + (bx & 1) * 16;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int o = c * 8;
            *reinterpret_cast<uint4*>(rowp + ((c ^ sw) << 4)) =
                make_uint4(pack_bf16x2(scaled(r[o + 0]), scaled(r[o + 1])),
                           pack_bf16x2(scaled(r[o + 2]), scaled(r[o + 3])),
                           pack_bf16x2(scaled(r[o + 4]), scaled(r[o + 5])),
                           pack_bf16x2(scaled(r[o + 6]), scaled(r[o + 7])));
          }
        } else {
          const uint32_t* r = v[bx >> 2] + (bx & 3) * 8;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            *reinterpret_cast<uint4*>(rowp + ((c ^ sw) << 4)) =
                make_uint4(__float_as_uint(scaled(r[4 * c])), __float_as_uint(scaled(r[4 * c + 1])),
                           __float_as_uint(scaled(r[4 * c + 2])), __float_as_uint(scaled(r[4 * c + 3])));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int x = n0 + bx * kColsPerBox;
        if (lane == 0 && row0 < P.S && x < P.M) {
          tma_store_2d(&P.tm_out, box, x, row0);
          tma_store_commit();
        }
        store_pending = true;
      }
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncwarp();
  cluster_sync_all();  // all MMAs done and all TMEM reads finished in both CTAs
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// Tensor maps and shape of one problem; false when a map cannot be encoded.
template <bool kOutBF16, int kFmt>
bool fill_problem(const GemmLaunch& L, int tile_begin, PairProblem* P) {
  using C = PairCfg<kFmt>;
  const uint64_t row_bytes = (uint64_t)(C::kFp8 ? L.N : L.N / 2);
  // Code tiles: boxes of 128 rows x 128 bytes (one swizzle atom); a stage takes kSwAtoms of them.
  // Scale columns per row: k = N / 32 rounded up to 4 (MX), N / 16 (NVFP4, a multiple of 4).
  const int kpad = C::kNv ? L.N / 16 : (L.N / 32 + 3) / 4 * 4;
  const uint64_t sf_row_tile_bytes = (uint64_t)(kpad / 4) * kSfAtom;
  const uint64_t a_tiles = (uint64_t)(L.S + 127) / 128;
  const uint64_t w_tiles = (uint64_t)(L.M + 127) / 128;
  if (!make_map_2d(&P->tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.a_codes, row_bytes, (uint64_t)L.S, row_bytes, 128,
                   kRowsPerCta, CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  if (!make_map_2d(&P->tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.w_codes, row_bytes, (uint64_t)L.M, row_bytes, 128,
                   kHalfN, CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  // Half units: 64 weight rows per CTA.
  if (!make_map_2d(&P->tm_w_half, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.w_codes, row_bytes, (uint64_t)L.M, row_bytes, 128,
                   kHalfN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  // Scale tiles as {256-byte chunks, chunks per row tile, row tiles}; one box = the stage's K
  // atoms (x 2 row tiles for the weights), clamped to the row tile when all of K is shorter.
  const uint64_t chunks = sf_row_tile_bytes / 256;
  const int box_chunks = (int)(chunks < (uint64_t)(2 * C::kAtoms) ? chunks : (uint64_t)(2 * C::kAtoms));
  if (!make_map_3d(&P->tm_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.a_scales, 256, chunks, a_tiles, 256,
                   sf_row_tile_bytes, 256, box_chunks, 1))
    return false;
  if (!make_map_3d(&P->tm_sfw, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.w_scales, 256, chunks, w_tiles, 256,
                   sf_row_tile_bytes, 256, box_chunks, 2))
    return false;
  const uint32_t esz = kOutBF16 ? 2 : 4;
  if (!make_map_2d(&P->tm_out, kOutBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, L.out,
                   (uint64_t)L.M, (uint64_t)L.S, (uint64_t)L.ldo * esz, 32 / esz, 32, CU_TENSOR_MAP_SWIZZLE_32B))
    return false;
  if (!make_map_2d(&P->tm_out_wide, kOutBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   L.out, (uint64_t)L.M, (uint64_t)L.S, (uint64_t)L.ldo * esz, 128 / esz, 32,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  P->S = L.S;
  P->M = L.M;
  P->N = L.N;
  P->tiles_n = (L.M + kTileN - 1) / kTileN;
  P->tile_begin = tile_begin;
  P->num_kstages = (L.N + C::kBK - 1) / C::kBK;
  P->sf_box_chunks = box_chunks;
  return true;
}

// Ls[0 .. count-1]: problems of one format and output type on one stream;
// the first supplies the launch-wide fields (error word, weights_ready, NVFP4 scales).
template <bool kOutBF16, int kFmt, int kG>
cudaError_t launch_pair_impl(const GemmLaunch* Ls, int count) {
  using C = PairCfg<kFmt>;
  if (count < 1 || count > kG) return cudaErrorInvalidValue;
  PairLaunch<kG> g = {};
  int tiles = 0;
  for (int p = 0; p < count; ++p) {
    if (!fill_problem<kOutBF16, kFmt>(Ls[p], tiles, &g.prob[p])) return cudaErrorInvalidValue;
    tiles += ((Ls[p].S + kTileM - 1) / kTileM) * g.prob[p].tiles_n;
  }
  g.count = count;
  g.num_tiles = tiles;
  // A last round of whole tiles that would occupy at most half of the clusters
  // runs as half tiles (M = 256 x N = 128) on twice as many: that round then
  // takes the time of half a tile's MMAs and operand stream instead of a whole
  // one's.  Each output element is still one K accumulation in one MMA chain.
  const int max_clusters = sm_count() / 2;
  const int rem = tiles % max_clusters;
  const bool split = rem > 0 && 2 * rem <= max_clusters;
  g.split_begin = split ? tiles - rem : tiles;
  g.num_units = split ? tiles + rem : tiles;
  g.err = Ls[0].err;
  g.early_weights = Ls[0].weights_ready ? 1 : 0;
  g.gs_a = Ls[0].gs_a;
  g.gs_w = Ls[0].gs_w;

  auto kern = k_gemm_pair<kOutBF16, kFmt, kG>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int clusters = g.num_units < max_clusters ? g.num_units : max_clusters;
  // Launched as a programmatic dependent of the preceding grid: set-up and
  // weight loads overlap the quantiser's tail; activations wait for it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = Ls[0].stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, g);
}

}  // namespace

cudaError_t launch_gemm_pair(const GemmLaunch& L) {
  switch (L.fmt) {
    case kFmtMxfp4:
      return L.out_bf16 ? launch_pair_impl<true, kFmtMxfp4, 1>(&L, 1) : launch_pair_impl<false, kFmtMxfp4, 1>(&L, 1);
    case kFmtMxfp8:
      return L.out_bf16 ? launch_pair_impl<true, kFmtMxfp8, 1>(&L, 1) : launch_pair_impl<false, kFmtMxfp8, 1>(&L, 1);
    case kFmtNvfp4:
      return L.out_bf16 ? launch_pair_impl<true, kFmtNvfp4, 1>(&L, 1) : launch_pair_impl<false, kFmtNvfp4, 1>(&L, 1);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_pair_group(const GemmLaunch* Ls, int count) {
  if (count < 1 || count > kMaxGemmGroup) return cudaErrorInvalidValue;
  for (int p = 0; p < count; ++p)
    if (Ls[p].fmt != kFmtMxfp4 || Ls[p].out_bf16 != Ls[0].out_bf16 || Ls[p].S <= 128) return cudaErrorInvalidValue;
  return Ls[0].out_bf16 ? launch_pair_impl<true, kFmtMxfp4, kMaxGemmGroup>(Ls, count)
                        : launch_pair_impl<false, kFmtMxfp4, kMaxGemmGroup>(Ls, count);
}

}  // namespace batq
