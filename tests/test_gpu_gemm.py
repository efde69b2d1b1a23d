"""GPU parity of batq_gemm_mxfp4, batq_prepare_weights and batq_linear against the oracle."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu


def _random_operands(S, M, N, seed):
    """Random MXFP4 operands: every code value (incl. -0) and scales over a wide range."""
    rng = np.random.default_rng(seed)
    k = N // 32
    a = rng.integers(0, 256, (S, N // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (M, N // 2), dtype=np.uint8)
    sa = rng.integers(100, 150, (S, k), dtype=np.uint8)
    sw = rng.integers(100, 150, (M, k), dtype=np.uint8)
    return a, sa, w, sw


def _run(a, sa, w, sw, out_dtype=torch.float32):
    S, M, N = a.shape[0], w.shape[0], 2 * a.shape[1]
    k = N // 32
    out = GU.gpu_gemm(GU.to_dev_u8(a), GU.to_dev_u8(PT.to_mma_layout(sa, S, k)), GU.to_dev_u8(w),
                      GU.to_dev_u8(PT.to_mma_layout(sw, M, k)), S, M, N, out_dtype)
    return out.float().cpu().numpy()


@pytest.mark.parametrize("S,M,N", [
    (16, 128, 256),     # decode path (activations in N), one K stage
    (4, 64, 64),        # M below one 128-row tile, single MMA
    (1, 272, 320),      # partial K stage, M not a multiple of 128
    (33, 160, 512),     # N = 64 decode tile
    (64, 256, 1024),
    (65, 256, 512),     # smallest prefill-path S
    (128, 256, 256),
    (200, 272, 320),    # ragged everything on the prefill path
    (300, 1024, 768),
    (129, 256, 256),    # smallest CTA-pair path, second CTA nearly empty
    (1000, 1280, 512),  # several pair tiles per cluster row
    (520, 4096, 256),   # 3 x 16 = 48 pair tiles (one per cluster), ragged last row band
    (2048, 4096, 256),  # 8 x 16 = 128 pair tiles on 74 clusters: 54 clusters run two
])
def test_gemm_random_operands(S, M, N):
    a, sa, w, sw = _random_operands(S, M, N, S * 7 + M + N)
    out = _run(a, sa, w, sw)
    ref, T = O.gemm(a, sa, w, sw)
    PT.assert_gemm_parity(out, ref, T, f"{S}x{M}x{N}")


def band_rows(S, seed):
    """Two rows from every 256-row band of pair tiles, one in each CTA's 128 rows, in 32-row quarters
    that rotate from band to band (each quarter is drained by its own epilogue warp), and the last
    row.  With all M columns these rows touch every output tile of the pair GEMM, so every tile of
    every cluster's persistent sequence, its last tile included, is compared."""
    rng = np.random.default_rng(seed)
    rows = [S - 1]
    for b in range(-(-S // 256)):
        for half in (0, 1):
            r = b * 256 + half * 128 + ((b + 2 * half) % 4) * 32 + int(rng.integers(0, 32))
            if r < S:
                rows.append(r)
    return np.unique(np.array(rows, dtype=np.int64))


@pytest.mark.parametrize("S,M,N", [
    (4096, 4096, 12288),   # down_proj: K = 12288 (24 K stages), 16 x 16 = 256 pair tiles (3-4 per cluster)
    (8192, 12288, 4096),   # layer gate / up: 32 x 48 = 1536 pair tiles (20-21 per cluster)
    (8192, 1024, 4096),    # layer k / v: 32 x 4 = 128 pair tiles
    (8192, 4096, 12288),   # layer down: 512 pair tiles, K = 12288
    (3000, 8192, 128),     # one partial K stage per tile, 12 x 32 = 384 pair tiles, ragged last band
])
def test_gemm_large_shapes_every_pair_tile(S, M, N):
    """The persistent pair GEMM at the prefill shapes of the down_proj and layer workloads (random
    operands over every code value), compared on rows that touch every pair tile."""
    a, sa, w, sw = _random_operands(S, M, N, S + 3 * M + 7 * N)
    k = N // 32
    out = GU.gpu_gemm(GU.to_dev_u8(a), GU.to_dev_u8(PT.to_mma_layout(sa, S, k)), GU.to_dev_u8(w),
                      GU.to_dev_u8(PT.to_mma_layout(sw, M, k)), S, M, N)
    rows = band_rows(S, S + M)
    got = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    del out
    ref, T = O.gemm_rows(a, sa, w, sw, rows)
    PT.assert_gemm_parity(got, ref, T, f"{S}x{M}x{N}")


@pytest.mark.parametrize("S", [16, 200])
def test_gemm_bf16_output(S):
    a, sa, w, sw = _random_operands(S, 256, 512, 3 + S)
    out = _run(a, sa, w, sw, torch.bfloat16)
    ref, T = O.gemm(a, sa, w, sw)
    # bf16 output: the fp32 result is rounded once more (relative 2^-8 of |out| <= T).
    err = np.abs(out - ref)
    assert np.all(err <= 1e-4 * T + 2.0 ** -8 * np.abs(ref) + 1e-30)


def test_gemm_tiny_config_oracle_codes():
    w = WL.tiny()
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    wp = O.prepare_weights(w.W, w.A, w.B)
    out = _run(act["codes"], act["scales"], wp["codes"], wp["scales"])
    ref, T = O.gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    PT.assert_gemm_parity(out, ref, T, "tiny")


def test_gemm_q_proj_full_sampled_rows():
    w = WL.q_proj()
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    wp = O.prepare_weights(w.W, w.A, w.B)
    out = _run(act["codes"], act["scales"], wp["codes"], wp["scales"])
    rows = np.sort(np.random.default_rng(21).choice(w.S, 96, replace=False))
    ref, T = O.gemm_rows(act["codes"], act["scales"], wp["codes"], wp["scales"], rows)
    PT.assert_gemm_parity(out[rows], ref, T, "q_proj")


@pytest.mark.parametrize("S", [1, 4, 16])
def test_gemm_decode_full(S):
    w = WL.decode(S, with_w=False)
    rng = np.random.default_rng(30 + S)
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    wc = rng.integers(0, 256, (w.M, w.N // 2), dtype=np.uint8)
    ws = rng.integers(110, 135, (w.M, w.k), dtype=np.uint8)
    out = _run(act["codes"], act["scales"], wc, ws)
    ref, T = O.gemm(act["codes"], act["scales"], wc, ws)
    PT.assert_gemm_parity(out, ref, T, f"decode{S}")


# ------------------------------------------------------------ weight side ----

@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(48, 320, 272, 41)])
def test_prepare_weights_parity(maker):
    w = maker()
    codes, scales = GU.gpu_prepare(w)
    ref = O.prepare_weights(w.W, w.A, w.B)
    lin = O.scales_from_mma_layout(scales.cpu().numpy(), w.M, w.k)
    r = PT.assert_quant_parity(codes.cpu().numpy(), lin, {"q": ref["q"], "Y_hat": ref["W_fused"],
                                                          "codes": ref["codes"], "scales": ref["scales"]},
                               "prepare", cond=PT.condition_scale_weights(w.W, w.A, w.B))
    print("prepare mismatches", r)


def test_prepare_weights_q_proj():
    w = WL.q_proj()
    codes, scales = GU.gpu_prepare(w)
    ref = O.prepare_weights(w.W, w.A, w.B)
    lin = O.scales_from_mma_layout(scales.cpu().numpy(), w.M, w.k)
    r = PT.assert_quant_parity(codes.cpu().numpy(), lin, {"q": ref["q"], "Y_hat": ref["W_fused"],
                                                          "codes": ref["codes"], "scales": ref["scales"]},
                               "prepare q_proj", cond=PT.condition_scale_weights(w.W, w.A, w.B))
    print("prepare q_proj mismatches", r)


def test_prepare_rejects_singular_transform():
    w = WL.tiny()
    w.B[3] = 0.0
    with pytest.raises(BQ.BatqError) as ei:
        GU.gpu_prepare(w)
    assert ei.value.status == 4


# ---------------------------------------------------------------- linear ----

def _linear(w, out_dtype=torch.float32):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc = GU.gpu_prepare(w)
    ws = torch.empty(BQ.batq_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=out_dtype, device="cuda")
    BQ.batq_linear(X, w.A, B, ratios, wc, wsc, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    return out, wc, wsc


@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(200, 320, 272, 51),
                                   lambda: WL.custom(100, 320, 272, 52),
                                   lambda: WL.q_proj(), lambda: WL.decode(4), lambda: WL.decode(16)])
def test_linear_matches_quant_then_gemm_and_oracle(maker):
    w = maker()
    out, wc, wsc = _linear(w)
    # composition: identical to the two calls made separately
    codes, lin, _, raw = GU.gpu_quant(w, BQ.BATQ_SCALES_MMA, y_debug=False)
    out2 = GU.gpu_gemm(GU.to_dev_u8(codes), GU.to_dev_u8(raw), wc, wsc, w.S, w.M, w.N)
    assert torch.equal(out, out2)
    # oracle GEMM on the same operands (sampled rows for the large case)
    rows = np.arange(w.S) if w.S <= 256 else np.sort(np.random.default_rng(5).choice(w.S, 64, replace=False))
    wl = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    ref, T = O.gemm_rows(codes, lin, wc.cpu().numpy(), wl, rows)
    PT.assert_gemm_parity(out.cpu().numpy()[rows], ref, T, "linear")
    # and the activations themselves match the oracle's (boundary exemptions only)
    act = O.quant_act(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity(codes[rows], lin[rows], act, "linear act", cond=PT.condition_scale(w.x[rows], w.A, w.B))


def test_linear_error_vs_unquantised_matches_oracle():
    """The W4A4 output's distance from the unquantised x W^T is the oracle's."""
    w = WL.tiny()
    out, _, _ = _linear(w)
    exact = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    ref, _, _, _ = O.linear(w.x, w.A, w.B, w.alpha_min, w.alpha_max, w.W)
    rel_gpu = np.linalg.norm(out.cpu().numpy() - exact) / np.linalg.norm(exact)
    rel_ref = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert abs(rel_gpu - rel_ref) < 1e-3 * rel_ref + 1e-6, (rel_gpu, rel_ref)


def test_linear_with_block_hadamard_transform():
    """Block Hadamard P_i (orthogonal, so the fused weights are W P_i) through batq_linear matches
    the oracle, and its distance from x W^T is the oracle's."""
    w = WL.with_block_hadamard(WL.custom(96, 512, 256, 77))
    out, wc, wsc = _linear(w)
    ref, T, act, wp = O.linear(w.x, w.A, w.B, w.alpha_min, w.alpha_max, w.W)
    lin = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    PT.assert_quant_parity(wc.cpu().numpy(), lin, {"q": wp["q"], "Y_hat": wp["W_fused"], "codes": wp["codes"],
                                                    "scales": wp["scales"]}, "hadamard weights",
                           cond=PT.condition_scale_weights(w.W, w.A, w.B), literal_limit=PT.LITERAL_LIMIT_HADAMARD)
    exact = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    rel_gpu = np.linalg.norm(out.cpu().numpy() - exact) / np.linalg.norm(exact)
    rel_ref = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert abs(rel_gpu - rel_ref) < 2e-3 * rel_ref + 1e-6, (rel_gpu, rel_ref)


@pytest.mark.parametrize("maker", [lambda: WL.down_proj(), lambda: WL.layer_linear(1), lambda: WL.layer_linear(4),
                                   lambda: WL.layer_linear(6)],
                         ids=["down_proj", "layer_k", "layer_gate", "layer_down"])
def test_linear_large_end_to_end(maker):
    """batq_linear at the down_proj shape and three linears of the S = 8192 layer, checked stage by
    stage against the oracle: the activation codes and scales it left in its workspace on rows that
    touch every pair tile, the prepared weights on sampled rows, and the GEMM output on the same
    activation rows and every output column (the oracle's fp64 product of the linear's own codes)."""
    w = maker()
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc = GU.gpu_prepare(w)
    ws = torch.empty(BQ.batq_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_linear(X, w.A, B, ratios, wc, wsc, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    rows = band_rows(w.S, w.seed)
    got = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    del out, X
    ws_h = ws.cpu().numpy()
    ncode = w.S * w.N // 2
    codes = ws_h[:ncode].reshape(w.S, w.N // 2)
    off = -(-ncode // 256) * 256
    a_sc = O.scales_from_mma_layout(ws_h[off:off + O.mma_layout_bytes(w.S, w.k)], w.S, w.k)
    act = O.quant_act(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity(codes[rows], a_sc[rows], act, f"{w.name} activations",
                           cond=PT.condition_scale(w.x[rows], w.A, w.B))
    wc_h = wc.cpu().numpy()
    w_sc = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    wrows = np.unique(np.concatenate([np.random.default_rng(w.seed).choice(w.M, 48, replace=False), [w.M - 1]]))
    wp = O.prepare_weights(w.W[wrows], w.A, w.B)
    PT.assert_quant_parity(wc_h[wrows], w_sc[wrows], {"q": wp["q"], "Y_hat": wp["W_fused"], "codes": wp["codes"],
                                                      "scales": wp["scales"]}, f"{w.name} weights",
                           cond=PT.condition_scale_weights(w.W[wrows], w.A, w.B))
    ref, T = O.gemm_rows(codes, a_sc, wc_h, w_sc, rows)
    PT.assert_gemm_parity(got, ref, T, f"{w.name} linear")
