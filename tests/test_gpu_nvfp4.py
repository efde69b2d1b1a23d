"""GPU parity of the NVFP4 output variant (E2M1 codes, E4M3 scale per 16 elements,
per-tensor encode scale; kind::mxf4nvf4 block-scaled GEMM) against the oracle."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu

NV_PAD = 0x38  # E4M3 1.0 in padding rows of the MMA layout


def _gs_tensor(gs):
    return None if gs is None else torch.tensor([gs], dtype=torch.float32, device="cuda")


def _lin_scales(raw, rows, N, layout):
    if layout == BQ.BATQ_SCALES_MMA:
        return O.scales_from_mma_layout(raw, rows, N // 16)
    return raw.reshape(rows, N // 16)


def _quant_nv(w, gs=None, layout=BQ.BATQ_SCALES_MMA, y_debug=True, X=None):
    X = GU.x_tensor(w) if X is None else X
    B, ratios = GU.params(w)
    codes, scales = BQ.empty_nvfp4_buffers(w.S, w.N, layout)
    scales.fill_(0xAB)  # poison: every byte the call owns must be written
    y = torch.empty((w.S, w.N), dtype=torch.float32, device="cuda") if y_debug else None
    BQ.batq_quant_act_nvfp4(X, w.A, B, ratios, codes, scales, gs=_gs_tensor(gs), layout=layout, y_debug=y)
    assert BQ.batq_device_error() == 0
    raw = scales.cpu().numpy()
    return codes.cpu().numpy(), _lin_scales(raw, w.S, w.N, layout), (y.cpu().numpy() if y is not None else None), raw


def _prepare_nv(w, layout=BQ.BATQ_SCALES_MMA):
    Wt = torch.from_numpy(np.ascontiguousarray(w.W)).cuda()
    codes, scales = BQ.empty_nvfp4_buffers(w.M, w.N, layout)
    scales.fill_(0xAB)
    gs = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(BQ.batq_prepare_weights_nvfp4_workspace_size(w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights_nvfp4(Wt, w.A, w.B, codes, scales, gs, ws, layout)
    assert BQ.batq_device_error() == 0
    return codes, scales, gs


# ------------------------------------------------------------ activations ----

@pytest.mark.parametrize("maker,layout,gs", [
    (WL.tiny, BQ.BATQ_SCALES_LINEAR, None),
    (WL.tiny, BQ.BATQ_SCALES_MMA, 37.5),
    (lambda: WL.custom(200, 320, 16, 71), BQ.BATQ_SCALES_MMA, None),
    (lambda: WL.custom(77, 192, 16, 72, x_dtype="f32"), BQ.BATQ_SCALES_LINEAR, 0.125),
    (lambda: WL.decode(4), BQ.BATQ_SCALES_MMA, 3.0),
    (lambda: WL.q_proj(with_w=False), BQ.BATQ_SCALES_MMA, 2.0),
])
def test_quant_nvfp4_matches_oracle(maker, layout, gs):
    w = maker()
    codes, lin, y, raw = _quant_nv(w, gs, layout)
    ref = O.quant_act_nvfp4(w.x, w.A, w.B, w.alpha_min, w.alpha_max, 1.0 if gs is None else gs)
    bad, worst = PT.check_y(y, w.x, w.A, w.B, ref["Y"])
    assert bad == 0, worst
    cond = PT.condition_scale(w.x, w.A, w.B)
    r = PT.assert_quant_parity_nvfp4(codes, lin, ref, cond, label="nvfp4")
    print("nvfp4 mismatches", r)
    # given the GPU's own transformed values, clip + scales + codes are bit-exact
    own = O.nvfp4_quantize(O.clip_blocks(y, O.clip_ratios(w.alpha_min), O.clip_ratios(w.alpha_max))[0],
                           1.0 if gs is None else gs)
    np.testing.assert_array_equal(codes, own[0])
    np.testing.assert_array_equal(lin, own[1])
    if layout == BQ.BATQ_SCALES_MMA:  # padding rows hold E4M3 1.0
        np.testing.assert_array_equal(raw, PT.to_mma_layout(lin, w.S, w.N // 16, pad=NV_PAD))


@pytest.mark.parametrize("gs", [1.0, 8.0, 3.0, 1e-3])
def test_quant_nvfp4_identity_transform_bit_exact(gs):
    """P = I, no clip: the transform is exact, so every scale and code (ties at the
    midpoints, subnormal, zero and saturated scales, non-finite blocks) is fixed by the
    format's fp32 steps and must match the oracle bit for bit."""
    rng = np.random.default_rng(81)
    S, N = 40, 128
    k = N // 32
    X = (rng.standard_normal((S, N)) * np.exp2(rng.integers(-8, 8, (S, 1)))).astype(np.float32)
    X[0, :16] = [6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, -0.25, 0, 1, 2, 3, 4, -6, 0.5]
    X[0, 16:32] = np.array([48, -24, 12, 4, 0, -8, 16, 32, 2, -2, 1, 0.5, 40, -44, 20, 28]) / 8
    X[1, :16] = 6 * 2.0 ** -9 / gs
    X[1, 16:32] = [-1e-30, 1e-30] + [0.0] * 14
    X[2, :16] = 3000.0 / gs
    X[3, 40] = np.inf
    X[4, 70] = np.nan
    X[5, :] = 0.0
    w = WL.Workload("nvgrid", 81, S, N, 16, "f32", X, X, np.eye(8, dtype=np.float32),
                    np.tile(np.eye(4, dtype=np.float32), (k, 1, 1)), np.full(k, 40, np.float32),
                    np.full(k, 40, np.float32), None)
    for layout in (BQ.BATQ_SCALES_LINEAR, BQ.BATQ_SCALES_MMA):
        codes, lin, y, _ = _quant_nv(w, gs, layout)
        ref = O.quant_act_nvfp4(X, w.A, w.B, w.alpha_min, w.alpha_max, gs)
        np.testing.assert_array_equal(lin, ref["scales"])
        np.testing.assert_array_equal(codes, ref["codes"])
    assert lin[3, 2] == 0x7F and lin[3, 3] == 0x7F and lin[4, 4] == 0x7F and (lin[5] == 0).all()


# ------------------------------------------------------------ weight side ----

@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(48, 320, 272, 73), WL.q_proj])
def test_prepare_weights_nvfp4_parity(maker):
    w = maker()
    codes, scales, gs = _prepare_nv(w)
    ref = O.prepare_weights_nvfp4(w.W, w.A, w.B)
    gs_gpu = float(gs.item())
    gs_rel = abs(gs_gpu - ref["gs"]) / ref["gs"]
    assert gs_rel <= 1e-5, (gs_gpu, ref["gs"])
    lin = O.scales_from_mma_layout(scales.cpu().numpy(), w.M, w.N // 16)
    cond = PT.condition_scale_weights(w.W, w.A, w.B)
    r = PT.assert_quant_parity_nvfp4(codes.cpu().numpy(), lin, {"q": ref["q"], "Y_hat": ref["W_fused"],
                                                                "codes": ref["codes"], "scales": ref["scales"],
                                                                "gs": ref["gs"]},
                                     cond, gs_rel=max(gs_rel, 1e-7), label="prepare nvfp4")
    print("prepare nvfp4 mismatches", r, "gs", gs_gpu, ref["gs"])
    # the tensor amax lands on the largest E4M3 scale
    assert lin.max() in (0x7E, 0x7D)


def test_prepare_weights_nvfp4_zero_weights():
    w = WL.tiny()
    w.W[:] = 0.0
    codes, scales, gs = _prepare_nv(w, BQ.BATQ_SCALES_LINEAR)
    assert float(gs.item()) == 1.0
    assert not codes.any().item() and not scales.any().item()


# ------------------------------------------------------------------- GEMM ----

def _random_nv_operands(S, M, N, seed):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, 256, (S, N // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (M, N // 2), dtype=np.uint8)
    sa = rng.integers(0x18, 0x58, (S, N // 16), dtype=np.uint8)   # E4M3 2^-4 .. 2^4
    sw = rng.integers(0x18, 0x58, (M, N // 16), dtype=np.uint8)
    sa[0, 0] = 0x00                                               # a zero scale
    return a, sa, w, sw


@pytest.mark.parametrize("S,M,N", [
    (16, 128, 256), (4, 64, 64), (1, 272, 320), (33, 160, 512), (65, 256, 512), (128, 256, 256),
    (200, 272, 320), (129, 256, 256), (300, 1024, 768), (1000, 1280, 512), (520, 4096, 256),
])
def test_gemm_nvfp4_random_operands(S, M, N):
    a, sa, w, sw = _random_nv_operands(S, M, N, S * 7 + M + N)
    out = torch.empty((S, M), dtype=torch.float32, device="cuda")
    ga, gw = 2.0, 0.75
    BQ.batq_gemm_nvfp4(GU.to_dev_u8(a), GU.to_dev_u8(PT.to_mma_layout(sa, S, N // 16, pad=NV_PAD)), _gs_tensor(ga),
                       GU.to_dev_u8(w), GU.to_dev_u8(PT.to_mma_layout(sw, M, N // 16, pad=NV_PAD)), _gs_tensor(gw),
                       S, M, N, out)
    assert BQ.batq_device_error() == 0
    ref, T = O.gemm_nvfp4(a, sa, w, sw, O.nvfp4_alpha(ga, gw))
    PT.assert_gemm_parity(out.cpu().numpy(), ref, T, f"gemm nvfp4 {S}x{M}x{N}")


@pytest.mark.parametrize("S", [16, 300])
def test_gemm_nvfp4_bf16_output_and_no_tensor_scales(S):
    M, N = 256, 512
    a, sa, w, sw = _random_nv_operands(S, M, N, 90 + S)
    out = torch.empty((S, M), dtype=torch.bfloat16, device="cuda")
    BQ.batq_gemm_nvfp4(GU.to_dev_u8(a), GU.to_dev_u8(PT.to_mma_layout(sa, S, N // 16, pad=NV_PAD)), None,
                       GU.to_dev_u8(w), GU.to_dev_u8(PT.to_mma_layout(sw, M, N // 16, pad=NV_PAD)), None,
                       S, M, N, out)
    assert BQ.batq_device_error() == 0
    ref, T = O.gemm_nvfp4(a, sa, w, sw, 1.0)
    got = out.float().cpu().numpy()
    # bf16 output: the fp32 result rounded once (relative 2^-9) on top of the GEMM tolerance
    assert (np.abs(got - ref) <= 1e-4 * T + 2.0 ** -8 * np.abs(ref)).all()


# ----------------------------------------------------------------- linear ----

def _linear_nv(w, gs_a=None, out_dtype=torch.float32):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc, wgs = _prepare_nv(w)
    ws = torch.empty(BQ.batq_linear_nvfp4_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=out_dtype, device="cuda")
    ags = _gs_tensor(gs_a)
    BQ.batq_linear_nvfp4(X, w.A, B, ratios, ags, wc, wsc, wgs, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    return out, wc, wsc, wgs, ags


@pytest.mark.parametrize("maker,gs_a", [(WL.tiny, None), (lambda: WL.custom(200, 320, 272, 74), 4.0),
                                        (lambda: WL.q_proj(), 2.0), (lambda: WL.decode(16), None)])
def test_linear_nvfp4_matches_quant_then_gemm_and_oracle(maker, gs_a):
    w = maker()
    out, wc, wsc, wgs, ags = _linear_nv(w, gs_a)
    codes, lin, _, raw = _quant_nv(w, gs_a, BQ.BATQ_SCALES_MMA, y_debug=False)
    out2 = torch.empty_like(out)
    BQ.batq_gemm_nvfp4(GU.to_dev_u8(codes), GU.to_dev_u8(raw), ags, wc, wsc, wgs, w.S, w.M, w.N, out2)
    assert BQ.batq_device_error() == 0
    assert torch.equal(out, out2)
    rows = np.arange(w.S) if w.S <= 256 else np.sort(np.random.default_rng(6).choice(w.S, 64, replace=False))
    wl = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.N // 16)
    alpha = O.nvfp4_alpha(1.0 if gs_a is None else gs_a, float(wgs.item()))
    ref, T = O.gemm_nvfp4(codes[rows], lin[rows], wc.cpu().numpy(), wl, alpha)
    PT.assert_gemm_parity(out.cpu().numpy()[rows], ref, T, "linear nvfp4")
    act = O.quant_act_nvfp4(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max, 1.0 if gs_a is None else gs_a)
    PT.assert_quant_parity_nvfp4(codes[rows], lin[rows], act, PT.condition_scale(w.x[rows], w.A, w.B),
                                 label="linear nvfp4 act")


def test_linear_nvfp4_error_matches_oracle_and_beats_mxfp4():
    """Distance of the NVFP4 output from the unquantised x W^T equals the oracle's, and is
    below that of the MXFP4 linear on the same inputs."""
    w = WL.custom(64, 512, 256, 75)
    out, _, _, wgs, _ = _linear_nv(w)
    exact = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    act = O.quant_act_nvfp4(w.x, w.A, w.B, w.alpha_min, w.alpha_max, 1.0)
    wp = O.prepare_weights_nvfp4(w.W, w.A, w.B)
    ref, _ = O.gemm_nvfp4(act["codes"], act["scales"], wp["codes"], wp["scales"], O.nvfp4_alpha(1.0, wp["gs"]))
    rel_gpu = np.linalg.norm(out.cpu().numpy() - exact) / np.linalg.norm(exact)
    rel_ref = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert abs(rel_gpu - rel_ref) < 1e-3 * rel_ref + 1e-6, (rel_gpu, rel_ref)
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc4, ws4 = GU.gpu_prepare(w)
    ws = torch.empty(BQ.batq_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out4 = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_linear(X, w.A, B, ratios, wc4, ws4, w.M, ws, out4)
    rel_mx = np.linalg.norm(out4.cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel_gpu < rel_mx, (rel_gpu, rel_mx)


def test_quant_nvfp4_tensor_core_transform_large():
    """A shape large enough for the tensor-core transform (sampled rows, gs from the device)."""
    w = WL.custom(4173, 8192, 16, 78, with_w=False)
    codes, lin, y, raw = _quant_nv(w, 5.0)
    rows = np.unique(np.concatenate([np.random.default_rng(78).choice(w.S, 128, replace=False),
                                     np.arange(w.S - 20, w.S)]))
    ref = O.quant_act_nvfp4(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max, 5.0)
    bad, worst = PT.check_y(y[rows], w.x[rows], w.A, w.B, ref["Y"])
    assert bad == 0, worst
    PT.assert_quant_parity_nvfp4(codes[rows], lin[rows], ref, PT.condition_scale(w.x[rows], w.A, w.B),
                                 label="nvfp4 tc")
    own = O.nvfp4_quantize(O.clip_blocks(y[rows], O.clip_ratios(w.alpha_min), O.clip_ratios(w.alpha_max))[0], 5.0)
    np.testing.assert_array_equal(codes[rows], own[0])
    np.testing.assert_array_equal(lin[rows], own[1])


def test_prepare_weights_nvfp4_tensor_core_measuring_pass():
    """bf16 weights large enough for the tensor-core transform: both passes (amax, then codes)."""
    w = WL.custom(16, 4096, 8192, 79)
    Wb = torch.from_numpy(np.ascontiguousarray(w.W)).cuda().to(torch.bfloat16)
    Wv = Wb.float().cpu().numpy()
    codes, scales = BQ.empty_nvfp4_buffers(w.M, w.N)
    gs = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(BQ.batq_prepare_weights_nvfp4_workspace_size(w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights_nvfp4(Wb, w.A, w.B, codes, scales, gs, ws)
    assert BQ.batq_device_error() == 0
    rows = np.sort(np.random.default_rng(79).choice(w.M, 96, replace=False))
    ref_all = O.prepare_weights_nvfp4(Wv, w.A, w.B)
    gs_rel = abs(float(gs.item()) - ref_all["gs"]) / ref_all["gs"]
    assert gs_rel <= 1e-5
    lin = O.scales_from_mma_layout(scales.cpu().numpy(), w.M, w.N // 16)[rows]
    ref = {"q": ref_all["q"][rows], "Y_hat": ref_all["W_fused"][rows], "codes": ref_all["codes"][rows],
           "scales": ref_all["scales"][rows], "gs": ref_all["gs"]}
    PT.assert_quant_parity_nvfp4(codes.cpu().numpy()[rows], lin, ref, PT.condition_scale_weights(Wv[rows], w.A, w.B),
                                 gs_rel=max(gs_rel, 1e-7), label="prepare nvfp4 tc")
