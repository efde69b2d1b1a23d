"""GPU parity of the fused RMSNorm -> transform -> clip -> MXFP4 path against the oracle.

The norm ahead of every linear, z = x / sqrt(mean x^2 + eps) * gamma, is fused into the online
activation path (ARCQuant reading notes, section "融合核函数设计"; BATQuant thelatestinai.com page,
Figure 3 caption: the activation transform runs online before each linear).  z never leaves the
library's kernels; the oracle computes it in fp64 (``rmsnorm_quant_act``).  Tolerances are those
of batq_quant_act with the condition scale taken on z.
"""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _run(w, gamma, layout=BQ.BATQ_SCALES_MMA, eps=EPS, X=None):
    X = GU.x_tensor(w) if X is None else X
    B, ratios = GU.params(w)
    g = torch.from_numpy(gamma).cuda()
    codes, scales = BQ.empty_act_buffers(w.S, w.N, layout)
    scales.fill_(0xAB)
    y = torch.empty((w.S, w.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(BQ.batq_rmsnorm_workspace_size(w.S), dtype=torch.uint8, device="cuda")
    BQ.batq_rmsnorm_quant_act(X, g, eps, w.A, B, ratios, codes, scales, ws, layout, y_debug=y)
    assert BQ.batq_device_error() == 0
    raw = scales.cpu().numpy()
    lin = O.scales_from_mma_layout(raw, w.S, w.k) if layout == BQ.BATQ_SCALES_MMA else raw.reshape(w.S, w.k)
    return codes.cpu().numpy(), lin, y.cpu().numpy(), raw


def _check(w, gamma, codes, scales, y, rows=None, label="", eps=EPS):
    x = w.x if rows is None else w.x[rows]
    if rows is not None:
        codes, scales, y = codes[rows], scales[rows], y[rows]
    ref = O.rmsnorm_quant_act(x, gamma, eps, w.A, w.B, w.alpha_min, w.alpha_max)
    nbad, worst = PT.check_y(y, ref["Z"], w.A, w.B, ref["Y"])
    assert nbad == 0, f"{label}: {nbad} transformed values outside 1e-5 (worst {worst})"
    strict = O.encode_from_transformed(y, O.clip_ratios(w.alpha_min), O.clip_ratios(w.alpha_max))
    np.testing.assert_array_equal(scales, strict["scales"], err_msg=label + " scales (strict)")
    np.testing.assert_array_equal(codes, strict["codes"], err_msg=label + " codes (strict)")
    return PT.assert_quant_parity(codes, scales, ref, label, cond=PT.condition_scale(ref["Z"], w.A, w.B))


@pytest.mark.parametrize("layout", [BQ.BATQ_SCALES_LINEAR, BQ.BATQ_SCALES_MMA])
def test_tiny_fp32(layout):
    w = WL.tiny(with_w=False)
    gamma = WL.rmsnorm_gamma(w.N, 1)
    codes, scales, y, raw = _run(w, gamma, layout)
    _check(w, gamma, codes, scales, y, label="tiny rmsnorm")


@pytest.mark.parametrize("S,N,seed", [(1, 64, 5), (200, 320, 7), (129, 448, 8)])
def test_ragged_shapes_bf16(S, N, seed):
    w = WL.custom(S, N, 16, seed, with_w=False)
    gamma = WL.rmsnorm_gamma(N, seed)
    codes, scales, y, _ = _run(w, gamma)
    _check(w, gamma, codes, scales, y, label=f"rmsnorm {S}x{N}")


def test_q_proj_full():
    """q_proj (S=2048, N=4096): the CUDA-core transform with gamma staged per tile."""
    w = WL.q_proj(with_w=False)
    gamma = WL.rmsnorm_gamma(w.N, 2)
    codes, scales, y, _ = _run(w, gamma)
    _check(w, gamma, codes, scales, y, label="rmsnorm q_proj")


@pytest.mark.parametrize("S", [1, 16])
def test_decode(S):
    w = WL.decode(S, with_w=False)
    gamma = WL.rmsnorm_gamma(w.N, 4)
    codes, scales, y, _ = _run(w, gamma)
    _check(w, gamma, codes, scales, y, label=f"rmsnorm decode{S}")


@pytest.mark.parametrize("j", [0, 6])
def test_layer_tensor_core_sampled_rows(j):
    """The S = 8192 layer shapes take the tensor-core transform (gamma folded into P_i, 1 / rms
    applied in the encoder); sampled rows, the last rows included."""
    w = WL.layer_linear(j, with_w=False)
    gamma = WL.rmsnorm_gamma(w.N, 10 + j)
    codes, scales, y, _ = _run(w, gamma)
    rows = np.unique(np.concatenate([np.random.default_rng(j).choice(w.S, 256, replace=False),
                                     np.arange(w.S - 8, w.S)]))
    _check(w, gamma, codes, scales, y, rows=rows, label=f"rmsnorm layer{j}")


def test_zero_rows_and_scale_invariance():
    """A zero token with eps > 0 gives all-zero blocks (scale byte 0, zero codes); with eps = 0 a
    token and 8 times that token give the same codes and scales (the norm removes the factor)."""
    w = WL.custom(40, 256, 16, 31, x_dtype="f32", with_w=False)
    gamma = WL.rmsnorm_gamma(w.N, 31)
    X = w.x.copy()
    X[3] = 0.0
    X[7] = 8.0 * X[6]
    w.x, w.x_bits = X, X
    codes, scales, y, _ = _run(w, gamma, BQ.BATQ_SCALES_LINEAR)
    assert (scales[3] == 0).all() and not codes[3].any()
    _check(w, gamma, codes, scales, y, label="rmsnorm zero row")
    X[3] = 1.0
    codes0, scales0, _, _ = _run(w, gamma, BQ.BATQ_SCALES_LINEAR, eps=0.0)
    np.testing.assert_array_equal(codes0[7], codes0[6])
    np.testing.assert_array_equal(scales0[7], scales0[6])


def _linear(w, gamma):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc = GU.gpu_prepare(w)
    g = torch.from_numpy(gamma).cuda()
    ws = torch.empty(BQ.batq_rmsnorm_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_rmsnorm_linear(X, g, EPS, w.A, B, ratios, wc, wsc, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    return out, wc, wsc, ws


@pytest.mark.parametrize("maker", [lambda: WL.custom(200, 320, 272, 51), lambda: WL.q_proj(), lambda: WL.decode(16)],
                         ids=["ragged", "q_proj", "decode16"])
def test_rmsnorm_linear_end_to_end(maker):
    """batq_rmsnorm_linear: its activation codes against the oracle's fused norm + quantiser, and its
    output against the oracle's fp64 GEMM of the same codes (sampled rows for the large case)."""
    w = maker()
    gamma = WL.rmsnorm_gamma(w.N, w.seed)
    out, wc, wsc, ws = _linear(w, gamma)
    ws_h = ws.cpu().numpy()
    ncode = w.S * w.N // 2
    codes = ws_h[:ncode].reshape(w.S, w.N // 2)
    off = -(-ncode // 256) * 256
    a_sc = O.scales_from_mma_layout(ws_h[off:off + O.mma_layout_bytes(w.S, w.k)], w.S, w.k)
    rows = np.arange(w.S) if w.S <= 256 else np.sort(np.random.default_rng(6).choice(w.S, 64, replace=False))
    ref = O.rmsnorm_quant_act(w.x[rows], gamma, EPS, w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity(codes[rows], a_sc[rows], ref, "rmsnorm linear act",
                           cond=PT.condition_scale(ref["Z"], w.A, w.B))
    wl = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    g_ref, T = O.gemm_rows(codes, a_sc, wc.cpu().numpy(), wl, rows)
    PT.assert_gemm_parity(out.cpu().numpy()[rows], g_ref, T, "rmsnorm linear")
