"""GPU parity of the naive Kronecker decomposition (one 8x8 A_i per block, P_i = B_i (x) A_i) against
the oracle: activations (both quantiser kernels), weight preparation and the linear."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu


def _a_dev(w):
    return torch.from_numpy(np.ascontiguousarray(w.A.reshape(-1), dtype=np.float32)).cuda()


def _quant_kron(w, layout=BQ.BATQ_SCALES_MMA):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    codes, scales = BQ.empty_act_buffers(w.S, w.N, layout)
    scales.fill_(0xAB)
    y = torch.empty((w.S, w.N), dtype=torch.float32, device="cuda")
    BQ.batq_quant_act_kron(X, _a_dev(w), B, ratios, codes, scales, layout, y_debug=y)
    assert BQ.batq_device_error() == 0
    raw = scales.cpu().numpy()
    lin = O.scales_from_mma_layout(raw, w.S, w.k) if layout == BQ.BATQ_SCALES_MMA else raw.reshape(w.S, w.k)
    return codes.cpu().numpy(), lin, y.cpu().numpy()


def _check(w, codes, lin, y, rows, label):
    x = w.x[rows]
    ref = O.quant_act(x, w.A, w.B, w.alpha_min, w.alpha_max)
    bad, worst = PT.check_y(y[rows], x, w.A, w.B, ref["Y"])
    assert bad == 0, f"{label}: {worst}"
    r = O.clip_ratios(w.alpha_min), O.clip_ratios(w.alpha_max)
    own = O.encode_from_transformed(y[rows], r[0], r[1])
    np.testing.assert_array_equal(codes[rows], own["codes"])
    np.testing.assert_array_equal(lin[rows], own["scales"])
    PT.assert_quant_parity(codes[rows], lin[rows], ref, label, cond=PT.condition_scale(x, w.A, w.B))


@pytest.mark.parametrize("maker,layout", [
    (WL.tiny, BQ.BATQ_SCALES_LINEAR),                                   # fp32, CUDA-core kernel
    (lambda: WL.custom(200, 320, 16, 95, with_w=False), BQ.BATQ_SCALES_MMA),   # bf16, CUDA-core kernel
    (lambda: WL.custom(8192, 4096, 16, 96, with_w=False), BQ.BATQ_SCALES_MMA),  # bf16, tensor-core kernel
])
def test_quant_act_kron_matches_oracle(maker, layout):
    w = WL.with_naive_kronecker(maker(), 7)
    codes, lin, y = _quant_kron(w, layout)
    rows = np.arange(w.S) if w.S <= 256 else np.unique(np.concatenate(
        [np.random.default_rng(95).choice(w.S, 192, replace=False), np.arange(w.S - 16, w.S)]))
    _check(w, codes, lin, y, rows, "kron")


@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(8192, 4096, 16, 97, with_w=False)])
def test_equal_factors_reproduce_the_gpk_calls(maker):
    """A_i = A for every block: the naive call returns the GPK call's bytes exactly."""
    w = maker()
    wk = WL.with_naive_kronecker(w, 0)
    wk.A = np.repeat(w.A[None], w.k, axis=0).astype(np.float32)
    codes_k, lin_k, _ = _quant_kron(wk)
    codes, lin, _, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_MMA, y_debug=False)
    np.testing.assert_array_equal(codes_k, codes)
    np.testing.assert_array_equal(lin_k, lin)


def _prepare_kron(w):
    Wt = torch.from_numpy(np.ascontiguousarray(w.W)).cuda()
    codes, scales = BQ.empty_act_buffers(w.M, w.N)
    ws = torch.empty(BQ.batq_prepare_weights_kron_workspace_size(w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights_kron(Wt, w.A, w.B, codes, scales, ws)
    assert BQ.batq_device_error() == 0
    return codes, scales


@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(48, 320, 272, 98)])
def test_prepare_weights_kron_parity(maker):
    w = WL.with_naive_kronecker(maker(), 8)
    codes, scales = _prepare_kron(w)
    ref = O.prepare_weights(w.W, w.A, w.B)
    lin = O.scales_from_mma_layout(scales.cpu().numpy(), w.M, w.k)
    PT.assert_quant_parity(codes.cpu().numpy(), lin, {"q": ref["q"], "Y_hat": ref["W_fused"], "codes": ref["codes"],
                                                      "scales": ref["scales"]}, "prepare kron",
                           cond=PT.condition_scale_weights(w.W, w.A, w.B))


def test_linear_kron_matches_oracle():
    w = WL.with_naive_kronecker(WL.custom(200, 320, 272, 99), 9)
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc = _prepare_kron(w)
    ws = torch.empty(BQ.batq_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_linear_kron(X, _a_dev(w), B, ratios, wc, wsc, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    codes, lin, _ = _quant_kron(w)
    wl = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    ref, T = O.gemm(codes, lin, wc.cpu().numpy(), wl)
    PT.assert_gemm_parity(out.cpu().numpy(), ref, T, "linear kron")
    exact = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    oref, _, _, _ = O.linear(w.x, w.A, w.B, w.alpha_min, w.alpha_max, w.W)
    rel_gpu = np.linalg.norm(out.cpu().numpy() - exact) / np.linalg.norm(exact)
    rel_ref = np.linalg.norm(oref - exact) / np.linalg.norm(exact)
    assert abs(rel_gpu - rel_ref) < 2e-3 * rel_ref + 1e-6, (rel_gpu, rel_ref)
