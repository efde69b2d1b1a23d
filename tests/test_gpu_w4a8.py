"""GPU parity of the W4A8 variant (MXFP8 E4M3 activations, MXFP4 weights in E4M3
containers, kind::mxf8f6f4 block-scaled GEMM) against the oracle."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
from tests import gpu_util as GU
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _quant8(w, layout=BQ.BATQ_SCALES_MMA, y_debug=True):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    codes, scales = BQ.empty_mxfp8_buffers(w.S, w.N, layout)
    scales.fill_(0xAB)
    y = torch.empty((w.S, w.N), dtype=torch.float32, device="cuda") if y_debug else None
    BQ.batq_quant_act_mxfp8(X, w.A, B, ratios, codes, scales, layout, y_debug=y)
    assert BQ.batq_device_error() == 0
    raw = scales.cpu().numpy()
    lin = O.scales_from_mma_layout(raw, w.S, w.k) if layout == BQ.BATQ_SCALES_MMA else raw.reshape(w.S, w.k)
    return codes.cpu().numpy(), lin, (y.cpu().numpy() if y is not None else None), raw


@pytest.mark.parametrize("maker,layout", [(WL.tiny, BQ.BATQ_SCALES_LINEAR), (WL.tiny, BQ.BATQ_SCALES_MMA),
                                          (lambda: WL.custom(200, 320, 16, 61), BQ.BATQ_SCALES_MMA),
                                          (lambda: WL.decode(4), BQ.BATQ_SCALES_MMA),
                                          (lambda: WL.q_proj(with_w=False), BQ.BATQ_SCALES_MMA)])
def test_quant_mxfp8_matches_oracle(maker, layout):
    w = maker()
    codes, lin, y, raw = _quant8(w, layout)
    ref = O.quant_act_mxfp8(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    bad, worst = PT.check_y(y, w.x, w.A, w.B, ref["Y"])
    assert bad == 0, worst
    PT.assert_quant_parity_e4m3(codes, lin, ref, w.x, w.A, w.B, "mxfp8")
    if layout == BQ.BATQ_SCALES_MMA:  # padding rows / columns hold the neutral byte
        pad = PT.to_mma_layout(lin, w.S, w.k)
        np.testing.assert_array_equal(raw, pad)


def test_quant_mxfp8_identity_transform_saturation_and_subnormals():
    """P = I, no clip: every code is fixed by the E4M3 rule, including blocks whose
    largest elements saturate at 448 and elements in the E4M3 subnormal range."""
    rng = np.random.default_rng(62)
    S, N = 32, 64
    k = N // 32
    X = np.empty((S, N), np.float32)
    for r in range(S):
        e = int(rng.integers(-20, 20))
        v = rng.choice(O.E4M3_MAGNITUDE, N) * rng.choice([-1.0, 1.0], N)
        v[0] = 500.0 if r % 2 else 448.0           # scaled amax in [256, 512): saturates on odd rows
        v[33] = 2.0 ** -9 * 3                       # subnormal E4M3 element
        X[r] = (v * 2.0 ** e).astype(np.float32)
    w = WL.Workload("grid8", 62, S, N, 16, "f32", X, X, np.eye(8, dtype=np.float32),
                    np.tile(np.eye(4, dtype=np.float32), (k, 1, 1)), np.full(k, 40, np.float32),
                    np.full(k, 40, np.float32), None)
    codes, lin, y, _ = _quant8(w, BQ.BATQ_SCALES_LINEAR)
    np.testing.assert_array_equal(y, X)
    ref = O.quant_act_mxfp8(X, w.A, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(lin, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])


def test_prepare_weights_w4a8_holds_the_mxfp4_values():
    w = WL.custom(48, 320, 272, 63)
    c4, s4 = GU.gpu_prepare(w)
    Wt = torch.from_numpy(np.ascontiguousarray(w.W)).cuda()
    c8 = torch.empty((w.M, w.N), dtype=torch.uint8, device="cuda")
    _, sb = BQ.batq_mxfp8_buffer_sizes(w.M, w.N)
    s8 = torch.empty(sb, dtype=torch.uint8, device="cuda")
    ws = torch.empty(BQ.batq_prepare_weights_w4a8_workspace_size(w.M, w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights_w4a8(Wt, w.A, w.B, c8, s8, ws)
    assert BQ.batq_device_error() == 0
    np.testing.assert_array_equal(s8.cpu().numpy(), s4.cpu().numpy())
    np.testing.assert_array_equal(c8.cpu().numpy(), O.e4m3_containers_from_e2m1(c4.cpu().numpy()))


def _rand_e4m3(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3A  # no NaN codes
    return c


@pytest.mark.parametrize("S,M,N", [(1, 256, 256), (16, 272, 320), (40, 128, 512), (100, 272, 320),
                                   (200, 256, 512), (129, 512, 4096), (1000, 1280, 512)])
def test_gemm_w4a8_random_operands(S, M, N):
    rng = np.random.default_rng(S * 7 + M + N)
    k = N // 32
    a8 = _rand_e4m3(rng, (S, N))
    w4 = rng.integers(0, 256, (M, N // 2)).astype(np.uint8)
    w8 = O.e4m3_containers_from_e2m1(w4)
    sa = rng.integers(118, 136, (S, k)).astype(np.uint8)
    sw = rng.integers(118, 136, (M, k)).astype(np.uint8)
    out = torch.empty((S, M), dtype=torch.float32, device="cuda")
    BQ.batq_gemm_w4a8(GU.to_dev_u8(a8), GU.to_dev_u8(PT.to_mma_layout(sa, S, k)), GU.to_dev_u8(w8),
                      GU.to_dev_u8(PT.to_mma_layout(sw, M, k)), S, M, N, out)
    assert BQ.batq_device_error() == 0
    rows = np.arange(S) if S <= 256 else np.sort(rng.choice(S, 96, replace=False))
    ref, T = O.gemm_w4a8(a8[rows], sa[rows], w8, sw)
    PT.assert_gemm_parity(out.cpu().numpy()[rows], ref, T, f"w4a8 {S}x{M}x{N}")


@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(200, 320, 272, 64), lambda: WL.decode(16),
                                   lambda: WL.q_proj()])
def test_linear_w4a8_matches_quant_then_gemm_and_oracle(maker):
    w = maker()
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    Wt = torch.from_numpy(np.ascontiguousarray(w.W)).cuda()
    c8 = torch.empty((w.M, w.N), dtype=torch.uint8, device="cuda")
    _, sb = BQ.batq_mxfp8_buffer_sizes(w.M, w.N)
    s8 = torch.empty(sb, dtype=torch.uint8, device="cuda")
    pws = torch.empty(BQ.batq_prepare_weights_w4a8_workspace_size(w.M, w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights_w4a8(Wt, w.A, w.B, c8, s8, pws)
    lws = torch.empty(BQ.batq_linear_w4a8_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_linear_w4a8(X, w.A, B, ratios, c8, s8, w.M, lws, out)
    assert BQ.batq_device_error() == 0
    # composition: identical to the two calls made separately
    codes, lin, _, raw = _quant8(w, BQ.BATQ_SCALES_MMA, y_debug=False)
    out2 = torch.empty_like(out)
    BQ.batq_gemm_w4a8(GU.to_dev_u8(codes), GU.to_dev_u8(raw), c8, s8, w.S, w.M, w.N, out2)
    assert torch.equal(out, out2)
    # oracle GEMM on the same operands, and the activations against the oracle's
    rows = np.arange(w.S) if w.S <= 256 else np.sort(np.random.default_rng(6).choice(w.S, 64, replace=False))
    wl = O.scales_from_mma_layout(s8.cpu().numpy(), w.M, w.k)
    ref, T = O.gemm_w4a8(codes[rows], lin[rows], c8.cpu().numpy(), wl)
    PT.assert_gemm_parity(out.cpu().numpy()[rows], ref, T, "linear w4a8")
    act = O.quant_act_mxfp8(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity_e4m3(codes[rows], lin[rows], act, w.x[rows], w.A, w.B, "linear w4a8 act")
    # W4A8 is closer to the unquantised product than W4A4 on the same weights
    if w.S <= 256:
        exact = w.x.astype(np.float64) @ w.W.astype(np.float64).T
        o4, _, _, _ = O.linear(w.x, w.A, w.B, w.alpha_min, w.alpha_max, w.W)
        e8 = np.linalg.norm(out.cpu().numpy() - exact)
        e4 = np.linalg.norm(o4 - exact)
        assert e8 < e4, (e8, e4)


def test_quant_mxfp8_tensor_core_transform_large():
    """A shape large enough for the tensor-core transform (sampled rows)."""
    w = WL.custom(4173, 8192, 16, 63, with_w=False)
    codes, lin, y, _ = _quant8(w)
    rows = np.unique(np.concatenate([np.random.default_rng(63).choice(w.S, 128, replace=False),
                                     np.arange(w.S - 20, w.S)]))
    ref = O.quant_act_mxfp8(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max)
    bad, worst = PT.check_y(y[rows], w.x[rows], w.A, w.B, ref["Y"])
    assert bad == 0, worst
    PT.assert_quant_parity_e4m3(codes[rows], lin[rows], ref, w.x[rows], w.A, w.B, "mxfp8 tc")
