"""batq_linear at decode sizes (S <= 16 tokens): the quantiser and the single-CTA GEMM with the
weights in M and the tokens in N, launched back to back with the GEMM prefetching its weights
while the quantiser runs.

Its output must be bit-identical to batq_quant_act followed by batq_gemm_mxfp4 (the same codes and
the same MMAs in the same order), the workspace must hold the quantiser's codes and MMA-layout scales
(padding included), and the result must match the oracle's fp64 GEMM of those codes within
1e-4 * sum |a||w|, with the codes themselves matching the oracle's activation path.
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


def _weights(w, real):
    if real:
        return GU.gpu_prepare(w)
    g = torch.Generator(device="cuda").manual_seed(w.seed + 17)
    wc, wsc = BQ.empty_act_buffers(w.M, w.N)
    wc.random_(0, 256, generator=g)
    wsc.random_(112, 140, generator=g)
    return wc, wsc


def _check(w, real_weights=False, out_dtype=torch.float32, X=None):
    X = GU.x_tensor(w) if X is None else X
    B, ratios = GU.params(w)
    wc, wsc = _weights(w, real_weights)
    ws = torch.full((BQ.batq_linear_workspace_size(w.S, w.N),), 0xAB, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.S, w.M), dtype=out_dtype, device="cuda")
    BQ.batq_linear(X, w.A, B, ratios, wc, wsc, w.M, ws, out)
    assert BQ.batq_device_error() == 0
    # the two-kernel path on the same inputs
    codes, scales = BQ.empty_act_buffers(w.S, w.N)
    scales.fill_(0xCD)
    BQ.batq_quant_act(X, w.A, B, ratios, codes, scales, BQ.BATQ_SCALES_MMA)
    out2 = GU.gpu_gemm(codes, scales, wc, wsc, w.S, w.M, w.N, out_dtype)
    assert torch.equal(out, out2), "fused decode linear differs from quantiser + GEMM"
    ncode = w.S * w.N // 2
    off = -(-ncode // 256) * 256
    assert torch.equal(ws[:ncode].view(w.S, w.N // 2), codes), "workspace codes"
    assert torch.equal(ws[off:off + scales.numel()], scales), "workspace scales (with padding)"
    # against the oracle: the activation codes, then the GEMM of the linear's own codes
    c_h = codes.cpu().numpy()
    a_sc = O.scales_from_mma_layout(scales.cpu().numpy(), w.S, w.k)
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    PT.assert_quant_parity(c_h, a_sc, act, f"decode linear {w.name}", cond=PT.condition_scale(w.x, w.A, w.B))
    ref, T = O.gemm(c_h, a_sc, wc.cpu().numpy(), O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k))
    got = out.float().cpu().numpy().astype(np.float64)
    if out_dtype == torch.bfloat16:
        assert np.all(np.abs(got - ref) <= 1e-4 * T + 2.0 ** -8 * np.abs(ref) + 1e-30)
    else:
        PT.assert_gemm_parity(got, ref, T, f"decode linear {w.name}")


@pytest.mark.parametrize("S", [1, 4, 16])
def test_decode_workload(S):
    """The decode workload (N = 4096, M = 24576 fused gate+up); real prepared weights at S = 16."""
    w = WL.decode(S, with_w=(S == 16))
    _check(w, real_weights=(S == 16))


@pytest.mark.parametrize("S,N,M,seed", [(3, 320, 272, 81), (16, 448, 144, 82), (7, 64, 16, 83), (9, 4096, 1040, 84)])
def test_ragged_shapes(S, N, M, seed):
    """Partial K stages (N = 320, 448, 64), a last weight tile of 16 rows, odd token counts."""
    _check(WL.custom(S, N, M, seed, with_w=False))


def test_fp32_activations_real_weights():
    """fp32 activations (the tiny workload) through prepared weights."""
    _check(WL.tiny(), real_weights=True)


def test_bf16_output_and_row_stride():
    w = WL.custom(5, 512, 384, 85, with_w=False)
    X = GU.x_tensor(w)
    Xw = torch.zeros((w.S, 768), dtype=X.dtype, device="cuda")
    Xw[:, :512] = X
    _check(w, out_dtype=torch.bfloat16, X=Xw[:, :512])
