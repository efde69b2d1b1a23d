"""batq_linear_no_alloc against batq_linear.

Some callers of the W4A4 linear cannot call cudaMalloc: a plugin that is handed
tensors but no allocator, a process whose device memory another allocator has
reserved up front, or a path where the device synchronisation that cudaMalloc /
cudaFree may cause is not allowed.  batq_linear_no_alloc serves them by taking
its scratch for the quantised activations from a fixed array inside the
library instead of a caller workspace.  These tests call it through the C-ABI
and check that its output matches batq_linear's (which uses a caller-allocated
workspace) within the GEMM tolerance the other tests use, on two calls in a
row with different inputs.  The refusal of problems too large for the array
happens before any CUDA call and is tested without a GPU (tests/test_abi.py).
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


def _both(w):
    """Output of batq_linear_no_alloc and of batq_linear (caller workspace) on the same inputs."""
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    wc, wsc = GU.gpu_prepare(w)
    out_na = torch.empty((w.S, w.M), dtype=torch.float32, device="cuda")
    BQ.batq_linear_no_alloc(X, w.A, B, ratios, wc, wsc, w.M, out_na)
    ws = torch.empty(BQ.batq_linear_workspace_size(w.S, w.N), dtype=torch.uint8, device="cuda")
    out_ws = torch.empty_like(out_na)
    BQ.batq_linear(X, w.A, B, ratios, wc, wsc, w.M, ws, out_ws)
    assert BQ.batq_device_error() == 0
    # tolerance scale sum |a||w| from the activation codes batq_linear left in its workspace
    ws_h = ws.cpu().numpy()
    ncode = w.S * w.N // 2
    codes = ws_h[:ncode].reshape(w.S, w.N // 2)
    off = -(-ncode // 256) * 256
    a_sc = O.scales_from_mma_layout(ws_h[off:off + O.mma_layout_bytes(w.S, w.k)], w.S, w.k)
    w_sc = O.scales_from_mma_layout(wsc.cpu().numpy(), w.M, w.k)
    rows = np.arange(w.S) if w.S <= 256 else np.sort(np.random.default_rng(3).choice(w.S, 64, replace=False))
    _, T = O.gemm_rows(codes, a_sc, wc.cpu().numpy(), w_sc, rows)
    return out_na.cpu().numpy(), out_ws.cpu().numpy(), rows, T


def test_no_alloc_matches_workspace_linear_on_two_calls_in_a_row():
    # first call: a prefill-sized problem; second: a different, smaller one, so a
    # stale scratch from the first call would show up in the second.
    for w in (WL.custom(1024, 4096, 512, 61), WL.custom(40, 320, 272, 62)):
        na, ref, rows, T = _both(w)
        err = np.abs(na[rows].astype(np.float64) - ref[rows].astype(np.float64))
        assert np.all(err <= 1e-4 * T), f"{w.name}: worst {np.max(err / np.maximum(T, 1e-300))}"
        assert np.array_equal(na, ref), f"{w.name}: outputs differ"

