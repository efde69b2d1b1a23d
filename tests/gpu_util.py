"""Device-side helpers for the GPU tests: move workloads to the GPU and call libbatq."""

from __future__ import annotations

import numpy as np
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from oracle import batq_oracle as O


def x_tensor(w):
    if w.x_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(w.x_bits).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w.x_bits)).cuda()


def params(w):
    B = torch.from_numpy(np.ascontiguousarray(w.B.reshape(-1))).cuda()
    ratios = torch.from_numpy(BQ.batq_clip_ratios(w.alpha_min, w.alpha_max)).cuda()
    return B, ratios


def gpu_quant(w, layout=BQ.BATQ_SCALES_MMA, y_debug=True, X=None):
    """Run batq_quant_act; returns (codes (S,N/2), scales linear (S,k), Y or None, raw scale buffer)."""
    X = x_tensor(w) if X is None else X
    B, ratios = params(w)
    codes, scales = BQ.empty_act_buffers(w.S, w.N, layout)
    scales.fill_(0xAB)  # poison: every byte the call owns must be written
    y = torch.empty((w.S, w.N), dtype=torch.float32, device="cuda") if y_debug else None
    BQ.batq_quant_act(X, w.A, B, ratios, codes, scales, layout, y_debug=y)
    assert BQ.batq_device_error() == 0
    raw = scales.cpu().numpy()
    if layout == BQ.BATQ_SCALES_MMA:
        lin = O.scales_from_mma_layout(raw, w.S, w.k)
    else:
        lin = raw.reshape(w.S, w.k)
    return codes.cpu().numpy(), lin, (y.cpu().numpy() if y is not None else None), raw


def gpu_prepare(w, layout=BQ.BATQ_SCALES_MMA):
    Wt = torch.from_numpy(np.ascontiguousarray(w.W)).cuda()
    codes, scales = BQ.empty_act_buffers(w.M, w.N, layout)
    scales.fill_(0xAB)
    ws = torch.empty(BQ.batq_prepare_workspace_size(w.N), dtype=torch.uint8, device="cuda")
    BQ.batq_prepare_weights(Wt, w.A, w.B, codes, scales, ws, layout)
    assert BQ.batq_device_error() == 0
    return codes, scales


def gpu_gemm(a_codes, a_scales_mma, w_codes, w_scales_mma, S, M, N, out_dtype=torch.float32):
    """Device tensors in, device out."""
    out = torch.empty((S, M), dtype=out_dtype, device="cuda")
    BQ.batq_gemm_mxfp4(a_codes, a_scales_mma, w_codes, w_scales_mma, S, M, N, out)
    assert BQ.batq_device_error() == 0
    return out


def to_dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()
