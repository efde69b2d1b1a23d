"""GPU parity of batq_quant_kv_cache (BAT on the KV cache, KV4 = MXFP4 and KV8 = MXFP8 rows written
into a paged cache at the slot mapping's rows) against the oracle."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu

POISON = 0xAB


def _run(w, slots, num_slots, fmt):
    X = GU.x_tensor(w)
    B, ratios = GU.params(w)
    width = w.N // 2 if fmt == BQ.BATQ_KV_MXFP4 else w.N
    cc = torch.full((num_slots, width), POISON, dtype=torch.uint8, device="cuda")
    cs = torch.full((num_slots, w.N // 32), POISON, dtype=torch.uint8, device="cuda")
    sm = torch.from_numpy(np.ascontiguousarray(slots, dtype=np.int32)).cuda()
    BQ.batq_quant_kv_cache(X, w.A, B, ratios, sm, cc, cs, fmt)
    assert BQ.batq_device_error() == 0
    return cc.cpu().numpy(), cs.cpu().numpy()


def _check_rows(w, rows, slots, cc, cs, fmt, label):
    x = w.x[rows]
    cond = PT.condition_scale(x, w.A, w.B)
    if fmt == BQ.BATQ_KV_MXFP4:
        ref = O.quant_act(x, w.A, w.B, w.alpha_min, w.alpha_max)
        PT.assert_quant_parity(cc[slots[rows]], cs[slots[rows]], ref, label, cond=cond)
    else:
        ref = O.quant_act_mxfp8(x, w.A, w.B, w.alpha_min, w.alpha_max)
        PT.assert_quant_parity_e4m3(cc[slots[rows]], cs[slots[rows]], ref, x, w.A, w.B, label)


@pytest.mark.parametrize("fmt", [BQ.BATQ_KV_MXFP4, BQ.BATQ_KV_MXFP8])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_kv_cache_write_matches_oracle(fmt, x_dtype):
    """8 KV heads x 128 (N = 1024), 37 new tokens into a 100-slot cache; two padding tokens
    (slot -1) and one slot past the cache are skipped; every other cache byte stays untouched."""
    w = WL.custom(37, 1024, 16, 91, x_dtype=x_dtype, with_w=False)
    rng = np.random.default_rng(91)
    num_slots = 100
    slots = rng.permutation(num_slots)[:37].astype(np.int64)
    slots[[4, 20]] = -1
    slots[30] = num_slots + 3
    cc, cs = _run(w, slots, num_slots, fmt)
    valid = np.flatnonzero((slots >= 0) & (slots < num_slots))
    _check_rows(w, valid, slots, cc, cs, fmt, "kv")
    untouched = np.setdiff1d(np.arange(num_slots), slots[valid])
    assert (cc[untouched] == POISON).all() and (cs[untouched] == POISON).all()
    # the oracle's whole-cache result agrees on every written byte's position
    width = cc.shape[1]
    oc, os_, _ = O.quant_kv_cache(w.x, w.A, w.B, w.alpha_min, w.alpha_max, slots,
                                  np.full((num_slots, width), POISON, np.uint8),
                                  np.full((num_slots, w.N // 32), POISON, np.uint8),
                                  "mxfp4" if fmt == BQ.BATQ_KV_MXFP4 else "mxfp8")
    assert ((oc == POISON) == (cc == POISON)).mean() > 0.99


def test_kv_cache_write_tensor_core_path():
    """A prefill-sized K write (S = 20000, N = 4096: enough tiles for the tensor-core transform),
    reversed slot order into a larger cache; sampled tokens against the oracle."""
    w = WL.custom(20000, 4096, 16, 92, with_w=False)
    num_slots = 24000
    slots = (num_slots - 1 - np.arange(w.S)).astype(np.int64)  # reversed: token r -> slot 23999 - r
    assert len(np.unique(slots)) == w.S and slots.min() >= 0
    cc, cs = _run(w, slots, num_slots, BQ.BATQ_KV_MXFP4)
    rows = np.unique(np.concatenate([np.random.default_rng(92).choice(w.S, 160, replace=False),
                                     np.arange(w.S - 16, w.S)]))
    _check_rows(w, rows, slots, cc, cs, BQ.BATQ_KV_MXFP4, "kv tc")
    untouched = np.setdiff1d(np.arange(num_slots), slots)
    assert (cc[untouched] == POISON).all() and (cs[untouched] == POISON).all()
