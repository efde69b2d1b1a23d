"""GPU parity of batq_quant_act against the CPU oracle (through the C-ABI)."""

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
from oracle import batq_oracle as O
import gpu_util as GU
import parity as PT

pytestmark = pytest.mark.gpu


def _oracle(w, rows=None):
    x = w.x if rows is None else w.x[rows]
    return O.quant_act(x, w.A, w.B, w.alpha_min, w.alpha_max)


def _check_all(w, codes, scales, y, rows=None, label="", literal_limit=PT.LITERAL_LIMIT):
    ref = _oracle(w, rows)
    if rows is not None:
        codes, scales = codes[rows], scales[rows]
        y = y[rows] if y is not None else None
    x = w.x if rows is None else w.x[rows]
    if y is not None:
        nbad, worst = PT.check_y(y, x, w.A, w.B, ref["Y"])
        assert nbad == 0, f"{label}: {nbad} transformed values outside 1e-5 (worst {worst})"
        # Given the GPU's own Y, clip + scale + encode must be bit-exact.
        r = O.clip_ratios(w.alpha_min), O.clip_ratios(w.alpha_max)
        strict = O.encode_from_transformed(y, r[0], r[1])
        np.testing.assert_array_equal(scales, strict["scales"], err_msg=label + " scales (strict)")
        np.testing.assert_array_equal(codes, strict["codes"], err_msg=label + " codes (strict)")
    return PT.assert_quant_parity(codes, scales, ref, label, cond=PT.condition_scale(x, w.A, w.B),
                                  literal_limit=literal_limit)


@pytest.mark.parametrize("layout", [BQ.BATQ_SCALES_LINEAR, BQ.BATQ_SCALES_MMA])
def test_tiny_fp32(layout):
    w = WL.tiny(with_w=False)
    codes, scales, y, raw = GU.gpu_quant(w, layout)
    _check_all(w, codes, scales, y, label="tiny")
    if layout == BQ.BATQ_SCALES_MMA:
        mask = np.ones(raw.size, bool)
        r, c = np.meshgrid(np.arange(w.S), np.arange(w.k), indexing="ij")
        mask[O.mma_scale_offset(r, c, w.k)] = False
        assert np.all(raw[mask] == 0x7F), "padding scales must be 0x7F"


@pytest.mark.parametrize("S,N,seed", [(1, 64, 5), (33, 64, 6), (200, 320, 7), (129, 448, 8), (64, 4096, 9)])
def test_ragged_shapes_bf16(S, N, seed):
    w = WL.custom(S, N, 16, seed, with_w=False)
    codes, scales, y, raw = GU.gpu_quant(w, BQ.BATQ_SCALES_MMA)
    _check_all(w, codes, scales, y, label=f"{S}x{N}")
    codes2, scales2, _, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR, y_debug=False)
    np.testing.assert_array_equal(codes2, codes)
    np.testing.assert_array_equal(scales2, scales)


def test_padded_row_stride():
    w = WL.custom(40, 256, 16, 11, with_w=False)
    X = GU.x_tensor(w)
    Xw = torch.zeros((w.S, 384), dtype=X.dtype, device="cuda")
    Xw[:, :256] = X
    codes, scales, y, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_MMA, X=Xw[:, :256])
    _check_all(w, codes, scales, y, label="ldx=384")


def test_q_proj_full():
    w = WL.q_proj(with_w=False)
    codes, scales, y, _ = GU.gpu_quant(w)
    r = _check_all(w, codes, scales, y, label="q_proj")
    print("q_proj boundary mismatches", r)


def test_down_proj_full():
    w = WL.down_proj(with_w=False)
    codes, scales, y, _ = GU.gpu_quant(w)
    r = _check_all(w, codes, scales, y, label="down_proj")
    print("down_proj boundary mismatches", r)


@pytest.mark.parametrize("S", [1, 4, 16])
def test_decode(S):
    w = WL.decode(S, with_w=False)
    codes, scales, y, _ = GU.gpu_quant(w)
    _check_all(w, codes, scales, y, label=f"decode{S}")


@pytest.mark.parametrize("j", range(7))
def test_layer_linear_sampled_rows(j):
    """Each linear of the S = 8192 layer: codes and scales on 384 sampled rows against the oracle,
    the transformed values on those rows within the Y tolerance, and the GPU's own Y re-encoded
    by the oracle bit for bit."""
    w = WL.layer_linear(j, with_w=False)
    codes, scales, y, _ = GU.gpu_quant(w, y_debug=True)
    rows = np.sort(np.random.default_rng(100 + j).choice(w.S, 384, replace=False))
    _check_all(w, codes, scales, y, rows=rows, label=f"layer{j}")


def test_encoder_grid_identity_transform_bit_exact():
    """P = I, no clip: Y equals X exactly, so every code and scale is fixed by the
    E2M1 round-to-nearest-even rule; covers every midpoint, its neighbours,
    negative values rounding to -0, saturation and a range of exponents."""
    vals = []
    for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
        vals += [m, np.nextafter(np.float32(m), np.float32(0)), np.nextafter(np.float32(m), np.float32(9))]
    vals += [0.0, 0.1, 0.2, 0.3, 0.5, 1.0, 5.9, 6.0, 7.9]
    vals = np.array(vals, np.float32)
    rows = []
    for e in range(-12, 13, 3):
        for sign in (1, -1):
            blk = np.zeros(32, np.float32)
            blk[0] = 6.0 * 2.0 ** e  # sets the shared exponent to e
            blk[1:1 + len(vals)] = sign * vals * np.float32(2.0 ** e)
            blk[31] = -0.05 * 2.0 ** e  # rounds to -0
            rows.append(np.concatenate([blk, blk[::-1]]))
    X = np.stack(rows).astype(np.float32)
    S, N = X.shape[0], 64
    k = N // 32
    w = WL.Workload("grid", 0, S, N, 16, "f32", X, X, np.eye(8, dtype=np.float32),
                    np.tile(np.eye(4, dtype=np.float32), (k, 1, 1)), np.full(k, 40, np.float32),
                    np.full(k, 40, np.float32), None)
    codes, scales, y, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR)
    np.testing.assert_array_equal(y, X)
    ref = O.quant_act(X, w.A, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(scales, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])


def test_zero_and_nonfinite_blocks():
    w = WL.custom(8, 128, 16, 12, x_dtype="f32", with_w=False)
    X = w.x.copy()
    X[0, 0:32] = 0.0
    X[1, 32 + 3] = np.inf
    X[2, 64 + 7] = np.nan
    X[3, 96:128] = -0.0
    w.x, w.x_bits = X, X
    codes, scales, y, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR)
    assert scales[0, 0] == 0 and not codes[0, 0:16].any()
    assert scales[1, 1] == 0xFF and not codes[1, 16:32].any()
    assert scales[2, 2] == 0xFF and not codes[2, 32:48].any()
    assert scales[3, 3] == 0 and not codes[3, 48:64].any()
    ref = O.quant_act(X, w.A, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(scales, ref["scales"])
    PT.assert_quant_parity(codes, scales, ref, "zero/nonfinite")


def test_clip_lo_above_hi_gives_constant_block():
    """Same-sign blocks with r_min > r_max: lo = r_min*mn exceeds hi = r_max*mx, so
    min(max(y, lo), hi) is hi everywhere (the clamp order the oracle fixes)."""
    rng = np.random.default_rng(21)
    S, N = 40, 128
    k = N // 32
    X = (5.0 + 0.5 * rng.standard_normal((S, N))).astype(np.float32)
    X[S // 2:] *= -1.0  # negative blocks too
    w = WL.Workload("lo_gt_hi", 21, S, N, 16, "f32", X, X, np.eye(8, dtype=np.float32),
                    np.tile(np.eye(4, dtype=np.float32), (k, 1, 1)), np.full(k, 3.0, np.float32),
                    np.full(k, -3.0, np.float32), None)
    codes, scales, y, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR)
    ref = O.quant_act(X, w.A, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(scales, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])
    # every positive block collapses to a single code (its hi, the clipped amax)
    u = O.unpack_nibbles(codes[: S // 2]).reshape(S // 2, k, 32)
    assert (u == u[:, :, :1]).all()


def test_subnormal_blocks_and_smallest_scale():
    """Blocks whose values are E2M1 grid points times 2^-127 (many of them fp32
    subnormals): the shared exponent clamps at -127 (byte 0) and every code is exact."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float64)
    rng = np.random.default_rng(22)
    S, N = 24, 64
    k = N // 32
    X = np.empty((S, N), np.float32)
    for r in range(S):
        v = rng.choice(grid, N) * rng.choice([-1.0, 1.0], N)
        v[0] = 6.0  # every block's amax is 6 * 2^-127 -> e = -127
        v[32] = -6.0
        X[r] = (v * 2.0 ** -127).astype(np.float32)
    assert (np.abs(X[X != 0]) < 2.0 ** -126).any()  # subnormal inputs present
    w = WL.Workload("subnormal", 22, S, N, 16, "f32", X, X, np.eye(8, dtype=np.float32),
                    np.tile(np.eye(4, dtype=np.float32), (k, 1, 1)), np.full(k, 40, np.float32),
                    np.full(k, 40, np.float32), None)
    codes, scales, y, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR)
    np.testing.assert_array_equal(y, X)
    ref = O.quant_act(X, w.A, w.B, w.alpha_min, w.alpha_max)
    assert (ref["scales"] == 0).all()
    np.testing.assert_array_equal(scales, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])


@pytest.mark.parametrize("maker", [WL.tiny, lambda: WL.custom(200, 320, 16, 76),
                                   lambda: WL.q_proj(S=512, with_w=False)])
def test_block_hadamard_as_transform(maker):
    """The block-rotation baseline (every P_i = H32 / sqrt(32), no clip) given as the method's
    input runs through the same kernel and matches the oracle."""
    w = WL.with_block_hadamard(maker())
    codes, scales, y, _ = GU.gpu_quant(w)
    _check_all(w, codes, scales, y, label="block hadamard", literal_limit=PT.LITERAL_LIMIT_HADAMARD)


@pytest.mark.parametrize("S,N,seed", [(3001, 12288, 21), (8192, 4096, 22)])
def test_tensor_core_transform_large_ragged(S, N, seed):
    """Shapes with at least six 128 x 128 tiles per SM take the tensor-core transform; ragged S
    leaves a partial last tile.  Sampled rows (including the last ones) against the oracle, the
    GPU's own Y re-encoded bit-exact, and the padding rows of the last 128-row scale tile."""
    w = WL.custom(S, N, 16, seed, with_w=False)
    codes, scales, y, raw = GU.gpu_quant(w)
    rows = np.unique(np.concatenate([np.random.default_rng(seed).choice(S, 200, replace=False),
                                     np.arange(S - 40, S)]))
    _check_all(w, codes, scales, y, rows=rows, label=f"tc {S}x{N}")
    pad_rows = np.arange(S, (S + 127) // 128 * 128)
    if len(pad_rows):
        r, c = np.meshgrid(pad_rows, np.arange(w.k), indexing="ij")
        assert (raw[O.mma_scale_offset(r, c, w.k)] == 0x7F).all()
