"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each test compares the oracle with something other than itself: the pages'
Table 1 counts, a hand-derived worked example, textbook identities computed a
different way, brute-force search, exact integer arithmetic.  A plausible slip
in the oracle (transposed factor, swapped ratios, off-by-one exponent, wrong
tie rule or nibble order, wrong fusion direction) fails at least one of them.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import batq_oracle as O
from mxfp4_w4a4_post_block_b200 import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- Table 1 ----

def test_table1_parameter_counts():
    g = _golden("table1_param_counts.json")
    got = O.param_counts(**{"N": g["setting"]["N"], "g": g["setting"]["g"],
                            "g1": g["setting"]["g1"], "g2": g["setting"]["g2"]})
    assert got == g["counts"]


def test_table1_reduction_percentages():
    g = _golden("table1_param_counts.json")
    c = O.param_counts(4096)
    red = g["reduction_percent"]
    assert round(100 * (1 - c["gpk"] / c["wo"]), 1) == red["gpk_vs_wo"]
    assert round(100 * (1 - c["gpk"] / c["flatquant"])) == red["gpk_vs_flatquant"]
    assert round(100 * (1 - c["gpk"] / c["naive_kronecker"])) == red["gpk_vs_naive_kronecker"]


def test_swapped_factor_sizes_do_not_reproduce_table1():
    # A 4x4 global factor with 8x8 private factors would give a different count.
    assert O.param_counts(4096, g1=4, g2=8)["gpk"] != 2112


# ------------------------------------------------------- GPK transform -------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_kron_block_matches_textbook_kronecker():
    A, Bi = _rand((8, 8), 1), _rand((4, 4), 2)
    np.testing.assert_array_equal(O.kron_block(A, Bi), np.kron(Bi, A))


def test_vec_identity_BtXA_equals_x_times_P():
    # vec_r(B^T X A) = x (B (x) A) with X the row-major 4x8 reshape of x.
    rng = np.random.default_rng(3)
    for _ in range(20):
        A, Bi, x = rng.standard_normal((8, 8)), rng.standard_normal((4, 4)), rng.standard_normal(32)
        lhs = (Bi.T @ x.reshape(4, 8) @ A).reshape(-1)
        rhs = x @ O.kron_block(A, Bi)
        np.testing.assert_allclose(rhs, lhs, rtol=0, atol=1e-13 * np.abs(x).sum() * 10)


def test_transform_blockwise_matches_matrix_form():
    rng = np.random.default_rng(4)
    S, k = 5, 6
    X = rng.standard_normal((S, 32 * k))
    A, B = rng.standard_normal((8, 8)), rng.standard_normal((k, 4, 4))
    Y = O.transform_f64(X, A, B)
    for s in range(S):
        for i in range(k):
            Xm = X[s, 32 * i:32 * i + 32].reshape(4, 8)
            np.testing.assert_allclose(Y[s, 32 * i:32 * i + 32], (B[i].T @ Xm @ A).reshape(-1),
                                       rtol=1e-12, atol=1e-12)


def test_unit_vectors_reproduce_rows_of_P():
    A, Bi = _rand((8, 8), 5), _rand((4, 4), 6)
    X = np.eye(32)
    Y = O.transform_f64(X, A, Bi[None])
    np.testing.assert_array_equal(Y, np.kron(Bi, A))


def test_identity_transform_is_exact():
    X = _rand((7, 128), 7).astype(np.float32)
    B = np.broadcast_to(np.eye(4), (4, 4, 4))
    np.testing.assert_array_equal(O.transform(X, np.eye(8), B), X)


def test_transform_rounds_fp64_result_once_to_fp32():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((3, 64)).astype(np.float32)
    A, B = rng.standard_normal((8, 8)).astype(np.float32), rng.standard_normal((2, 4, 4)).astype(np.float32)
    exact = np.zeros((3, 64), dtype=object)
    for s in range(3):
        for i in range(2):
            Xm = [[Fraction(float(v)) for v in X[s, 32 * i + 8 * r:32 * i + 8 * r + 8]] for r in range(4)]
            for c in range(4):
                for b in range(8):
                    acc = Fraction(0)
                    for r in range(4):
                        for a in range(8):
                            acc += Fraction(float(B[i, r, c])) * Fraction(float(A[a, b])) * Xm[r][a]
                    exact[s, 32 * i + 8 * c + b] = acc
    want = np.array([[np.float32(float(v)) for v in row] for row in exact], dtype=np.float32)
    got = O.transform(X, A, B)
    # fp64 summation error is far below fp32 resolution; allow one fp32 ulp for double rounding.
    ulps = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1


def test_block_locality():
    w = WL.tiny(with_w=False)
    base = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    X2 = w.x.copy()
    X2[:, 32 * 3:32 * 4] *= -7.5
    pert = O.quant_act(X2, w.A, w.B, w.alpha_min, w.alpha_max)
    for i in range(w.k):
        same = slice(16 * i, 16 * i + 16)
        if i == 3:
            continue
        np.testing.assert_array_equal(pert["codes"][:, same], base["codes"][:, same])
        np.testing.assert_array_equal(pert["scales"][:, i], base["scales"][:, i])


# ------------------------------------------------------------- clipping ------

def test_clip_ratio_values():
    r = O.clip_ratios(np.array([0.0, 30.0, -30.0, 2.0, -2.0], dtype=np.float32))
    assert r[0] == np.float32(0.5)
    assert r[1] == np.float32(1.0)
    assert 0 < r[2] < 1e-12
    assert abs(float(r[3]) + float(r[4]) - 1.0) < 1e-7
    assert r[3] == np.float32(1 / (1 + math.exp(-2.0)))


def test_clip_with_unit_ratios_is_noop():
    Y = _rand((9, 96), 9).astype(np.float32)
    Yh, lo, hi, nf = O.clip_blocks(Y, np.ones(3, np.float32), np.ones(3, np.float32))
    np.testing.assert_array_equal(Yh, Y)
    assert not nf.any()


def test_clip_extremes_and_bounds():
    Y = _rand((11, 64), 10).astype(np.float32) * 5
    rmin = np.array([0.3, 0.9], np.float32)
    rmax = np.array([0.6, 0.1], np.float32)
    Yh, lo, hi, _ = O.clip_blocks(Y, rmin, rmax)
    Yb, Yhb = Y.reshape(11, 2, 32), Yh.reshape(11, 2, 32)
    for s in range(11):
        for i in range(2):
            mn, mx = Yb[s, i].min(), Yb[s, i].max()
            assert lo[s, i] == np.float32(float(rmin[i]) * float(mn))
            assert hi[s, i] == np.float32(float(rmax[i]) * float(mx))
            assert Yhb[s, i].min() == min(max(mn, lo[s, i]), hi[s, i])
            assert Yhb[s, i].max() == min(max(mx, lo[s, i]), hi[s, i])
            assert np.all(Yhb[s, i] >= min(lo[s, i], hi[s, i])) and np.all(Yhb[s, i] <= hi[s, i])
    # monotone: order preserved
    o = np.argsort(Yb[0, 0], kind="stable")
    assert np.all(np.diff(Yhb[0, 0][o]) >= 0)


def test_clip_lo_above_hi_gives_constant_hi():
    Y = np.linspace(1.0, 2.0, 32, dtype=np.float32)[None]
    Yh, lo, hi, _ = O.clip_blocks(Y, np.array([0.99], np.float32), np.array([0.1], np.float32))
    assert lo[0, 0] > hi[0, 0]
    assert np.all(Yh == hi[0, 0])


# ------------------------------------------------------ scale + encode -------

def _e2m1_value(code):
    # E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal.
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def test_magnitude_table_matches_format_definition():
    assert tuple(_e2m1_value(c) for c in range(8)) == O.E2M1_MAGNITUDE
    np.testing.assert_array_equal(O.e2m1_decode(np.arange(16)), [_e2m1_value(c) for c in range(16)])


def _brute_code(q):
    mags = [abs(_e2m1_value(c)) for c in range(8)]
    a = abs(q)
    d = [abs(a - m) for m in mags]
    best = min(d)
    cands = [c for c in range(8) if d[c] == best]
    even = [c for c in cands if c % 2 == 0]
    c = (even or cands)[0]
    return (8 if math.copysign(1.0, q) < 0 else 0) | c


def _brute_scale_exponent(amax):
    if amax == 0:
        return -127
    e = -160
    while not (2.0 ** (e + 2) <= amax < 2.0 ** (e + 3)):
        e += 1
    return max(-127, min(127, e))


def test_encoder_matches_brute_force_nearest_even():
    pts = [0.0, -0.0]
    for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
        pts += [m, np.nextafter(m, 0), np.nextafter(m, 10)]
    pts += list(np.linspace(0, 7.99, 4001))
    pts = np.array(pts + [-p for p in pts])
    got = O.e2m1_encode(pts)
    want = np.array([_brute_code(float(p)) for p in pts])
    np.testing.assert_array_equal(got, want)


def test_scale_exponent_matches_brute_force():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        np.float32(2.0) ** np.arange(-149, 128, dtype=np.float64),
        (rng.random(3000) * 10.0 ** rng.uniform(-40, 38, 3000)),
        [0.0, 1e-45, 3.4e38, 4.0, np.nextafter(4.0, 0), 0.7],
    ]).astype(np.float32).astype(np.float64)
    got = O.e8m0_exponent(vals)
    want = np.array([_brute_scale_exponent(float(v)) for v in vals])
    np.testing.assert_array_equal(got, want)


def test_identity_transform_unit_ratios_is_plain_mxfp4_rtn():
    rng = np.random.default_rng(12)
    S, k = 6, 5
    X = (rng.standard_t(3, (S, 32 * k)) * 10.0 ** rng.uniform(-3, 3, (S, 1))).astype(np.float32)
    B = np.broadcast_to(np.eye(4, dtype=np.float32), (k, 4, 4))
    big = np.full(k, 30.0, np.float32)  # sigma(30) rounds to exactly 1.0f
    out = O.quant_act(X, np.eye(8, dtype=np.float32), B, big, big)
    codes = O.unpack_nibbles(out["codes"])
    for s in range(S):
        for i in range(k):
            blk = X[s, 32 * i:32 * i + 32].astype(np.float64)
            e = _brute_scale_exponent(float(np.abs(blk).max()))
            assert out["scales"][s, i] == e + 127
            want = [_brute_code(float(v) / 2.0 ** e) for v in blk]
            assert list(codes[s, 32 * i:32 * i + 32]) == want


def test_roundtrip_of_representable_values():
    for e in range(-20, 21):
        vals = np.array([_e2m1_value(c) for c in range(16)] * 2, dtype=np.float64) * 2.0 ** e
        vals[0] = 6.0 * 2.0 ** e  # pin amax so the shared exponent is e
        packed, scale, _ = O.mxfp4_quantize(vals.astype(np.float32)[None])
        assert scale[0, 0] == e + 127
        np.testing.assert_array_equal(O.dequantize(packed, scale)[0], vals)


def test_amax_element_encodes_to_magnitude_4_or_6():
    w = WL.tiny(with_w=False)
    out = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    codes = O.unpack_nibbles(out["codes"]).reshape(w.S, w.k, 32)
    Yh = out["Y_hat"].reshape(w.S, w.k, 32)
    idx = np.abs(Yh).argmax(axis=2)
    top = np.take_along_axis(codes, idx[:, :, None], axis=2)[:, :, 0] & 7
    assert np.all((top == 6) | (top == 7))


def test_worked_example_bytes():
    g = _golden("clip_encode_worked_example.json")
    for blk in g["blocks"]:
        y = np.zeros(32, np.float32)
        y[:len(blk["y"])] = blk["y"]
        Yh, _, _, nf = O.clip_blocks(y[None], np.float32([blk["r_min"]]), np.float32([blk["r_max"]]))
        packed, scale, _ = O.mxfp4_quantize(Yh, nf)
        assert int(scale[0, 0]) == blk["scale"]
        assert list(packed[0]) == blk["bytes"]


def test_zero_and_nonfinite_blocks():
    Y = np.zeros((1, 96), np.float32)
    Y[0, 32 + 5] = np.inf
    Y[0, 64 + 9] = np.nan
    Yh, _, _, nf = O.clip_blocks(Y, np.ones(3, np.float32), np.ones(3, np.float32))
    packed, scale, _ = O.mxfp4_quantize(Yh, nf)
    assert list(scale[0]) == [0x00, 0xFF, 0xFF]
    assert not packed.any()


def test_nibble_order():
    codes = np.arange(16, dtype=np.uint8)[None].repeat(2, 0)
    packed = O.pack_nibbles(codes)
    assert packed[0, 0] == 0x10 and packed[0, 7] == 0xFE
    np.testing.assert_array_equal(O.unpack_nibbles(packed), codes)


def test_mma_scale_layout_is_a_bijection():
    for rows, k in ((16, 8), (128, 4), (300, 10), (2048, 128)):
        r, c = np.meshgrid(np.arange(rows), np.arange(k), indexing="ij")
        off = O.mma_scale_offset(r, c, k).reshape(-1)
        assert len(np.unique(off)) == off.size
        assert off.max() < O.mma_layout_bytes(rows, k)


def test_mma_scale_layout_worked_entries():
    """Entries worked by hand from the tcgen05 block-scale atom: a 512-byte atom holds 128 rows x 4
    scales as 32 lines of 16 bytes, line i carrying rows i, i + 32, i + 64, i + 96 (4 bytes each, one
    per block column); atoms run along K within a 128-row tile, then tile after tile (k padded to a
    multiple of 4).  A layout that is one-to-one but swaps any of these roles fails here."""
    worked = [  # (row, kb, k, offset)
        (0, 0, 8, 0), (1, 0, 8, 16), (32, 0, 8, 4), (33, 2, 8, 22), (96, 3, 8, 15), (127, 3, 8, 511),
        (0, 4, 8, 512), (5, 7, 8, 512 + 80 + 3), (128, 0, 8, 1024), (130, 5, 8, 1569),
        (128, 9, 10, 2561), (255, 11, 10, 3 * 512 + 2 * 512 + 511),
    ]
    for row, kb, k, off in worked:
        assert int(O.mma_scale_offset(row, kb, k)) == off, (row, kb, k)


# ------------------------------------------------------- weight side ---------

def test_gauss_jordan_inverse_matches_kronecker_inverse():
    rng = np.random.default_rng(13)
    A = np.eye(8) + 0.3 * rng.standard_normal((8, 8))
    Bi = np.eye(4) + 0.3 * rng.standard_normal((4, 4))
    Pinv = O.gauss_jordan_inverse(O.kron_block(A, Bi))
    np.testing.assert_allclose(Pinv, np.kron(np.linalg.inv(Bi), np.linalg.inv(A)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.kron_block(A, Bi) @ Pinv, np.eye(32), rtol=0, atol=1e-12)


def test_singular_transform_rejected():
    with pytest.raises(np.linalg.LinAlgError):
        O.gauss_jordan_inverse(O.kron_block(np.eye(8), np.zeros((4, 4))))


def test_weight_fusion_invariance_before_quantization():
    # (X P)(P^{-1} W^T) = X W^T
    w = WL.tiny()
    lhs = O.transform_f64(w.x, w.A, w.B) @ O.fuse_weights_f64(w.W, w.A, w.B).T
    rhs = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    scale = np.abs(w.x).astype(np.float64) @ np.abs(w.W).astype(np.float64).T
    assert np.max(np.abs(lhs - rhs) / scale) < 1e-12


def test_weight_fusion_direction_matters():
    w = WL.tiny()
    rhs = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    # transpose error on the inverse: W P^{-1} instead of W P^{-T}
    Wt = np.empty_like(w.W, dtype=np.float64)
    for i in range(w.k):
        Pinv = np.linalg.inv(O.kron_block(w.A, w.B[i]))
        Wt[:, 32 * i:32 * i + 32] = w.W[:, 32 * i:32 * i + 32] @ Pinv
    bad = O.transform_f64(w.x, w.A, w.B) @ Wt.T
    assert not np.allclose(bad, rhs, rtol=1e-6)


def test_prepare_weights_is_unclipped_rtn_of_fused_weights():
    w = WL.tiny()
    wp = O.prepare_weights(w.W, w.A, w.B)
    Wf = O.fuse_weights_f64(w.W, w.A, w.B).astype(np.float32)
    np.testing.assert_array_equal(wp["W_fused"], Wf)
    codes = O.unpack_nibbles(wp["codes"])
    for m in range(0, w.M, 17):
        for i in range(w.k):
            blk = Wf[m, 32 * i:32 * i + 32].astype(np.float64)
            e = _brute_scale_exponent(float(np.abs(blk).max()))
            assert wp["scales"][m, i] == e + 127
            assert list(codes[m, 32 * i:32 * i + 32]) == [_brute_code(float(v) / 2.0 ** e) for v in blk]


# -------------------------------------------------------------- GEMM ---------

def _exact_dot(ca, sa, cw, sw):
    """Exact sum of products of E2M1 values with E8M0 scales as a Fraction."""
    total = Fraction(0)
    for n in range(len(ca)):
        va = Fraction(_e2m1_value(int(ca[n]))) * Fraction(2) ** (int(sa[n // 32]) - 127)
        vw = Fraction(_e2m1_value(int(cw[n]))) * Fraction(2) ** (int(sw[n // 32]) - 127)
        total += va * vw
    return total


def test_gemm_brute_force_tiny_shapes():
    rng = np.random.default_rng(14)
    for S, M in ((1, 1), (2, 3), (4, 4)):
        a = rng.integers(0, 256, (S, 32), dtype=np.uint8)
        b = rng.integers(0, 256, (M, 32), dtype=np.uint8)
        sa = rng.integers(110, 140, (S, 2), dtype=np.uint8)
        sb = rng.integers(110, 140, (M, 2), dtype=np.uint8)
        out, T = O.gemm(a, sa, b, sb)
        ca, cb = O.unpack_nibbles(a), O.unpack_nibbles(b)
        for s in range(S):
            for m in range(M):
                ex = _exact_dot(ca[s], sa[s], cb[m], sb[m])
                assert out[s, m] == float(ex)
                tt = sum(abs(_e2m1_value(int(ca[s, n])) * _e2m1_value(int(cb[m, n]))) *
                         2.0 ** (int(sa[s, n // 32]) + int(sb[m, n // 32]) - 254) for n in range(64))
                assert T[s, m] == tt


def test_gemm_exact_on_tiny_config():
    w = WL.tiny()
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    wp = O.prepare_weights(w.W, w.A, w.B)
    out, T = O.gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    ca, cw = O.unpack_nibbles(act["codes"]), O.unpack_nibbles(wp["codes"])
    rng = np.random.default_rng(15)
    for s, m in zip(rng.integers(0, w.S, 24), rng.integers(0, w.M, 24)):
        ex = _exact_dot(ca[s], act["scales"][s], cw[m], wp["scales"][m])
        assert abs(out[s, m] - float(ex)) <= 1e-15 * T[s, m]


def test_gemm_linear_in_codes_order():
    w = WL.tiny()
    act = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    wp = O.prepare_weights(w.W, w.A, w.B)
    out, _ = O.gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    # reverse the block order on both operands: same sums
    perm = np.arange(w.k)[::-1]
    ac = act["codes"].reshape(w.S, w.k, 16)[:, perm].reshape(w.S, -1)
    wc = wp["codes"].reshape(w.M, w.k, 16)[:, perm].reshape(w.M, -1)
    out2, _ = O.gemm(ac, act["scales"][:, perm], wc, wp["scales"][:, perm])
    np.testing.assert_allclose(out2, out, rtol=1e-13, atol=1e-13)


# ------------------------------------------------- W4A8 (MXFP8 E4M3) ----

def _e4m3_value_from_bits(c):
    """E4M3 from its bit fields, written independently of the oracle's table:
    sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0; exponent 0 is subnormal."""
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 7
    if e == 0xF and m == 7:
        return math.nan
    return s * (m / 8.0 * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))


def test_e4m3_table_matches_bit_fields_and_extremes():
    vals = [_e4m3_value_from_bits(c) for c in range(0x7F)]
    np.testing.assert_array_equal(O.E4M3_MAGNITUDE, vals)
    assert O.E4M3_MAGNITUDE[0x7E] == 448.0 and O.E4M3_MAGNITUDE[1] == 2.0 ** -9
    assert O.E4M3_MAGNITUDE[8] == 2.0 ** -6  # smallest normal
    for c in range(256):
        if (c & 0x7F) != 0x7F:
            v = O.e4m3_decode(np.array([c]))[0]
            assert v == _e4m3_value_from_bits(c) or (v == 0 and _e4m3_value_from_bits(c) == 0)


def test_e4m3_encode_brute_force_nearest_even_saturating():
    """Against a search over all finite codes: nearest value, ties to the even code,
    |q| > 448 saturates, sign from the sign of q."""
    rng = np.random.default_rng(7)
    mags = np.concatenate([rng.uniform(0, 500, 3000), np.exp2(rng.uniform(-12, 9, 3000)),
                           (O.E4M3_MAGNITUDE[:-1] + O.E4M3_MAGNITUDE[1:]) / 2,  # every midpoint
                           O.E4M3_MAGNITUDE, [448.0, 456.0, 464.0, 470.0, 1e6]])
    q = mags * rng.choice([-1.0, 1.0], len(mags))
    table = np.array([_e4m3_value_from_bits(c) for c in range(0x7F)])
    got = O.e4m3_encode(q)
    for qi, ci in zip(q, got):
        a = min(abs(qi), 448.0)
        d = np.abs(table - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert ci == (want | (0x80 if np.signbit(qi) else 0)), (qi, ci, want)


def test_e4m3_round_trip_and_sign_of_zero():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = _e4m3_value_from_bits(c)
        want = c if not (c == 0x80) else 0x80
        assert O.e4m3_encode(np.array([v if c != 0x80 else -0.0]))[0] == want
    assert O.e4m3_encode(np.array([-1e-9]))[0] == 0x80


def test_mxfp8_scale_rule_and_amax_range():
    """e = floor(log2 amax) - 8: the scaled amax lies in [256, 512) and encodes to a
    magnitude in [256, 448] (saturating above 448)."""
    rng = np.random.default_rng(8)
    V = (rng.standard_normal((64, 256)) * np.exp2(rng.integers(-20, 20, (64, 1)))).astype(np.float32)
    codes, scales, q = O.mxfp8_quantize(V)
    amax = np.abs(V.reshape(64, 8, 32).astype(np.float64)).max(axis=2)
    e = scales.astype(np.int64) - 127
    np.testing.assert_array_equal(e, np.floor(np.log2(amax)).astype(np.int64) - 8)
    qa = amax * np.exp2(-e)
    assert (qa >= 256).all() and (qa < 512).all()
    mag_codes = codes.reshape(64, 8, 32) & 0x7F
    top = np.take_along_axis(mag_codes, np.abs(V.reshape(64, 8, 32)).argmax(axis=2)[:, :, None], axis=2)[:, :, 0]
    assert (O.E4M3_MAGNITUDE[top] >= 256).all() and (O.E4M3_MAGNITUDE[top] <= 448).all()


def test_mxfp8_identity_transform_reduces_to_plain_rtn():
    w = WL.custom(8, 128, 16, 31, x_dtype="f32", with_w=False)
    k = 4
    A, B = np.eye(8), np.tile(np.eye(4), (k, 1, 1))
    act = O.quant_act_mxfp8(w.x, A, B, np.full(k, 40.0), np.full(k, 40.0))
    codes, scales, _ = O.mxfp8_quantize(w.x)
    np.testing.assert_array_equal(act["codes"], codes)
    np.testing.assert_array_equal(act["scales"], scales)
    # dequantized values: within half an E4M3 step of x (relative 2^-4, or 2^-10 of the
    # scale among the subnormals), except that |q| > 448 saturates to exactly 448 * scale
    deq = O.dequantize_e4m3(codes, scales).reshape(8, k, 32)
    x = w.x.astype(np.float64).reshape(8, k, 32)
    s = np.exp2(scales.astype(np.float64) - 127)[:, :, None]
    sat = np.abs(x) / s > 448
    assert (np.abs(deq[sat]) == (448 * np.broadcast_to(s, x.shape))[sat]).all()
    half = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s)
    assert (np.abs(deq - x)[~sat] <= half[~sat]).all()


def test_e4m3_containers_hold_the_e2m1_values_exactly():
    packed = O.pack_nibbles(np.arange(16, dtype=np.uint8).reshape(1, 16))
    c8 = O.e4m3_containers_from_e2m1(packed)
    np.testing.assert_array_equal(O.e4m3_decode(c8)[0], O.e2m1_decode(np.arange(16)))
    # positive E2M1 values sit at E4M3 bytes 0x00, 0x30, 0x38, 0x3C, 0x40, 0x44, 0x48, 0x4C
    assert c8[0, :8].tolist() == [0x00, 0x30, 0x38, 0x3C, 0x40, 0x44, 0x48, 0x4C]


def test_gemm_w4a8_exact_on_small_random_codes():
    """The fp64 GEMM equals an exact rational sum of the dequantized products."""
    rng = np.random.default_rng(9)
    S, M, N = 3, 4, 64
    a8 = rng.integers(0, 256, (S, N)).astype(np.uint8)
    a8[(a8 & 0x7F) == 0x7F] = 0x11
    w4 = rng.integers(0, 256, (M, N // 2)).astype(np.uint8)
    w8 = O.e4m3_containers_from_e2m1(w4)
    sa = rng.integers(110, 140, (S, 2)).astype(np.uint8)
    sw = rng.integers(110, 140, (M, 2)).astype(np.uint8)
    out, T = O.gemm_w4a8(a8, sa, w8, sw)
    for s in range(S):
        for m in range(M):
            tot = Fraction(0)
            for n in range(N):
                va = Fraction(_e4m3_value_from_bits(int(a8[s, n]))) * Fraction(2) ** (int(sa[s, n // 32]) - 127)
                vw = Fraction(O.e2m1_decode(np.array([int(O.unpack_nibbles(w4)[m, n])]))[0]) \
                    * Fraction(2) ** (int(sw[m, n // 32]) - 127)
                tot += va * vw
            # fp64 accumulation of 64 terms: within n * 2^-53 of the sum of magnitudes
            assert abs(Fraction(float(out[s, m])) - tot) <= Fraction(N, 2 ** 53) * Fraction(float(T[s, m]))


# ------------------------------------------------------- NVFP4 output ----

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _nearest_e4m3_code(u: Fraction) -> int:
    """Brute force over the finite non-negative E4M3 codes: nearest value, ties to even, >448 -> 448."""
    table = [Fraction(_e4m3_value_from_bits(c)) for c in range(0x7F)]
    u = min(u, Fraction(448))
    d = [abs(t - u) for t in table]
    best = [c for c in range(0x7F) if d[c] == min(d)]
    return best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]


def _nearest_e2m1_mag(q: Fraction) -> int:
    vals = [Fraction(v) for v in E2M1_VALUES]
    a = min(abs(q), Fraction(6))
    d = [abs(v - a) for v in vals]
    best = [c for c in range(8) if d[c] == min(d)]
    return best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]


def test_nvfp4_worked_example_two_groups():
    """Hand-derived: group 0 has amax 6 (scale 6/6 = 1.0, byte 0x38) and holds every
    E2M1 midpoint, so each rounds to its even neighbour; group 1 has amax 48 (scale 8,
    byte 0x50 = exponent field 10, mantissa 0) and holds values that are exact codes x 8."""
    g0 = [6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, -0.25, 0, 1, 2, 3, 4, -6, 0.5]
    g1 = [48, -24, 12, 4, 0, -8, 16, 32, 2, -2, 1, 0.5, 40, -44, 20, 28]
    codes, scales, _ = O.nvfp4_quantize(np.array([g0 + g1], np.float32))
    assert scales.tolist() == [[0x38, 0x50]]
    want0 = [7, 6, 6, 4, 4, 2, 2, 0, 8, 0, 2, 4, 5, 6, 15, 1]
    # group 1 / 8: 6, -3, 1.5, 0.5, 0, -1, 2, 4, 0.25->0, -0.25->-0, 0.125->0, 0.0625->0,
    # 5 -> 4 (tie, even), -5.5 -> -6, 2.5 -> 2 (tie, even), 3.5 -> 4 (tie, even)
    want1 = [7, 13, 3, 1, 0, 10, 4, 6, 0, 8, 0, 0, 6, 15, 4, 6]
    assert O.unpack_nibbles(codes)[0].tolist() == want0 + want1


def test_nvfp4_scale_is_nearest_e4m3_of_amax_times_gs_over_six():
    rng = np.random.default_rng(21)
    amax = (np.exp2(rng.uniform(-14, 10, 400)) * rng.uniform(1, 2, 400)).astype(np.float32)
    for gs in (1.0, 3.0, 1234.5678, 2.0 ** -5):
        byte, sval, mult = O.nvfp4_group_scale(amax, gs)
        g32 = Fraction(float(np.float32(gs)))
        for a, b, s, m in zip(amax, byte, sval, mult):
            u = Fraction(float(a)) * g32 / 6
            want = _nearest_e4m3_code(u)
            # the steps round to fp32 twice on the way: skip values within 2^-21 of an E4M3 midpoint
            mids = [abs(u - (Fraction(_e4m3_value_from_bits(c)) + Fraction(_e4m3_value_from_bits(c + 1))) / 2)
                    for c in range(0x7E)]
            if u > 0 and min(mids) <= u * Fraction(1, 2 ** 21):
                continue
            assert b == want, (a, gs, b, want)
            assert s == _e4m3_value_from_bits(int(b))
            assert (m == 0) if s == 0 else abs(Fraction(float(m)) - g32 / Fraction(float(s))) <= \
                g32 / Fraction(float(s)) * Fraction(1, 2 ** 24)


def test_nvfp4_codes_brute_force_against_exact_quotient():
    """Every element's code is the nearest E2M1 value (ties even, saturating) to v * gs / scale,
    for elements not within 2^-21 of a rounding boundary."""
    rng = np.random.default_rng(22)
    V = (rng.standard_t(4, (8, 64)) * np.exp2(rng.integers(-6, 6, (8, 1)))).astype(np.float32)
    for gs in (1.0, 77.0):
        codes, scales, _ = O.nvfp4_quantize(V, gs)
        c = O.unpack_nibbles(codes)
        g32 = Fraction(float(np.float32(gs)))
        checked = 0
        for r in range(8):
            for n in range(64):
                s = Fraction(_e4m3_value_from_bits(int(scales[r, n // 16])))
                v = Fraction(float(V[r, n]))
                if s == 0:
                    continue
                q = v * g32 / s
                if any(abs(abs(q) - Fraction(mid)) <= abs(q) * Fraction(1, 2 ** 21)
                       for mid in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)):
                    continue
                want = _nearest_e2m1_mag(q) | (8 if v < 0 or (v == 0 and np.signbit(V[r, n])) else 0)
                assert c[r, n] == want, (r, n, float(q), c[r, n], want)
                checked += 1
        assert checked > 400


def test_nvfp4_group_amax_element_encodes_to_six():
    """With a normal, unsaturated scale, amax * gs / scale lies in [6 / (1 + 2^-4), 6 / (1 - 2^-4)],
    so the group's largest element always takes magnitude code 7 (value 6)."""
    rng = np.random.default_rng(23)
    V = (rng.standard_normal((32, 128)) * np.exp2(rng.integers(-3, 5, (32, 1)))).astype(np.float32)
    codes, scales, q = O.nvfp4_quantize(V, 1.0)
    c = O.unpack_nibbles(codes).reshape(32, 8, 16)
    top = np.abs(V.reshape(32, 8, 16)).argmax(axis=2)
    sval = O.e4m3_decode(scales)
    normal = (sval >= 2.0 ** -6) & (sval < 448)
    got = np.take_along_axis(c, top[:, :, None], axis=2)[:, :, 0] & 7
    assert normal.sum() > 200 and (got[normal] == 7).all()
    qa = np.take_along_axis(np.abs(q).reshape(32, 8, 16), top[:, :, None], axis=2)[:, :, 0]
    assert (qa[normal] >= 6 / (1 + 2 ** -4) - 1e-9).all() and (qa[normal] <= 6 / (1 - 2 ** -4) + 1e-9).all()


def test_nvfp4_power_of_two_global_scale_moves_only_the_scales():
    rng = np.random.default_rng(24)
    V = rng.standard_normal((16, 64)).astype(np.float32)
    c1, s1, _ = O.nvfp4_quantize(V, 1.0)
    c8, s8, _ = O.nvfp4_quantize(V, 8.0)
    np.testing.assert_array_equal(c1, c8)
    np.testing.assert_array_equal(O.e4m3_decode(s8), 8 * O.e4m3_decode(s1))
    np.testing.assert_array_equal(O.dequantize_nvfp4(c8, s8, 8.0), O.dequantize_nvfp4(c1, s1, 1.0))


def test_nvfp4_subnormal_zero_and_saturated_scales():
    """amax 6 * 2^-9 gives u = 2^-9, the smallest subnormal scale (byte 0x01, multiplier 512);
    a group whose u rounds to zero gets byte 0 and zero codes that keep their sign; amax 3000
    gives u = 500, which saturates to 448 (byte 0x7E), and the largest elements to +-6."""
    g_sub = [6 * 2.0 ** -9, 2.0 ** -9] + [0.0] * 14
    g_zero = [-1e-30, 1e-30] + [0.0] * 14
    g_sat = [3000.0, -2900.0, 100.0] + [0.0] * 13
    V = np.array([g_sub + g_zero, g_sat + [0.0] * 16], np.float32)
    codes, scales, _ = O.nvfp4_quantize(V, 1.0)
    c = O.unpack_nibbles(codes)
    assert scales.tolist() == [[0x01, 0x00], [0x7E, 0x00]]
    assert c[0, :2].tolist() == [7, 2] and c[0, 16:18].tolist() == [8, 0]
    assert c[1, :3].tolist() == [7, 15, 0]
    assert (c[1, 16:] == 0).all()


def test_nvfp4_nonfinite_block_gives_nan_scales_for_both_groups():
    V = np.ones((1, 64), np.float32)
    V[0, 20] = np.inf                      # second group of block 0
    codes, scales, _ = O.nvfp4_quantize(V, 1.0)
    assert scales.tolist() == [[0x7F, 0x7F, 0x23, 0x23]]   # 1/6 -> 2^-3 x 1.375 = 0.171875 (0x23)
    c = O.unpack_nibbles(codes)[0]
    assert (c[:32] == 0).all() and (c[32:] == 7).all()


def test_nvfp4_identity_transform_and_whole_block_clip():
    """With P = I the path is plain NVFP4 of the clipped values, and the clip thresholds come
    from the whole 32-element block, not from each 16-element group."""
    w = WL.custom(8, 128, 16, 33, x_dtype="f32", with_w=False)
    k = 4
    A, B = np.eye(8), np.tile(np.eye(4), (k, 1, 1))
    act = O.quant_act_nvfp4(w.x, A, B, np.full(k, 40.0), np.full(k, 40.0), 2.0)
    codes, scales, _ = O.nvfp4_quantize(w.x, 2.0)
    np.testing.assert_array_equal(act["codes"], codes)
    np.testing.assert_array_equal(act["scales"], scales)
    # ratios 1/2: each block is clipped to [min/2, max/2] of the whole block
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = np.linspace(-1, 1, 16)     # group 0: extrema +-1
    x[0, 16] = 8.0                         # group 1 holds the block max
    act = O.quant_act_nvfp4(x, np.eye(8), np.eye(4)[None], [0.0], [0.0])
    np.testing.assert_array_equal(act["Y_hat"][0, :16], np.clip(x[0, :16], -0.5, 4.0))
    assert act["Y_hat"][0, 16] == 4.0
    # group 0 keeps +1 (below hi = 4), so its amax is 1; group 1's amax is the clipped max 4
    assert act["scales"].tolist() == [[0x23, O.e4m3_encode(np.array([4 / 6]))[0]]]


def test_nvfp4_dequantization_error_within_half_a_step():
    """|deq - v| <= half the E2M1 spacing at |q| (0.25, 0.5 or 1) x scale / gs, plus the
    fp32 rounding of the multiplier; saturated elements decode to exactly 6 x scale / gs."""
    rng = np.random.default_rng(25)
    V = (rng.standard_normal((32, 256)) * 3).astype(np.float32)
    gs = 10.0
    codes, scales, q = O.nvfp4_quantize(V, gs)
    deq = O.dequantize_nvfp4(codes, scales, gs)
    s = np.repeat(O.e4m3_decode(scales), 16, axis=1) / np.float32(gs)
    aq = np.abs(q)
    half = np.where(aq <= 2, 0.25, np.where(aq <= 4, 0.5, 1.0))
    sat = aq > 6
    err = np.abs(deq - V.astype(np.float64))
    assert (err[~sat] <= (half * s * (1 + 2.0 ** -20))[~sat]).all()
    assert sat.sum() > 10
    np.testing.assert_allclose(np.abs(deq[sat]), (6 * s)[sat], rtol=1e-15, atol=0)


def test_nvfp4_global_scale_maps_tensor_amax_to_the_largest_scale():
    rng = np.random.default_rng(26)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    amax = float(np.abs(W).max())
    gs = O.nvfp4_global_scale(amax)
    assert gs == float(np.float32(np.float64(2688.0) / np.float64(np.float32(amax))))
    codes, scales, _ = O.nvfp4_quantize(W, gs)
    r, c = np.unravel_index(np.abs(W).argmax(), W.shape)
    assert scales[r, c // 16] == 0x7E      # amax * gs / 6 = 448 (up to fp32 rounding)
    assert O.nvfp4_global_scale(0.0) == 1.0
    a = O.nvfp4_alpha(gs, 4.0)
    assert a == float(np.float32(1.0 / float(np.float32(gs * 4.0))))


def test_nvfp4_fp32_steps_match_single_precision_arithmetic():
    """The oracle's fp32 rounding of fp64 products and quotients equals IEEE single arithmetic."""
    rng = np.random.default_rng(27)
    a = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    b = (rng.standard_normal(20000) * np.exp2(rng.integers(-30, 30, 20000))).astype(np.float32)
    np.testing.assert_array_equal(O.f32(a.astype(np.float64) * b), (a * b).astype(np.float64))
    np.testing.assert_array_equal(O.f32(a.astype(np.float64) / b), (a / b).astype(np.float64))


def test_nvfp4_scales_in_mma_layout_round_trip():
    rows, k16 = 200, 24
    rng = np.random.default_rng(28)
    lin = rng.integers(0, 0x7F, (rows, k16)).astype(np.uint8)
    buf = np.zeros(O.mma_layout_bytes(rows, k16), np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(k16), indexing="ij")
    buf[O.mma_scale_offset(r, c, k16)] = lin
    np.testing.assert_array_equal(O.scales_from_mma_layout(buf, rows, k16), lin)
    assert O.mma_layout_bytes(rows, k16) == 256 * 24


def test_gemm_nvfp4_exact_on_small_random_codes():
    """alpha x (fp64 GEMM) equals the exact rational sum of (code x E4M3 scale) products."""
    rng = np.random.default_rng(29)
    S, M, N = 3, 4, 64
    a4 = rng.integers(0, 256, (S, N // 2)).astype(np.uint8)
    w4 = rng.integers(0, 256, (M, N // 2)).astype(np.uint8)
    sa = rng.integers(0, 0x7F, (S, 4)).astype(np.uint8)
    sw = rng.integers(0, 0x7F, (M, 4)).astype(np.uint8)
    alpha = 0.375
    out, T = O.gemm_nvfp4(a4, sa, w4, sw, alpha)
    ca, cw = O.unpack_nibbles(a4), O.unpack_nibbles(w4)
    for s in range(S):
        for m in range(M):
            tot = Fraction(0)
            for n in range(N):
                va = Fraction(float(O.e2m1_decode(np.array([int(ca[s, n])]))[0])) * \
                    Fraction(_e4m3_value_from_bits(int(sa[s, n // 16])))
                vw = Fraction(float(O.e2m1_decode(np.array([int(cw[m, n])]))[0])) * \
                    Fraction(_e4m3_value_from_bits(int(sw[m, n // 16])))
                tot += va * vw
            tot *= Fraction(alpha)
            assert abs(Fraction(float(out[s, m])) - tot) <= Fraction(N + 1, 2 ** 53) * Fraction(float(T[s, m]))


def test_nvfp4_error_below_mxfp4_on_gaussian_blocks():
    """Finer groups with mantissa-carrying scales: on Gaussian data the NVFP4 round trip has a
    smaller mean squared error than MXFP4's (a property of the two formats, checked on a
    seeded sample)."""
    rng = np.random.default_rng(30)
    V = rng.standard_normal((64, 1024)).astype(np.float32)
    c4, s4, _ = O.mxfp4_quantize(V)
    cn, sn, _ = O.nvfp4_quantize(V, 1.0)
    e_mx = np.mean((O.dequantize(c4, s4) - V) ** 2)
    e_nv = np.mean((O.dequantize_nvfp4(cn, sn) - V) ** 2)
    assert e_nv < 0.8 * e_mx, (e_nv, e_mx)


# ------------------------------------------------ block Hadamard as P_i ----

def test_block_hadamard_factors_give_h32_over_sqrt32():
    """A = H8/sqrt(8), B_i = H4/2 (Sylvester) give P_i = H32/sqrt(32): checked against scipy's
    independent Hadamard construction; P_i is orthogonal, so the fused weights use P_i itself."""
    from scipy.linalg import hadamard
    w = WL.with_block_hadamard(WL.tiny())
    P = O.dense_blocks(w.A, w.B)
    ref = hadamard(32) / np.sqrt(32.0)
    assert np.abs(P - ref[None]).max() < 1e-7
    np.testing.assert_allclose(P[0] @ P[0].T, np.eye(32), atol=1e-6)
    np.testing.assert_allclose(O.gauss_jordan_inverse(P[0]), P[0].T, atol=1e-6)
    assert (O.clip_ratios(w.alpha_min) == 1.0).all()


def test_block_hadamard_of_a_unit_vector_is_a_sign_row():
    """x = e_j gives y = row j of H32 / sqrt(32): every |y| = 2^-2.5, scale exponent -5, every
    scaled value +-5.66 -> magnitude 6, with the signs of row j of scipy's H32."""
    from scipy.linalg import hadamard
    w = WL.with_block_hadamard(WL.tiny(with_w=False))
    X = np.zeros((32, 256), np.float32)
    for j in range(32):
        X[j, 32 + j] = 1.0                      # block column 1
    act = O.quant_act(X, w.A, w.B, w.alpha_min, w.alpha_max)
    codes = O.unpack_nibbles(act["codes"])
    assert (act["scales"][:, 1] == 127 - 5).all()
    H = hadamard(32)
    for j in range(32):
        assert ((codes[j, 32:64] & 7) == 7).all()
        np.testing.assert_array_equal(codes[j, 32:64] >> 3, (H[j] < 0).astype(np.uint8))


# ------------------------------------------------------------- KV cache ----

def test_kv_cache_scatter_invariants():
    """A skipped token changes nothing, the cache does not depend on the order of the new tokens,
    and each written row depends only on its own token (rows of another token perturbed: unchanged)."""
    w = WL.custom(12, 256, 16, 41, x_dtype="f32", with_w=False)
    rng = np.random.default_rng(41)
    n = 20
    cc0 = rng.integers(0, 256, (n, 128), dtype=np.uint8)
    cs0 = rng.integers(0, 256, (n, 8), dtype=np.uint8)
    slots = rng.permutation(n)[:12]
    slots[3] = -1
    slots[7] = n + 5
    for fmt in ("mxfp4", "mxfp8"):
        width = 128 if fmt == "mxfp4" else 256
        cc = rng.integers(0, 256, (n, width), dtype=np.uint8)
        c1, s1, act = O.quant_kv_cache(w.x, w.A, w.B, w.alpha_min, w.alpha_max, slots, cc, cs0, fmt)
        untouched = np.setdiff1d(np.arange(n), slots[(slots >= 0) & (slots < n)])
        np.testing.assert_array_equal(c1[untouched], cc[untouched])
        np.testing.assert_array_equal(s1[untouched], cs0[untouched])
        perm = rng.permutation(12)
        c2, s2, _ = O.quant_kv_cache(w.x[perm], w.A, w.B, w.alpha_min, w.alpha_max, slots[perm], cc, cs0, fmt)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1, s2)
        x3 = w.x.copy()
        x3[5] *= 7.0
        c3, s3, _ = O.quant_kv_cache(x3, w.A, w.B, w.alpha_min, w.alpha_max, slots, cc, cs0, fmt)
        others = np.array([s for r, s in enumerate(slots) if r != 5 and 0 <= s < n])
        np.testing.assert_array_equal(c3[others], c1[others])
        np.testing.assert_array_equal(s3[others], s1[others])
        assert not np.array_equal(c3[slots[5]], c1[slots[5]]) or not np.array_equal(s3[slots[5]], s1[slots[5]])


# ---------------------------------------------- naive Kronecker (per-block A_i) ----

def test_naive_kronecker_blocks_are_numpy_kron_of_the_pair():
    """P_i = B_i (x) A_i against numpy's Kronecker product, block by block."""
    w = WL.with_naive_kronecker(WL.tiny(with_w=False), 5)
    P = O.dense_blocks(w.A, w.B)
    for i in range(w.k):
        np.testing.assert_array_equal(P[i], np.kron(w.B[i].astype(np.float64), w.A[i].astype(np.float64)))
    assert O.param_counts(4096)["naive_kronecker"] == 128 * (64 + 16)


def test_naive_kronecker_with_equal_factors_is_gpk():
    """A_i = A for every block reproduces the GPK path bit for bit (activations and weights)."""
    w = WL.tiny()
    Ak = np.repeat(w.A[None], w.k, axis=0)
    a1 = O.quant_act(w.x, w.A, w.B, w.alpha_min, w.alpha_max)
    a2 = O.quant_act(w.x, Ak, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(a1["codes"], a2["codes"])
    np.testing.assert_array_equal(a1["scales"], a2["scales"])
    np.testing.assert_array_equal(a1["Y"], a2["Y"])
    w1, w2 = O.prepare_weights(w.W, w.A, w.B), O.prepare_weights(w.W, Ak, w.B)
    np.testing.assert_array_equal(w1["codes"], w2["codes"])


def test_naive_kronecker_block_locality_and_fusion_invariance():
    """Changing A_j changes block j only; (x P)(P^-1 W^T) = x W^T with per-block factors."""
    w = WL.with_naive_kronecker(WL.tiny(), 6)
    Y = O.transform_f64(w.x, w.A, w.B)
    A2 = w.A.copy()
    A2[3] = A2[3] * 1.5 + 0.1
    Y2 = O.transform_f64(w.x, A2, w.B)
    changed = np.abs(Y2 - Y).reshape(w.S, w.k, 32).max(axis=(0, 2)) > 0
    assert changed.tolist() == [j == 3 for j in range(w.k)]
    Wf = O.fuse_weights_f64(w.W, w.A, w.B)
    ref = w.x.astype(np.float64) @ w.W.astype(np.float64).T
    got = Y @ Wf.T
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(w.x).sum(1).max() * np.abs(w.W).max() * 10


# ------------------------------------------------- RMSNorm ahead of the transform ----

def test_rmsnorm_matches_torch_rms_norm():
    """Against torch's own RMSNorm (fp64 CPU), with a non-trivial weight and eps."""
    import torch
    rng = np.random.default_rng(51)
    X = rng.standard_normal((9, 256)) * np.exp2(rng.integers(-4, 4, (9, 1)))
    g = rng.uniform(0.5, 1.5, 256)
    for eps in (0.0, 1e-6, 0.3):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(X), (256,), torch.from_numpy(g), eps).numpy()
        np.testing.assert_allclose(O.rmsnorm(X, g, eps), ref, rtol=1e-13, atol=0)


def test_rmsnorm_quant_closed_forms_and_invariances():
    """A constant row c normalises to sign(c) gamma exactly (eps = 0): with P = I, no clip and
    gamma = 1 every value is +-1, scale exponent -2, code magnitude 6 (value 4).  Scaling a row by a
    power of two changes nothing (eps = 0); a zero row with eps > 0 gives zero blocks; rows are
    independent."""
    k = 8
    A, B = np.eye(8), np.tile(np.eye(4), (k, 1, 1))
    big = np.full(k, 40.0)
    X = np.full((2, 256), 3.25)
    X[1] *= -1
    r = O.rmsnorm_quant_act(X, np.ones(256), 0.0, A, B, big, big)
    codes = O.unpack_nibbles(r["codes"])
    assert (r["scales"] == 127 - 2).all()
    assert (codes[0] == 6).all() and (codes[1] == 14).all()
    w = WL.custom(6, 256, 16, 52, x_dtype="f32", with_w=False)
    g = np.random.default_rng(52).uniform(0.5, 1.5, 256)
    r1 = O.rmsnorm_quant_act(w.x, g, 0.0, w.A, w.B, w.alpha_min, w.alpha_max)
    r2 = O.rmsnorm_quant_act(w.x * 8.0, g, 0.0, w.A, w.B, w.alpha_min, w.alpha_max)
    np.testing.assert_array_equal(r1["codes"], r2["codes"])
    np.testing.assert_array_equal(r1["scales"], r2["scales"])
    Xz = w.x.copy()
    Xz[2] = 0.0
    rz = O.rmsnorm_quant_act(Xz, g, 1e-6, w.A, w.B, w.alpha_min, w.alpha_max)
    assert (rz["scales"][2] == 0).all() and (rz["codes"][2] == 0).all()
    np.testing.assert_array_equal(rz["codes"][[0, 1, 3, 4, 5]], O.rmsnorm_quant_act(
        w.x[[0, 1, 3, 4, 5]], g, 1e-6, w.A, w.B, w.alpha_min, w.alpha_max)["codes"])
