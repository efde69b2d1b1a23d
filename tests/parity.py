"""Parity rules shared by the GPU tests (CUDA path vs the CPU oracle).

Tolerances:
* transformed activations Y: |y_gpu - y_ref| <= 1e-5 * sum_j |x_j| |P_ji|
  (the condition-scaled reading of "within 1e-5 relative": a plain relative
  error is ill-posed for entries near cancellation);
* FP4 codes and E8M0 scales bit-exact, except elements whose pre-rounding value
  q lies within the Y tolerance 1e-5 * max(|y|, sum_j |x_j| |P_ji|), carried
  into scaled units (and never less than 1e-5 of q), of an E2M1 rounding
  boundary (midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5), values within the
  tolerance of zero (the sign of a zero code), and whole blocks whose clipped
  amax lies within the tolerance of a power of two (the shared exponent may
  flip); the mismatching elements must number fewer than 1e-4 of all elements.
  Weight codes use the condition scale of the fused weights,
  sum_j |w_j| |(P_i^-T)_ji|;
* GEMM: |out_gpu - out_ref| <= 1e-4 * sum_n |a_n| |w_n| against the oracle's
  fp64 product of the same codes.
* W4A8 (E4M3 codes): as for FP4, except that the band around each rounding
  boundary is the Y tolerance itself, 1e-5 * max(|y|, sum_j |x_j| |P_ji|),
  carried into scaled units (E4M3 boundaries are 1/16 apart down to the
  subnormals, so an element with cancellation can cross one within the fp32
  error of the transform).
* NVFP4 (E2M1 codes, E4M3 scale per 16): the same condition-scaled band around
  each E2M1 midpoint, carried into scaled units by the group's multiplier
  gs / scale; a whole group may differ in scale when amax * gs / 6 lies within
  the band of an E4M3 midpoint; for weights, whose gs the CUDA path derives from
  its own amax, the band also covers the relative difference of the two gs.
"""

from __future__ import annotations

import numpy as np

from oracle import batq_oracle as O

MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
REL = 1e-5


def condition_scale(X, A, B):
    """sum_j |x_j| |P_ji| per output element (fp64)."""
    X = np.abs(np.asarray(X, np.float64))
    S, N = X.shape
    k = N // 32
    P = np.abs(O.dense_blocks(A, B))
    return np.matmul(X.reshape(S, k, 32).transpose(1, 0, 2), P).transpose(1, 0, 2).reshape(S, N)


def check_y(y_gpu, X, A, B, y_ref):
    scale = condition_scale(X, A, B)
    err = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64))
    bad = err > REL * scale
    return int(bad.sum()), float(np.max(err / np.maximum(scale, 1e-300)))


def exempt_mask(ref, cond=None):
    """Boolean (S, N): elements whose code may legitimately differ.

    Without ``cond``: q within 1e-5 relative of a midpoint, blocks whose amax is
    within 1e-5 relative of a power of two.  With ``cond`` (the condition scale
    sum_j |x_j| |P_ji| of each element, for values that went through the
    transform): the band is the Y tolerance 1e-5 * max(|y|, cond) carried into
    scaled units, which also covers values with cancellation (|y| << cond),
    together with the sign of values within the tolerance of 0, and blocks
    whose amax lies within 1e-5 * max(amax, largest cond of the block) of a
    power of two.
    """
    q = np.abs(ref["q"])
    S, N = q.shape
    k = N // 32
    yh = np.abs(ref["Y_hat"].astype(np.float64))
    near_mid = np.zeros(q.shape, dtype=bool)
    if cond is None:
        for m in MIDPOINTS:
            near_mid |= np.abs(q - m) <= REL * m
    else:
        e = ref["scales"].astype(np.int64) - 127
        inv = np.repeat(np.exp2(-np.clip(e, -127, 127).astype(np.float64)), 32, axis=1)
        err_y = REL * np.maximum(yh, cond)
        band = np.maximum(err_y * inv, REL * q)
        for m in MIDPOINTS:
            near_mid |= np.abs(q - m) <= band
        near_mid |= yh <= err_y
    amax = yh.reshape(S, k, 32).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        p2 = np.exp2(np.round(np.log2(np.where(amax > 0, amax, 1.0))))
    tol = REL * p2 if cond is None else REL * np.maximum(p2, cond.reshape(S, k, 32).max(axis=2))
    near_pow2 = (amax > 0) & (np.abs(amax - p2) <= tol)
    return near_mid | np.repeat(near_pow2, 32, axis=1), near_pow2


def compare_codes(codes_gpu, scales_gpu_linear, ref, cond=None):
    """Returns dict(mismatch, unexplained, scale_mismatch, scale_unexplained, outside_literal,
    scale_outside_literal, total).

    ``unexplained`` counts mismatches outside the band in use (the condition-scaled band when
    ``cond`` is given); ``outside_literal`` counts mismatching elements outside the literal band
    of the stated tolerance (pre-rounding q within 1e-5 relative of an E2M1 midpoint, or a block
    amax within 1e-5 relative of a power of two), whatever band the test uses, so that the
    widening of that band for values with cancellation stays visible and bounded.
    """
    cg = O.unpack_nibbles(codes_gpu)
    cr = O.unpack_nibbles(ref["codes"])
    ex, ex_blk = exempt_mask(ref, cond)
    lit, lit_blk = exempt_mask(ref, None) if cond is not None else (ex, ex_blk)
    diff = cg != cr
    sdiff = np.asarray(scales_gpu_linear) != ref["scales"]
    S, N = cg.shape
    # every element of a block whose scale differs counts as mismatching
    diff_all = diff | np.repeat(sdiff, 32, axis=1)
    return {
        "mismatch": int(diff_all.sum()),
        "unexplained": int((diff_all & ~ex).sum()),
        "scale_mismatch": int(sdiff.sum()),
        "scale_unexplained": int((sdiff & ~ex_blk).sum()),
        "outside_literal": int((diff_all & ~lit).sum()),
        "scale_outside_literal": int((sdiff & ~lit_blk).sum()),
        "total": S * N,
    }


# Counts of every assert_quant_parity call of the session, by label (written out by conftest.py
# when BATQ_PARITY_REPORT names a file).
REPORT = {}


# Mismatches allowed outside the literal 1e-5-of-q band, as a fraction of the elements.  None for
# the GPK transforms of the workloads (every mismatch there lies within 1e-5 relative of an E2M1
# midpoint or of a power of two); the block Hadamard as P_i (every entry +-1/sqrt(32), so blocks
# cancel heavily) moves a few codes whose fp32 error, bounded by the condition scale, crosses a
# midpoint from further away: 1 of 64,000 and 4 of 2,097,152 elements on the test shapes.
LITERAL_LIMIT = 0.0
LITERAL_LIMIT_HADAMARD = 3e-5


def assert_quant_parity(codes_gpu, scales_gpu_linear, ref, label="", cond=None, literal_limit=LITERAL_LIMIT):
    """Codes and scales bit-exact outside the exemption band, exempt mismatches below 1e-4 of the
    elements, and mismatches outside the literal 1e-5-of-q band at most ``literal_limit`` of them."""
    r = compare_codes(codes_gpu, scales_gpu_linear, ref, cond)
    REPORT.setdefault(label, []).append(r)
    print(f"parity {label}: {r}")
    assert r["unexplained"] == 0 and r["scale_unexplained"] == 0, f"{label}: {r}"
    assert r["mismatch"] < 1e-4 * r["total"], f"{label}: too many boundary mismatches {r}"
    assert r["outside_literal"] <= literal_limit * r["total"], f"{label}: outside the literal band {r}"
    return r


def assert_gemm_parity(out_gpu, out_ref, T, label=""):
    out_gpu = np.asarray(out_gpu, np.float64)
    err = np.abs(out_gpu - out_ref)
    bad = err > 1e-4 * T
    assert not bad.any(), f"{label}: {int(bad.sum())} outputs out of tolerance, worst {np.max(err / np.maximum(T, 1e-300))}"
    return float(np.max(err / np.maximum(T, 1e-300)))


def to_mma_layout(scales_linear, rows, k, pad=0x7F):
    """Place a (rows, k) linear scale matrix into the tiled MMA layout buffer (test-side helper)."""
    buf = np.full(O.mma_layout_bytes(rows, k), pad, dtype=np.uint8)
    r, c = np.meshgrid(np.arange(rows), np.arange(k), indexing="ij")
    buf[O.mma_scale_offset(r, c, k)] = np.asarray(scales_linear, np.uint8)
    return buf


# ------------------------------------------------------- W4A8 (MXFP8 E4M3) ----

E4M3_MIDPOINTS = (O.E4M3_MAGNITUDE[:-1] + O.E4M3_MAGNITUDE[1:]) / 2


def exempt_mask_e4m3(ref, X, A, B):
    """Elements whose E4M3 code may legitimately differ from the oracle's.

    E4M3 has a rounding boundary every 1/16 (relative) all the way down to the
    subnormals, so an element whose transformed value suffers cancellation can
    cross one within the fp32 error of the transform, which is bounded relative
    to the condition scale sum_j |x_j| |P_ji|, not to |y|.  The band is therefore
    that of the Y tolerance: a code may differ if a midpoint of neighbouring E4M3
    magnitudes lies within 1e-5 * max(|y|, condition scale) * 2^-e of the
    oracle's pre-rounding value q.  Whole blocks may differ in scale when the
    clipped amax lies within 1e-5 * max(amax, largest condition scale of the
    block) of a power of two.
    """
    q = np.abs(ref["q"])
    S, N = q.shape
    k = N // 32
    cond = condition_scale(X, A, B)
    e = ref["scales"].astype(np.int64) - 127
    inv = np.repeat(np.exp2(-np.clip(e, -127, 127).astype(np.float64)), 32, axis=1)
    band = REL * np.maximum(np.abs(ref["Y_hat"].astype(np.float64)), cond) * inv
    idx = np.clip(np.searchsorted(E4M3_MIDPOINTS, q), 1, len(E4M3_MIDPOINTS) - 1)
    near = np.minimum(np.abs(q - E4M3_MIDPOINTS[idx - 1]), np.abs(q - E4M3_MIDPOINTS[idx]))
    near_mid = near <= band
    amax = np.abs(ref["Y_hat"].astype(np.float64)).reshape(S, k, 32).max(axis=2)
    cmax = cond.reshape(S, k, 32).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        p2 = np.exp2(np.round(np.log2(np.where(amax > 0, amax, 1.0))))
    near_pow2 = (amax > 0) & (np.abs(amax - p2) <= REL * np.maximum(p2, cmax))
    return near_mid | np.repeat(near_pow2, 32, axis=1), near_pow2


def assert_quant_parity_e4m3(codes_gpu, scales_gpu_linear, ref, X, A, B, label=""):
    """E4M3 codes and E8M0 scales bit-exact outside the exemptions; exempt mismatches < 1e-4."""
    ex, ex_blk = exempt_mask_e4m3(ref, X, A, B)
    diff = np.asarray(codes_gpu) != ref["codes"]
    sdiff = np.asarray(scales_gpu_linear) != ref["scales"]
    diff_all = diff | np.repeat(sdiff, 32, axis=1)
    r = {"mismatch": int(diff_all.sum()), "unexplained": int((diff_all & ~ex).sum()),
         "scale_unexplained": int((sdiff & ~ex_blk).sum()), "total": diff.size}
    assert r["unexplained"] == 0 and r["scale_unexplained"] == 0, f"{label}: {r}"
    assert r["mismatch"] < 1e-4 * r["total"], f"{label}: too many boundary mismatches {r}"
    return r


# ------------------------------------------------------------ NVFP4 output ----

def condition_scale_weights(W, A, B):
    """sum_j |w_j| |(P_i^-T)_ji| per fused weight element (fp64), from the oracle's dense inverses."""
    W = np.abs(np.asarray(W, np.float64))
    M, N = W.shape
    out = np.empty_like(W)
    for i in range(N // 32):
        pinv_t = O.gauss_jordan_inverse(O.kron_block(A[i] if np.ndim(A) == 3 else A, B[i])).T
        out[:, 32 * i:32 * (i + 1)] = W[:, 32 * i:32 * (i + 1)] @ np.abs(pinv_t)
    return out


def exempt_mask_nvfp4(ref, cond, gs_rel=0.0):
    """Elements (rows, N) and groups (rows, N/16) whose NVFP4 code / scale may differ from the oracle's.

    The CUDA path's transformed value differs from the oracle's by at most
    1e-5 * max(|y|, condition scale) (the Y tolerance), and its per-tensor gs
    (weights: derived from its own amax) by a relative gs_rel.  An element is
    exempt when an E2M1 midpoint lies within that error, carried into scaled
    units, of the oracle's q, or when |y| itself is within it of 0 (the sign of
    a zero code); a whole group is exempt when fp32(amax gs) / 6 lies within the
    error of its amax of an E4M3 midpoint (the group scale may flip).
    """
    yh = np.abs(ref["Y_hat"].astype(np.float64))
    rows, N = yh.shape
    q = np.abs(ref["q"])
    gs = ref["gs"]
    sval = O.e4m3_decode(ref["scales"])
    with np.errstate(divide="ignore", invalid="ignore"):
        mult = np.where(sval > 0, gs / np.where(sval > 0, sval, 1.0), 0.0)
    mult = np.repeat(np.nan_to_num(mult), 16, axis=1)
    err_y = REL * np.maximum(yh, cond)
    band = err_y * mult + 2.0 * gs_rel * q
    near = yh <= err_y
    for m in MIDPOINTS:
        near |= np.abs(q - m) <= band
    amax = yh.reshape(rows, N // 16, 16).max(axis=2)
    cmax = cond.reshape(rows, N // 16, 16).max(axis=2)
    u = amax * gs / 6.0
    band_u = REL * np.maximum(amax, cmax) * gs / 6.0 + 2.0 * gs_rel * u + 1e-300
    idx = np.clip(np.searchsorted(E4M3_MIDPOINTS, u), 1, len(E4M3_MIDPOINTS) - 1)
    du = np.minimum(np.abs(u - E4M3_MIDPOINTS[idx - 1]), np.abs(u - E4M3_MIDPOINTS[idx]))
    near_u = du <= band_u
    return near | np.repeat(near_u, 16, axis=1), near_u


def assert_quant_parity_nvfp4(codes_gpu, scales_gpu_linear, ref, cond, gs_rel=0.0, label=""):
    """Codes and E4M3 group scales bit-exact outside the exemptions; exempt mismatches < 1e-4."""
    ex, ex_grp = exempt_mask_nvfp4(ref, cond, gs_rel)
    diff = O.unpack_nibbles(codes_gpu) != O.unpack_nibbles(ref["codes"])
    sdiff = np.asarray(scales_gpu_linear) != ref["scales"]
    diff_all = diff | np.repeat(sdiff, 16, axis=1)
    r = {"mismatch": int(diff_all.sum()), "unexplained": int((diff_all & ~ex).sum()),
         "scale_mismatch": int(sdiff.sum()), "scale_unexplained": int((sdiff & ~ex_grp).sum()),
         "total": diff.size}
    assert r["unexplained"] == 0 and r["scale_unexplained"] == 0, f"{label}: {r}"
    assert r["mismatch"] < 1e-4 * r["total"], f"{label}: too many boundary mismatches {r}"
    return r
