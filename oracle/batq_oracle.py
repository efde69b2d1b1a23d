"""CPU oracle for the BATQuant W4A4 MXFP4 linear path -- TEST INFRASTRUCTURE ONLY.

This is a plain, slow, obviously-correct restatement of what the path
computes, written from the method's description.  It shares no code with the
CUDA library and imports nothing from it.  Only the test suite, the smoke
check and the benchmark's CPU-baseline / reference arm may import it; the
product path never calls it.

Sources (BATQuant: Outlier-resilient MXFP4 Quantization via Learnable
Block-wise Optimization, arXiv 2603.16590), cited by page and section:

* [p1] zhaoyang97.github.io daily-arxiv summary, sections "块仿射变换 (BAT)",
  "Global-Private Kronecker (GPK) 分解", "块级可学习裁剪".
* [p2] gist.science technical summary ("Résumé Technique"), §2.A-§2.D.
* [p3] thelatestinai.com page: abstract, Figure 2 and Figure 3 captions,
  Table 1.
* MXFP4 element / scale rules: OCP Microscaling Formats (MX) v1.0 (E8M0 shared
  scale 2^(floor(log2 amax) - emax_elem), emax_elem = 2 for E2M1; E2M1 elements
  rounded to nearest even and saturated at +-6).  The pages state only that 32
  elements share one E8M0 scale (p3, DuQuant++ abstract) and that values are
  divided by the scale before rounding (p3, Figure 2 caption).

Readings taken where the pages are silent (each is listed with its reason in
the design notes):

* A 32-element block x is reshaped row-major to X in R^{4x8}; with the
  row-vector convention of Table 1 ("XP") the block transform is
  y = x . P_i with P_i = B_i (x) A (4x4 private B_i, 8x8 global A).
* Clip after the transform, with per-block-column ratios sigma(alpha) computed
  in fp64 and rounded to fp32 once; min/max are per token and block.
* lo > hi: clamp(y, lo, hi) = min(max(y, lo), hi), so hi wins.
* All-zero block: scale byte 0x00, codes 0.  Any non-finite transformed value
  in a block: scale byte 0xFF, codes 0.
* An exact-zero transformed value is +0 (a sum has no sign of its own).
* Two E2M1 codes per byte, element 2j in the low nibble; code = sign<<3 | mag.
* Weights: W' = W . P^{-T} per block, from the fp64 Gauss-Jordan inverse of
  the dense 32x32 P_i, rounded to fp32, then MXFP4 round-to-nearest along K
  without clipping.

W4A8 variant (the pages' second main setting, MXFP8 activations against the
MXFP4 weights; p3 abstract and Table 2):

* E4M3 elements (bias 7, 3 mantissa bits, subnormals m * 2^-9, largest 448),
  shared scale 2^(floor(log2 amax) - 8) (OCP MX v1.0, emax_elem = 8), round to
  nearest even, and magnitudes above 448 saturate to 448 (the scaled amax lies
  in [256, 512), so the largest elements of a block can saturate; OCP leaves
  overflow to the implementation, and saturation is the reading taken).
* The same clip, zero-block and non-finite rules as MXFP4.
* The MXFP4 weights are consumed from one-byte E4M3 containers that hold the
  same E2M1 values exactly (every E2M1 value is an E4M3 value).

NVFP4 output variant (format named on the ARCQuant page: 16 E2M1 elements
share one E4M3 scale; the pages give no other rule, so these are readings):

* The transform and the clip stay on 32-element blocks (the method's own
  granularity); each clipped block is then stored as two 16-element groups.
* Per-tensor fp32 encode scale gs (decoded value = code * scale / gs), as the
  block-scaled FP4 tensor-core GEMM consumes only the group scales and applies
  a per-tensor factor afterwards; gs = 1 is the format with no tensor scale.
  For weights gs = fp32(448 * 6 / amax of the fused fp32 weights).
* Group scale = E4M3 of fp32(fp32(amax * gs) / 6), nearest even, saturating at
  448; element q = fp32(v * fp32(gs / scale)) (0 multiplier for a zero scale),
  then the E2M1 table.  All steps are fp32 operations so that the CUDA path
  can take the same decisions in the same precision.
* A non-finite 32-block gives scale byte 0x7F (E4M3 NaN) to both groups and
  zero codes.
* GEMM: out = fp32(1 / fp32(gs_a * gs_w)) * sum (code_a s_a)(code_w s_w).

Naive Kronecker (Table 1's middle row, [p3]): one 8x8 A_i per block instead of
the shared A, P_i = B_i (x) A_i; every function that takes A accepts either
shape (8, 8) or (k, 8, 8).

KV cache (the pages' KV8 / KV4 settings): new key or value rows (kv_heads x
head_dim elements per token) take the same transform, clip and MXFP4 / MXFP8
encoding and are written to the cache rows a slot mapping names; negative slots
are skipped.  The attention side is not part of the path.

RMSNorm fused ahead of the transform (a reading of the ARCQuant page's fused
reorder -> RMSNorm -> quantise kernel applied to this path): z = x / sqrt(mean
over the token of x^2 + eps) * gamma in fp64, not rounded before the transform.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, brute force and the pages' Table 1.
"""

from __future__ import annotations

import numpy as np

G = 32  # MXFP block size g [p3 Table 1 caption]
G1 = 8  # size of the global factor A [p3 Table 1 caption; p1 GPK]
G2 = 4  # size of the private factor B_i [p3 Table 1 caption; p1 GPK]

# E2M1 magnitudes for magnitude codes 0..7 (OCP MX v1.0, FP4 E2M1: bias 1,
# subnormal 0.5 at exponent 0).
E2M1_MAGNITUDE = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)

# Round-to-nearest-even decision table on |q| (q = value / scale).  Each row
# is (upper bound, bound included?, magnitude code); the first row whose bound
# admits |q| gives the code.  Bounds are the midpoints between neighbouring
# magnitudes; a midpoint belongs to the neighbour with an even code (mantissa
# bit 0).  Anything above 5 rounds to 6, which also saturates (6, 8) -> 6.
E2M1_RNE_TABLE = (
    (0.25, True, 0),
    (0.75, False, 1),
    (1.25, True, 2),
    (1.75, False, 3),
    (2.5, True, 4),
    (3.5, False, 5),
    (5.0, True, 6),
    (np.inf, True, 7),
)


# ---------------------------------------------------------------------------
# Table 1: parameter counts of the transform P for each decomposition
# ---------------------------------------------------------------------------

def param_counts(N: int, g: int = G, g1: int = G1, g2: int = G2) -> dict:
    """Number of stored parameters of P under each decomposition [p3 Table 1].

    Counted from the shapes of the arrays each decomposition stores:
    FlatQuant stores two sqrt(N) x sqrt(N) Kronecker factors (2N in Table 1);
    "w/o" stores k dense g x g blocks; naive Kronecker stores an
    8x8 and a 4x4 factor per block; GPK stores one shared 8x8 A and one 4x4
    B_i per block.
    """
    k = N // g
    n_side = int(round(np.sqrt(N)))
    flat_1 = np.zeros((n_side, n_side))
    flat_2 = np.zeros((n_side, n_side))
    dense_blocks = np.zeros((k, g, g))
    naive_A = np.zeros((k, g1, g1))
    naive_B = np.zeros((k, g2, g2))
    gpk_A = np.zeros((g1, g1))
    gpk_B = np.zeros((k, g2, g2))
    return {
        "flatquant": flat_1.size + flat_2.size,
        "wo": dense_blocks.size,
        "naive_kronecker": naive_A.size + naive_B.size,
        "gpk": gpk_A.size + gpk_B.size,
    }


# ---------------------------------------------------------------------------
# Block-wise affine transform with the GPK decomposition
# ---------------------------------------------------------------------------

def kron_block(A: np.ndarray, Bi: np.ndarray) -> np.ndarray:
    """Dense P_i = B_i (x) A, 32x32 in fp64, built entry by entry [p1 GPK; p2 §2.B].

    P_i[8r + a, 8c + b] = B_i[r, c] * A[a, b].
    """
    A = np.asarray(A, dtype=np.float64)
    Bi = np.asarray(Bi, dtype=np.float64)
    P = np.zeros((G, G), dtype=np.float64)
    for r in range(G2):
        for c in range(G2):
            for a in range(G1):
                for b in range(G1):
                    P[G1 * r + a, G1 * c + b] = Bi[r, c] * A[a, b]
    return P


def dense_blocks(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """All k dense blocks P_i = B_i (x) A, shape (k, 32, 32), fp64 [p1 BAT: P = diag(P_1..P_k)].

    Same entry-by-entry rule as ``kron_block``, applied to every block at once.
    ``A`` is either the shared 8x8 factor (GPK) or one 8x8 factor per block,
    shape (k, 8, 8): P_i = B_i (x) A_i, the "naive Kronecker" row of Table 1 [p3].
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    k = B.shape[0]
    Ak = A if A.ndim == 3 else np.broadcast_to(A, (k, G1, G1))
    P = np.zeros((k, G, G), dtype=np.float64)
    for r in range(G2):
        for c in range(G2):
            for a in range(G1):
                for b in range(G1):
                    P[:, G1 * r + a, G1 * c + b] = B[:, r, c] * Ak[:, a, b]
    return P


def transform_f64(X: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """y_i = x_i . P_i for every token and block, in fp64 (no rounding) [p3 Table 1 "XP"; p1 BAT]."""
    X = np.asarray(X, dtype=np.float64)
    S, N = X.shape
    k = N // G
    P = dense_blocks(A, B)
    Xb = X.reshape(S, k, G).transpose(1, 0, 2)  # (k, S, 32)
    Y = np.matmul(Xb, P)  # (k, S, 32): row vector times P_i
    return Y.transpose(1, 0, 2).reshape(S, N)


def transform(X: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Transformed activations, computed in fp64 and rounded to fp32 once.

    Exact zeros are returned as +0.
    """
    Y = transform_f64(X, A, B) + 0.0
    return Y.astype(np.float32)


# ---------------------------------------------------------------------------
# Block-wise learnable clipping
# ---------------------------------------------------------------------------

def clip_ratios(alpha: np.ndarray) -> np.ndarray:
    """sigma(alpha) = 1 / (1 + exp(-alpha)) in fp64, rounded to fp32 [p1 块级可学习裁剪; p2 §2.C]."""
    a = np.asarray(alpha, dtype=np.float64)
    return (1.0 / (1.0 + np.exp(-a))).astype(np.float32)


def clip_blocks(Y: np.ndarray, r_min: np.ndarray, r_max: np.ndarray):
    """x_hat = clip(y, sigma(a_min) * min(y), sigma(a_max) * max(y)) per token and block [p1 块级可学习裁剪].

    ``Y`` is fp32 (S, N); ``r_min``/``r_max`` are the fp32 ratios per block
    column.  Returns (Y_hat fp32 (S, N), lo (S, k), hi (S, k), nonfinite (S, k)).
    lo and hi are single-rounded fp32 products.
    """
    Y = np.asarray(Y, dtype=np.float32)
    S, N = Y.shape
    k = N // G
    Yb = Y.reshape(S, k, G)
    nonfinite = ~np.all(np.isfinite(Yb), axis=2)
    with np.errstate(invalid="ignore"):
        mn = Yb.min(axis=2)
        mx = Yb.max(axis=2)
        lo = (np.asarray(r_min, np.float64)[None, :] * mn.astype(np.float64)).astype(np.float32)
        hi = (np.asarray(r_max, np.float64)[None, :] * mx.astype(np.float64)).astype(np.float32)
        Yh = np.minimum(np.maximum(Yb, lo[:, :, None]), hi[:, :, None])
    return Yh.reshape(S, N).astype(np.float32), lo, hi, nonfinite


# ---------------------------------------------------------------------------
# MXFP4: shared E8M0 scale and E2M1 elements
# ---------------------------------------------------------------------------

def e8m0_exponent(amax: np.ndarray) -> np.ndarray:
    """Shared-scale exponent e = floor(log2 amax) - 2, clamped to [-127, 127] (OCP MX v1.0).

    amax == 0 gives -127.  Uses frexp (amax = m * 2^ex with m in [0.5, 1), so
    floor(log2 amax) = ex - 1), exact for every finite fp32 value.
    """
    a = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1 - 2
    e = np.where(a == 0.0, -127, e)
    return np.clip(e, -127, 127)


def e2m1_encode(q: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes of q (already divided by the shared scale) by table lookup [p3 Figure 2 caption].

    The sign bit (bit 3) is the sign of q, so negative values that round to 0
    keep the sign (code 0x8).
    """
    q = np.asarray(q, dtype=np.float64)
    mag = np.abs(q)
    code = np.full(q.shape, -1, dtype=np.int64)
    for bound, inclusive, c in E2M1_RNE_TABLE:
        hit = (mag <= bound) if inclusive else (mag < bound)
        code = np.where((code < 0) & hit, c, code)
    sign = np.signbit(q).astype(np.int64)
    return (sign << 3) | code


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each 4-bit code."""
    codes = np.asarray(codes, dtype=np.int64)
    mag = np.asarray(E2M1_MAGNITUDE, dtype=np.float64)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """(rows, N) 4-bit codes -> (rows, N/2) bytes; element 2j in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """(rows, N/2) bytes -> (rows, N) 4-bit codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, 2 * half), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def mxfp4_quantize(V: np.ndarray, nonfinite: np.ndarray | None = None):
    """MXFP4 of fp32 rows V (rows, N): per 32-block scale, divide, round [p3 Figure 2 caption; OCP MX].

    Returns (packed codes (rows, N/2) uint8, scale bytes (rows, N/32) uint8,
    q (rows, N) fp64 = V / 2^e before rounding).
    """
    V = np.asarray(V, dtype=np.float32)
    rows, N = V.shape
    k = N // G
    Vb = V.reshape(rows, k, G).astype(np.float64)
    if nonfinite is None:
        nonfinite = ~np.all(np.isfinite(Vb), axis=2)
    with np.errstate(invalid="ignore"):
        amax = np.abs(Vb).max(axis=2)
    amax = np.where(nonfinite, 0.0, amax)
    e = e8m0_exponent(amax)
    q = Vb * np.exp2(-e.astype(np.float64))[:, :, None]  # exact: power-of-two scaling in fp64
    q = np.where(nonfinite[:, :, None], 0.0, q)
    codes = e2m1_encode(q)
    scale = (e + 127).astype(np.int64)
    scale = np.where(nonfinite, 0xFF, scale).astype(np.uint8)
    return pack_nibbles(codes.reshape(rows, N)), scale, q.reshape(rows, N)


def dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 values code * 2^(byte - 127); byte 0xFF decodes to NaN."""
    codes = unpack_nibbles(packed)
    rows, N = codes.shape
    k = N // G
    vals = e2m1_decode(codes).reshape(rows, k, G)
    s = np.asarray(scales, dtype=np.int64)
    factor = np.where(s == 0xFF, np.nan, np.exp2((s - 127).astype(np.float64)))
    return (vals * factor[:, :, None]).reshape(rows, N)


# ---------------------------------------------------------------------------
# Scale-factor layout consumed by the block-scaled tensor-core MMA
# ---------------------------------------------------------------------------

def mma_scale_offset(row: np.ndarray, kb: np.ndarray, k: int) -> np.ndarray:
    """Byte offset of scale (row, block column kb) in the 128x4 tiled layout.

    Tiles of 128 rows x 4 block columns (512 bytes) are stored row-tile major;
    inside a tile, row r and column c sit at (r % 32) * 16 + (r // 32) * 4 + c.
    """
    kpad = -(-k // 4) * 4
    row = np.asarray(row, dtype=np.int64)
    kb = np.asarray(kb, dtype=np.int64)
    return ((row // 128) * (kpad // 4) + kb // 4) * 512 + (row % 32) * 16 + ((row // 32) % 4) * 4 + kb % 4


def scales_from_mma_layout(buf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Read a (rows, k) LINEAR scale matrix back out of the tiled layout buffer."""
    r, c = np.meshgrid(np.arange(rows), np.arange(k), indexing="ij")
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[mma_scale_offset(r, c, k)]


def mma_layout_bytes(rows: int, k: int) -> int:
    return (-(-rows // 128) * 128) * (-(-k // 4) * 4)


# ---------------------------------------------------------------------------
# Online activation side: transform + clip + MXFP4 [p2 §2.D; p3 Figure 3 caption]
# ---------------------------------------------------------------------------

def quant_act(X, A, B, alpha_min, alpha_max) -> dict:
    """Online activation path for one linear: y = x P_i, clip, MXFP4.

    Returns a dict with Y (fp32 transformed), Y_hat (clipped), codes
    (S, N/2), scales (S, k) linear, q (fp64 pre-rounding), nonfinite (S, k).
    """
    Y = transform(X, A, B)
    r_min = clip_ratios(alpha_min)
    r_max = clip_ratios(alpha_max)
    Yh, lo, hi, nonfinite = clip_blocks(Y, r_min, r_max)
    codes, scales, q = mxfp4_quantize(Yh, nonfinite)
    return {"Y": Y, "Y_hat": Yh, "codes": codes, "scales": scales, "q": q,
            "nonfinite": nonfinite, "lo": lo, "hi": hi}


def encode_from_transformed(Y, r_min, r_max) -> dict:
    """Clip + MXFP4 starting from already-transformed fp32 values (steps after the transform)."""
    Yh, lo, hi, nonfinite = clip_blocks(Y, r_min, r_max)
    codes, scales, q = mxfp4_quantize(Yh, nonfinite)
    return {"Y_hat": Yh, "codes": codes, "scales": scales, "q": q, "nonfinite": nonfinite}


# ---------------------------------------------------------------------------
# Offline weight side [p1 (weights fused offline); p2 §2.D; p3 Figure 3 caption]
# ---------------------------------------------------------------------------

def gauss_jordan_inverse(P: np.ndarray) -> np.ndarray:
    """Inverse of a square matrix by Gauss-Jordan elimination with partial pivoting, fp64."""
    P = np.array(P, dtype=np.float64)
    n = P.shape[0]
    aug = np.concatenate([P, np.eye(n)], axis=1)
    for col in range(n):
        piv = col + int(np.argmax(np.abs(aug[col:, col])))
        if aug[piv, col] == 0.0:
            raise np.linalg.LinAlgError("singular block transform")
        if piv != col:
            aug[[col, piv]] = aug[[piv, col]]
        aug[col] = aug[col] / aug[col, col]
        for row in range(n):
            if row != col:
                aug[row] = aug[row] - aug[row, col] * aug[col]
    return aug[:, n:]


def fuse_weights_f64(W: np.ndarray, A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """W' = W . P^{-T} block by block, fp64: (x P)(P^{-1} W^T) = x W^T."""
    W = np.asarray(W, dtype=np.float64)
    M, N = W.shape
    k = N // G
    out = np.empty_like(W)
    for i in range(k):
        Pinv = gauss_jordan_inverse(kron_block(A[i] if np.ndim(A) == 3 else A, B[i]))
        out[:, G * i:G * (i + 1)] = W[:, G * i:G * (i + 1)] @ Pinv.T
    return out


def prepare_weights(W, A, B) -> dict:
    """Fused weights rounded to fp32, then MXFP4 round-to-nearest along K (no clip)."""
    Wf = fuse_weights_f64(W, A, B).astype(np.float32)
    codes, scales, q = mxfp4_quantize(Wf)
    return {"W_fused": Wf, "codes": codes, "scales": scales, "q": q}


# ---------------------------------------------------------------------------
# W4A4 block-scaled GEMM
# ---------------------------------------------------------------------------

def gemm(a_codes, a_scales, w_codes, w_scales):
    """out[s, m] = sum_n deq(a)[s, n] * deq(w)[m, n] in fp64, plus T = sum |a||w| (tolerance scale)."""
    Da = dequantize(a_codes, a_scales)
    Dw = dequantize(w_codes, w_scales)
    out = Da @ Dw.T
    T = np.abs(Da) @ np.abs(Dw).T
    return out, T


def gemm_rows(a_codes, a_scales, w_codes, w_scales, rows, cols=None):
    """Sampled outputs: only rows ``rows`` (and optionally columns ``cols``) of the fp64 GEMM."""
    Da = dequantize(a_codes[rows], a_scales[rows])
    if cols is None:
        Dw = dequantize(w_codes, w_scales)
    else:
        Dw = dequantize(w_codes[cols], w_scales[cols])
    return Da @ Dw.T, np.abs(Da) @ np.abs(Dw).T


def linear(X, A, B, alpha_min, alpha_max, W):
    """Whole W4A4 linear: activation path, weight preparation, GEMM."""
    act = quant_act(X, A, B, alpha_min, alpha_max)
    wp = prepare_weights(W, A, B)
    out, T = gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    return out, T, act, wp


# ---------------------------------------------------------------------------
# W4A8 variant: MXFP8 (E4M3) activations against the MXFP4 weights
# [p3 abstract and Table 2 (W4A8 rows); OCP MX v1.0 for FP8 E4M3]
# ---------------------------------------------------------------------------

def _e4m3_magnitudes() -> np.ndarray:
    """Values of the 127 finite non-negative E4M3 codes 0x00..0x7E (0x7F is NaN).

    Exponent bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
    m * 2^-9.  The largest value is 1.75 * 2^8 = 448.
    """
    vals = []
    for c in range(0x7F):
        ex, m = c >> 3, c & 7
        vals.append(m * 2.0 ** -9 if ex == 0 else (1.0 + m / 8.0) * 2.0 ** (ex - 7))
    return np.asarray(vals, dtype=np.float64)


E4M3_MAGNITUDE = _e4m3_magnitudes()
E4M3_MAX = 448.0
E4M3_EMAX = 8  # exponent of the largest normal (OCP MX v1.0: emax_elem for E4M3)


def e8m0_exponent_e4m3(amax: np.ndarray) -> np.ndarray:
    """Shared-scale exponent for E4M3 elements: floor(log2 amax) - 8, clamped to [-127, 127]."""
    a = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1 - E4M3_EMAX
    e = np.where(a == 0.0, -127, e)
    return np.clip(e, -127, 127)


def e4m3_encode(q: np.ndarray) -> np.ndarray:
    """8-bit E4M3 codes of q by round-to-nearest-even over the value table, saturating at +-448.

    For each |q| the two neighbouring table entries are found; the nearer one
    wins, and an exact midpoint goes to the even code (mantissa bit 0).
    Magnitudes above 448 give 448 (no NaN is produced).  The sign bit (bit 7)
    is the sign of q, so negative values that round to zero give 0x80.
    """
    q = np.asarray(q, dtype=np.float64)
    mag = np.minimum(np.abs(q), E4M3_MAX)
    hi = np.searchsorted(E4M3_MAGNITUDE, mag, side="left")  # first entry >= mag
    hi = np.clip(hi, 0, len(E4M3_MAGNITUDE) - 1)
    lo = np.clip(hi - 1, 0, len(E4M3_MAGNITUDE) - 1)
    d_lo = mag - E4M3_MAGNITUDE[lo]
    d_hi = E4M3_MAGNITUDE[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag == E4M3_MAGNITUDE[hi], hi, code)
    sign = np.signbit(q).astype(np.int64)
    return (sign << 7) | code


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each finite 8-bit E4M3 code (0x7F / 0xFF would be NaN; never produced here)."""
    codes = np.asarray(codes, dtype=np.int64)
    mag = E4M3_MAGNITUDE[np.minimum(codes & 0x7F, 0x7E)]
    mag = np.where((codes & 0x7F) == 0x7F, np.nan, mag)
    return np.where(codes & 0x80, -mag, mag)


def mxfp8_quantize(V: np.ndarray, nonfinite: np.ndarray | None = None):
    """MXFP8 (E4M3) of fp32 rows V: per 32-block scale 2^(floor(log2 amax) - 8), divide, round.

    Returns (codes (rows, N) uint8, scale bytes (rows, N/32) uint8, q (rows, N)
    fp64 before rounding).  A block with a non-finite value gets scale 0xFF and
    zero codes, as in the MXFP4 path.
    """
    V = np.asarray(V, dtype=np.float32)
    rows, N = V.shape
    k = N // G
    Vb = V.reshape(rows, k, G).astype(np.float64)
    if nonfinite is None:
        nonfinite = ~np.all(np.isfinite(Vb), axis=2)
    with np.errstate(invalid="ignore"):
        amax = np.abs(Vb).max(axis=2)
    amax = np.where(nonfinite, 0.0, amax)
    e = e8m0_exponent_e4m3(amax)
    q = Vb * np.exp2(-e.astype(np.float64))[:, :, None]  # exact: power-of-two scaling in fp64
    q = np.where(nonfinite[:, :, None], 0.0, q)
    codes = e4m3_encode(q).reshape(rows, N)
    codes = np.where(np.repeat(nonfinite, G, axis=1), 0, codes).astype(np.uint8)
    scale = np.where(nonfinite, 0xFF, e + 127).astype(np.uint8)
    return codes, scale, q.reshape(rows, N)


def dequantize_e4m3(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 values code * 2^(byte - 127) for (rows, N) E4M3 codes; byte 0xFF decodes to NaN."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows, N = codes.shape
    k = N // G
    vals = e4m3_decode(codes).reshape(rows, k, G)
    s = np.asarray(scales, dtype=np.int64)
    factor = np.where(s == 0xFF, np.nan, np.exp2((s - 127).astype(np.float64)))
    return (vals * factor[:, :, None]).reshape(rows, N)


def quant_act_mxfp8(X, A, B, alpha_min, alpha_max) -> dict:
    """Online activation path of the W4A8 variant: y = x P_i, the same clip, MXFP8 (E4M3)."""
    Y = transform(X, A, B)
    Yh, lo, hi, nonfinite = clip_blocks(Y, clip_ratios(alpha_min), clip_ratios(alpha_max))
    codes, scales, q = mxfp8_quantize(Yh, nonfinite)
    return {"Y": Y, "Y_hat": Yh, "codes": codes, "scales": scales, "q": q,
            "nonfinite": nonfinite, "lo": lo, "hi": hi}


def e4m3_containers_from_e2m1(packed: np.ndarray) -> np.ndarray:
    """(rows, N/2) packed E2M1 codes -> (rows, N) E4M3 bytes holding the same values (exact)."""
    return e4m3_encode(e2m1_decode(unpack_nibbles(packed))).astype(np.uint8)


def gemm_w4a8(a_codes8, a_scales, w_codes8, w_scales):
    """out = deq(a) deq(w)^T in fp64 for E4M3 activation and weight codes, plus T = sum |a||w|."""
    Da = dequantize_e4m3(a_codes8, a_scales)
    Dw = dequantize_e4m3(w_codes8, w_scales)
    return Da @ Dw.T, np.abs(Da) @ np.abs(Dw).T


# ---------------------------------------------------------------------------
# NVFP4 output variant: 16-element groups sharing one E4M3 scale
# [ARCQuant page (zhihu-style summary), section "背景：为什么 W4A4 在 NVFP4 上很难":
#  every 16 E2M1 elements share one E4M3 scale factor]
# ---------------------------------------------------------------------------

NV_G = 16                 # elements per NVFP4 scale group
NV_SCALE_NAN = 0x7F       # E4M3 NaN: scale byte of a group whose 32-block is non-finite
NV_GLOBAL_NUMERATOR = 448.0 * 6.0  # largest E4M3 scale x largest E2M1 magnitude


def f32(v):
    """Round fp64 values to fp32 (one IEEE round-to-nearest-even).

    Every fp32 operation below is written as the exact (or fp64) result
    rounded once to fp32.  A product of two fp32 values is exact in fp64; for
    a quotient, fp64 rounding followed by fp32 rounding equals the correctly
    rounded fp32 quotient because 53 >= 2 * 24 + 2 (double rounding is
    innocuous for one operation in that case).
    """
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def nvfp4_group_scale(amax, gs):
    """E4M3 scale byte, its value, and the element multiplier of 16-element groups.

    amax: clipped group amax (fp32 values); gs: per-tensor fp32 encode scale
    (decoded tensor = code * scale / gs).  Steps, each rounded to fp32:
    t = amax * gs, u = t / 6, scale = E4M3(u) (nearest even, saturating at 448),
    multiplier = gs / scale (0 when the scale is 0).
    """
    amax = np.asarray(amax, dtype=np.float64)
    gs = float(np.float32(gs))
    t = f32(amax * gs)
    u = f32(t / 6.0)
    byte = e4m3_encode(u).astype(np.int64)            # u >= 0: sign bit clear
    sval = e4m3_decode(byte)
    with np.errstate(divide="ignore"):
        mult = np.where(sval == 0.0, 0.0, f32(gs / np.where(sval == 0.0, 1.0, sval)))
    return byte, sval, mult


def nvfp4_quantize(V: np.ndarray, gs: float = 1.0, nonfinite: np.ndarray | None = None):
    """NVFP4 of fp32 rows V (rows, N): 16-element groups, E4M3 scale, E2M1 codes.

    Each element: q = fp32(v * multiplier), then the E2M1 table (nearest even,
    saturating at 6, sign kept on zero).  ``nonfinite`` flags 32-element
    blocks (rows, N/32) holding a non-finite value: both of their groups get
    scale byte 0x7F and codes 0.  Returns (packed codes (rows, N/2), scale
    bytes (rows, N/16) uint8, q (rows, N) fp64).
    """
    V = np.asarray(V, dtype=np.float32)
    rows, N = V.shape
    k16 = N // NV_G
    Vg = V.reshape(rows, k16, NV_G).astype(np.float64)
    if nonfinite is None:
        nonfinite = ~np.all(np.isfinite(V.reshape(rows, N // G, G)), axis=2)
    nf16 = np.repeat(nonfinite, G // NV_G, axis=1)
    with np.errstate(invalid="ignore"):
        amax = np.abs(Vg).max(axis=2)
    amax = np.where(nf16, 0.0, amax)
    byte, _, mult = nvfp4_group_scale(amax, gs)
    with np.errstate(invalid="ignore"):
        q = f32(Vg * mult[:, :, None])
    q = np.where(nf16[:, :, None], 0.0, q)
    codes = e2m1_encode(q).reshape(rows, N)
    codes = np.where(np.repeat(nf16, NV_G, axis=1), 0, codes)
    scale = np.where(nf16, NV_SCALE_NAN, byte).astype(np.uint8)
    return pack_nibbles(codes), scale, q.reshape(rows, N)


def dequantize_nvfp4(packed: np.ndarray, scales: np.ndarray, gs: float = 1.0) -> np.ndarray:
    """fp64 values code * E4M3(scale) / gs; a 0x7F scale decodes to NaN."""
    codes = unpack_nibbles(packed)
    rows, N = codes.shape
    vals = e2m1_decode(codes).reshape(rows, N // NV_G, NV_G)
    sval = e4m3_decode(np.asarray(scales, dtype=np.int64))
    return (vals * sval[:, :, None]).reshape(rows, N) / float(np.float32(gs))


def quant_act_nvfp4(X, A, B, alpha_min, alpha_max, gs: float = 1.0) -> dict:
    """Online activation path with NVFP4 output: y = x P_i and the clip on 32-blocks, then NVFP4."""
    Y = transform(X, A, B)
    Yh, lo, hi, nonfinite = clip_blocks(Y, clip_ratios(alpha_min), clip_ratios(alpha_max))
    codes, scales, q = nvfp4_quantize(Yh, gs, nonfinite)
    return {"Y": Y, "Y_hat": Yh, "codes": codes, "scales": scales, "q": q,
            "nonfinite": nonfinite, "lo": lo, "hi": hi, "gs": float(np.float32(gs))}


def nvfp4_global_scale(amax: float) -> float:
    """Per-tensor encode scale fp32(448 * 6 / amax), 1 for an all-zero (or too small) tensor."""
    a = float(np.float32(amax))
    if not a > 0.0:
        return 1.0
    g = float(f32(NV_GLOBAL_NUMERATOR / a))
    return g if np.isfinite(g) else 1.0


def prepare_weights_nvfp4(W, A, B) -> dict:
    """Fused weights rounded to fp32, per-tensor scale from their amax, NVFP4 along K (no clip)."""
    Wf = fuse_weights_f64(W, A, B).astype(np.float32)
    gs = nvfp4_global_scale(np.max(np.abs(Wf)))
    codes, scales, q = nvfp4_quantize(Wf, gs)
    return {"W_fused": Wf, "codes": codes, "scales": scales, "q": q, "gs": gs}


def nvfp4_alpha(gs_a: float, gs_w: float) -> float:
    """Epilogue factor fp32(1 / fp32(gs_a * gs_w)) undoing both per-tensor scales."""
    return float(f32(1.0 / f32(float(np.float32(gs_a)) * float(np.float32(gs_w)))))


def gemm_nvfp4(a_codes, a_scales, w_codes, w_scales, alpha: float = 1.0):
    """out = alpha * sum_n (code_a s_a)(code_w s_w) in fp64, plus T = |alpha| sum |a||w|."""
    Da = dequantize_nvfp4(a_codes, a_scales)
    Dw = dequantize_nvfp4(w_codes, w_scales)
    al = float(np.float32(alpha))
    return al * (Da @ Dw.T), abs(al) * (np.abs(Da) @ np.abs(Dw).T)


# ---------------------------------------------------------------------------
# BAT on the KV cache: new key / value rows quantised into a paged cache
# [thelatestinai.com BATQuant page, Table 2 caption (W4A8KV8, W4A8KV4);
#  gist.science summary, section 2.D (the transforms also cover the KV cache)]
# ---------------------------------------------------------------------------

def quant_kv_cache(X, A, B, alpha_min, alpha_max, slots, cache_codes, cache_scales, kv_format="mxfp4"):
    """Transform, clip and MXFP4 (KV4) or MXFP8 (KV8) of new rows X, written into copies of the cache.

    Row r of X goes to cache row slots[r]; a slot below 0 or past the cache is skipped, and rows the
    mapping does not name keep their contents.  Returns (codes, scales, the per-token result).
    """
    act = quant_act(X, A, B, alpha_min, alpha_max) if kv_format == "mxfp4" else \
        quant_act_mxfp8(X, A, B, alpha_min, alpha_max)
    codes = np.array(cache_codes, dtype=np.uint8, copy=True)
    scales = np.array(cache_scales, dtype=np.uint8, copy=True)
    n = codes.shape[0]
    for r, s in enumerate(np.asarray(slots).tolist()):
        if 0 <= s < n:
            codes[s] = act["codes"][r]
            scales[s] = act["scales"][r]
    return codes, scales, act


# ---------------------------------------------------------------------------
# RMSNorm ahead of the transform (the normalisation before each linear; the
# ARCQuant page's fused kernel runs reorder -> RMSNorm -> quantise in one pass)
# ---------------------------------------------------------------------------

def rmsnorm(X, gamma, eps: float):
    """Per token: z = x / sqrt(mean(x^2) + eps) * gamma, in fp64 (no intermediate rounding)."""
    X = np.asarray(X, dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64)
    ms = np.mean(X * X, axis=1, keepdims=True)
    return X / np.sqrt(ms + float(eps)) * g[None, :]


def rmsnorm_quant_act(X, gamma, eps, A, B, alpha_min, alpha_max) -> dict:
    """RMSNorm fused ahead of the activation path: the normalised values are transformed directly
    (they never leave the kernel, so they are not rounded to bf16), then clip and MXFP4."""
    Z = rmsnorm(X, gamma, eps)
    Y = transform(Z, A, B)
    r_min, r_max = clip_ratios(alpha_min), clip_ratios(alpha_max)
    Yh, lo, hi, nonfinite = clip_blocks(Y, r_min, r_max)
    codes, scales, q = mxfp4_quantize(Yh, nonfinite)
    return {"Z": Z, "Y": Y, "Y_hat": Yh, "codes": codes, "scales": scales, "q": q, "nonfinite": nonfinite}
