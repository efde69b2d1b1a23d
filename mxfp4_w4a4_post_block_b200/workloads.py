"""Seeded synthetic inputs for the BATQuant W4A4 linear path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no transform, clip, scale rule or encoding).  The same
arrays feed both the CUDA library and the CPU oracle, so parity tests compare
the two on identical bytes.

The source pages evaluate on Qwen3-8B / Qwen3-VL-8B activations and weights,
which are not available here.  These generators stand in for them with the
shapes of the pages' workloads (hidden size 4096, down_proj input 12288, MXFP
block g = 32) and heavy-tailed activations with a few outlier channels, the
structure the pages' activation figures show (thelatestinai.com BATQuant page,
Figure 2 caption: down_proj layer 35 with an extreme-outlier block; Figure 5:
q_proj layer 6).  The transform parameters A, B_i and the clip logits alpha are
given inputs of the method (calibration is out of scope), drawn near identity.

Recipes (numpy ``default_rng(seed)``, drawn in the order listed):

* ``tiny``      seed 0: S=16, N=256, M=128; X fp32 N(0,1), 2 outlier channels
  x50; A = I + 0.05 N, B_i = I + 0.05 N; alpha_min, alpha_max ~ N(3, 0.5);
  W ~ N(0, 0.02).
* ``q_proj``    seed 2: S=2048, N=4096, M=4096; X bf16 Student-t(nu=4) with 1 %
  of channels x100; A, B_i = I + 0.1 N; alpha ~ N(2, 1); W ~ N(0, 0.02).
* ``down_proj`` seed 3: S=4096, N=12288, M=4096; X bf16 N(0,1) with 0.5 % of
  channels x300 and 3 tokens x20; A, B_i = I + 0.1 N; alpha ~ N(1.5, 1).
* ``decode``    seed 4: S in {1, 4, 16}, N=4096, M=24576 (fused gate+up); X as
  q_proj.
* ``layer``     seeds 500+j for the seven linears of one decoder layer at
  S=8192 (q, k, v, o, gate, up, down); X as q_proj.
* ``with_naive_kronecker(w, seed)``: w's inputs with one A_i = I + 0.1 N per block.
* ``with_block_hadamard(w)``: w's X and W with P_i = H_32 / sqrt(32) (Sylvester) for every
  block and no clip, the block-rotation baseline as an input.
* ``rmsnorm_gamma(N, seed)``: RMSNorm weights 1 + 0.2 N(0, 1) for the fused norm ahead of the
  transform (eps = 1e-6 in the tests).
"""

from __future__ import annotations

import dataclasses

import numpy as np

BLOCK = 32  # MXFP block size g

# (name, N in-features, M out-features) of the seven linears of one Qwen3-8B-shaped layer
LAYER_LINEARS = (
    ("q", 4096, 4096),
    ("k", 4096, 1024),
    ("v", 4096, 1024),
    ("o", 4096, 4096),
    ("gate", 4096, 12288),
    ("up", 4096, 12288),
    ("down", 12288, 4096),
)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Workload:
    """One linear layer's inputs.

    ``x`` holds the activation values as fp32 (already rounded to bf16 when
    ``x_dtype == "bf16"``); ``x_bits`` holds the bytes handed to the device
    (uint16 bf16 patterns or the fp32 array itself).
    """

    name: str
    seed: int
    S: int
    N: int
    M: int
    x_dtype: str
    x: np.ndarray
    x_bits: np.ndarray
    A: np.ndarray  # (8, 8) fp32, global
    B: np.ndarray  # (k, 4, 4) fp32, one per block column
    alpha_min: np.ndarray  # (k,) fp32 clip logits
    alpha_max: np.ndarray  # (k,) fp32
    W: np.ndarray | None  # (M, N) fp32 or None when not drawn

    @property
    def k(self) -> int:
        return self.N // BLOCK


def _near_identity(rng, shape, sigma):
    n = shape[-1]
    eye = np.eye(n, dtype=np.float64)
    return (eye + sigma * rng.standard_normal(shape)).astype(np.float32)


def _finish(name, seed, rng, x, x_dtype, N, M, sigma, a_mu, a_sd, with_w):
    k = N // BLOCK
    A = _near_identity(rng, (8, 8), sigma)
    B = _near_identity(rng, (k, 4, 4), sigma)
    alpha_min = (a_mu + a_sd * rng.standard_normal(k)).astype(np.float32)
    alpha_max = (a_mu + a_sd * rng.standard_normal(k)).astype(np.float32)
    W = None
    if with_w:
        W = (0.02 * rng.standard_normal((M, N), dtype=np.float32)).astype(np.float32)
    if x_dtype == "bf16":
        bits = bf16_bits_from_f32(x)
        xv = f32_from_bf16_bits(bits)
    else:
        bits = np.ascontiguousarray(x, dtype=np.float32)
        xv = bits
    return Workload(name, seed, x.shape[0], N, M, x_dtype, xv, bits, A, B, alpha_min, alpha_max, W)


def _outlier_channels(rng, N, frac):
    count = max(1, int(round(frac * N)))
    return rng.choice(N, size=count, replace=False)


def tiny(with_w: bool = True) -> Workload:
    """S=16, N=256, M=128 fp32 activations; the case the oracle finishes instantly."""
    seed, S, N, M = 0, 16, 256, 128
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, N)).astype(np.float32)
    ch = rng.choice(N, size=2, replace=False)
    x[:, ch] *= 50.0
    return _finish("tiny", seed, rng, x, "f32", N, M, 0.05, 3.0, 0.5, with_w)


def _student_t_outliers(rng, S, N, frac, mult):
    x = rng.standard_t(4.0, size=(S, N)).astype(np.float32)
    ch = _outlier_channels(rng, N, frac)
    x[:, ch] *= mult
    return x


def q_proj(S: int = 2048, with_w: bool = True, seed: int = 2) -> Workload:
    """Qwen3-8B-shaped q_proj prefill: S=2048, N=4096, M=4096, bf16 Student-t(4) + 1 % x100 channels."""
    N, M = 4096, 4096
    rng = np.random.default_rng(seed)
    x = _student_t_outliers(rng, S, N, 0.01, 100.0)
    return _finish("q_proj", seed, rng, x, "bf16", N, M, 0.1, 2.0, 1.0, with_w)


def down_proj(S: int = 4096, with_w: bool = True, seed: int = 3) -> Workload:
    """down_proj with heavy outliers: S=4096, N=12288, M=4096; 0.5 % channels x300, 3 tokens x20."""
    N, M = 12288, 4096
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, N), dtype=np.float32)
    ch = _outlier_channels(rng, N, 0.005)
    x[:, ch] *= 300.0
    tok = rng.choice(S, size=min(3, S), replace=False)
    x[tok, :] *= 20.0
    return _finish("down_proj", seed, rng, x, "bf16", N, M, 0.1, 1.5, 1.0, with_w)


def decode(S: int = 16, with_w: bool = True, seed: int = 4) -> Workload:
    """Decode-shaped fused gate+up: S in {1,4,16}, N=4096, M=24576."""
    if S not in (1, 4, 16):
        raise ValueError("decode workload is defined for S in {1, 4, 16}")
    N, M = 4096, 24576
    rng = np.random.default_rng(seed)
    x = _student_t_outliers(rng, S, N, 0.01, 100.0)
    return _finish("decode", seed, rng, x, "bf16", N, M, 0.1, 2.0, 1.0, with_w)


def layer_linear(j: int, S: int = 8192, with_w: bool = True) -> Workload:
    """Linear j (0..6 = q,k,v,o,gate,up,down) of one Qwen3-8B-shaped decoder layer at S=8192."""
    name, N, M = LAYER_LINEARS[j]
    seed = 500 + j
    rng = np.random.default_rng(seed)
    x = _student_t_outliers(rng, S, N, 0.01, 100.0)
    return _finish("layer_" + name, seed, rng, x, "bf16", N, M, 0.1, 2.0, 1.0, with_w)


def custom(S: int, N: int, M: int, seed: int, x_dtype: str = "bf16", sigma: float = 0.1,
           with_w: bool = True, outlier_frac: float = 0.01, outlier_mult: float = 100.0) -> Workload:
    """Arbitrary shape with the q_proj recipe (used for ragged / edge-case tests)."""
    rng = np.random.default_rng(seed)
    x = _student_t_outliers(rng, S, N, outlier_frac, outlier_mult)
    return _finish(f"custom_{S}x{N}x{M}", seed, rng, x, x_dtype, N, M, sigma, 2.0, 1.0, with_w)


def sylvester_hadamard(n: int) -> np.ndarray:
    """Sylvester's +-1 Hadamard matrix of order n (a power of two): H_1 = [1], H_2m = [[H, H], [H, -H]]."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    if h.shape[0] != n:
        raise ValueError("order must be a power of two")
    return h


def with_block_hadamard(w: Workload) -> Workload:
    """The same activations and weights with the block Hadamard transform as every P_i and no clip.

    This is the block-rotation baseline the pages compare against (BRQ; thelatestinai.com BATQuant
    page, Figure 2 caption, panel (a)) given as an input of the method: Sylvester's construction
    makes H_32 = H_4 (x) H_8, so A = H_8 / sqrt(8) (fp32) and B_i = H_4 / 2 give
    P_i = H_32 / sqrt(32) up to the fp32 rounding of A; alpha = 40 makes sigma(alpha) = 1 in fp32.
    """
    k = w.N // BLOCK
    A = (sylvester_hadamard(8) / np.sqrt(8.0)).astype(np.float32)
    B = np.tile((sylvester_hadamard(4) / 2.0).astype(np.float32), (k, 1, 1))
    big = np.full(k, 40.0, np.float32)
    return dataclasses.replace(w, name=w.name + "_blockhadamard", A=A, B=B, alpha_min=big, alpha_max=big.copy())


def with_naive_kronecker(w: Workload, seed: int = 0, sigma: float = 0.1) -> Workload:
    """The same inputs with one 8x8 factor per block, A_i = I + sigma N(0, 1) (the "naive Kronecker"
    decomposition of Table 1, P_i = B_i (x) A_i), drawn from default_rng(seed)."""
    k = w.N // BLOCK
    rng = np.random.default_rng(seed)
    A = _near_identity(rng, (k, 8, 8), sigma)
    return dataclasses.replace(w, name=w.name + "_naivekron", A=A)


def rmsnorm_gamma(N: int, seed: int) -> np.ndarray:
    """RMSNorm weights for the fused norm ahead of the transform: fp32 (N,), 1 + 0.2 N(0, 1) from
    default_rng(seed) (the norm weight of a trained layer sits around 1; the pages give no values)."""
    rng = np.random.default_rng(seed)
    return (1.0 + 0.2 * rng.standard_normal(N)).astype(np.float32)


CONFIGS = {
    "tiny": tiny,
    "q_proj": q_proj,
    "down_proj": down_proj,
    "decode": decode,
}
