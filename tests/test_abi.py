"""The C-ABI library loads and exports every declared symbol; host-only calls and
argument checks work without a GPU (no compute call is made here)."""

import ctypes
import os
import re

import numpy as np
import pytest

from mxfp4_w4a4_post_block_b200 import _lib
from mxfp4_w4a4_post_block_b200 import batq as BQ
from oracle import batq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "batq.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BATQ_API\s+[\w\s\*]*?\b(batq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        from mxfp4_w4a4_post_block_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_expected_calls():
    names = _declared()
    for n in ("batq_quant_act", "batq_prepare_weights", "batq_gemm_mxfp4", "batq_linear"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) == set(_lib.SIGNATURES), "binding signatures out of sync with the header"


def test_status_strings_and_version(L):
    assert L.batq_status_string(0) == b"ok"
    assert b"aligned" in L.batq_status_string(3)
    assert L.batq_version() >= 100


def test_buffer_sizes(L):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.batq_act_buffer_sizes(2048, 4096, 1, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert cb.value == 2048 * 2048 and sb.value == 2048 * 128
    assert L.batq_act_buffer_sizes(16, 320, 1, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert sb.value == O.mma_layout_bytes(16, 10) == 128 * 12
    assert L.batq_act_buffer_sizes(16, 320, 0, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert sb.value == 16 * 10
    assert L.batq_act_buffer_sizes(16, 100, 0, ctypes.byref(cb), ctypes.byref(sb)) == _lib.BATQ_ERR_SHAPE
    assert L.batq_act_buffer_sizes(0, 256, 0, ctypes.byref(cb), ctypes.byref(sb)) == _lib.BATQ_ERR_SHAPE
    assert L.batq_act_buffer_sizes(16, 256, 7, ctypes.byref(cb), ctypes.byref(sb)) == _lib.BATQ_ERR_INVALID_ARG


def test_clip_ratios_match_oracle(L):
    rng = np.random.default_rng(0)
    amin = (rng.standard_normal(384) * 3).astype(np.float32)
    amax = (rng.standard_normal(384) * 3).astype(np.float32)
    out = np.empty(768, np.float32)
    assert L.batq_clip_ratios(amin.ctypes.data, amax.ctypes.data, 384, out.ctypes.data) == 0
    np.testing.assert_array_equal(out[0::2], O.clip_ratios(amin))
    np.testing.assert_array_equal(out[1::2], O.clip_ratios(amax))


def test_workspace_sizes(L):
    b = ctypes.c_size_t()
    assert L.batq_linear_workspace_size(2048, 4096, ctypes.byref(b)) == 0
    assert b.value >= 2048 * 2048 + 2048 * 128
    assert L.batq_prepare_workspace_size(4096, ctypes.byref(b)) == 0
    assert b.value >= 128 * 64


FAKE = 0x10000  # never dereferenced: every call below fails in host-side validation


def test_quant_argument_checks_fail_before_any_launch(L):
    A = np.eye(8, dtype=np.float32)
    qa = L.batq_quant_act
    # null pointer
    assert qa(None, 1, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_INVALID_ARG
    # N not a multiple of 64
    assert qa(FAKE, 1, 16, 250, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_SHAPE
    # ldx < N
    assert qa(FAKE, 1, 16, 256, 128, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_SHAPE
    # misaligned X
    assert qa(FAKE + 2, 1, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_ALIGNMENT
    # bf16 row stride not a multiple of 16 bytes
    assert qa(FAKE, 1, 16, 256, 260, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_ALIGNMENT
    # bad dtype / layout
    assert qa(FAKE, 5, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, None) == _lib.BATQ_ERR_INVALID_ARG
    assert qa(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 9, None, None) == _lib.BATQ_ERR_INVALID_ARG


def test_gemm_argument_checks_fail_before_any_launch(L):
    g = L.batq_gemm_mxfp4
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 100, 256, 0, FAKE, 100, None) == _lib.BATQ_ERR_SHAPE  # M % 16
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 128, 96, 0, FAKE, 128, None) == _lib.BATQ_ERR_SHAPE   # N % 64
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 128, 256, 0, FAKE, 128, None) == _lib.BATQ_ERR_SHAPE   # S < 1
    assert g(FAKE, FAKE, FAKE + 8, FAKE, 16, 128, 256, 0, FAKE, 128, None) == _lib.BATQ_ERR_ALIGNMENT
    assert g(FAKE, FAKE, FAKE, FAKE, 16, 128, 256, 0, FAKE, 130, None) == _lib.BATQ_ERR_ALIGNMENT  # ldo*4 % 16
    assert g(None, FAKE, FAKE, FAKE, 16, 128, 256, 0, FAKE, 128, None) == _lib.BATQ_ERR_INVALID_ARG


def test_linear_workspace_checks(L):
    A = np.eye(8, dtype=np.float32)
    st = L.batq_linear(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE, FAKE, 128, FAKE, 16, 0, FAKE, 128,
                       None)
    assert st == _lib.BATQ_ERR_WORKSPACE


def _group(shapes):
    arr = (BQ._LinearArgs * len(shapes))()
    for i, (S, N) in enumerate(shapes):
        arr[i].S, arr[i].N = S, N
    return arr


def test_grouped_workspace_size_is_the_256_aligned_sum(L):
    shapes = [(16, 256), (300, 1024), (4096, 12288), (1, 64)]
    want = 0
    for S, N in shapes:
        one = ctypes.c_size_t()
        assert L.batq_linear_workspace_size(S, N, ctypes.byref(one)) == _lib.BATQ_OK
        want += -(-one.value // 256) * 256
    got = ctypes.c_size_t()
    arr = _group(shapes)
    assert L.batq_linear_grouped_workspace_size(ctypes.addressof(arr), len(shapes), ctypes.byref(got)) == _lib.BATQ_OK
    assert got.value == want
    assert BQ.batq_linear_grouped_workspace_size(shapes) == want


def test_grouped_argument_checks_fail_before_any_launch(L):
    n = ctypes.c_size_t()
    arr = _group([(16, 256)] * 9)
    assert L.batq_linear_grouped_workspace_size(ctypes.addressof(arr), 0, ctypes.byref(n)) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_linear_grouped_workspace_size(ctypes.addressof(arr), 9, ctypes.byref(n)) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_linear_grouped_workspace_size(None, 1, ctypes.byref(n)) == _lib.BATQ_ERR_INVALID_ARG
    bad = _group([(16, 256), (16, 100)])  # N % 64 != 0
    assert L.batq_linear_grouped_workspace_size(ctypes.addressof(bad), 2, ctypes.byref(n)) == _lib.BATQ_ERR_SHAPE
    one = _group([(16, 256)])
    assert L.batq_linear_grouped(ctypes.addressof(one), 1, None, 1 << 20, None) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_linear_grouped(ctypes.addressof(one), 9, FAKE, 1 << 20, None) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_linear_grouped(ctypes.addressof(one), 1, FAKE, 16, None) == _lib.BATQ_ERR_WORKSPACE
    # enough workspace, but X is null: the quantiser's argument check refuses it
    assert L.batq_linear_grouped(ctypes.addressof(one), 1, FAKE, 1 << 20, None) == _lib.BATQ_ERR_INVALID_ARG


def test_grouped_quant_and_gemm_checks_fail_before_any_launch(L):
    A = np.eye(8, dtype=np.float32)
    q = (BQ._QuantArgs * 2)()
    q[0] = BQ._QuantArgs(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, 0, FAKE, FAKE, 1)
    q[1] = BQ._QuantArgs(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, 0, FAKE, FAKE, 1)
    assert L.batq_quant_act_grouped(ctypes.addressof(q), 0, None) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_quant_act_grouped(ctypes.addressof(q), 9, None) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_quant_act_grouped(None, 1, None) == _lib.BATQ_ERR_INVALID_ARG
    q[1].N = 100  # second activation's shape is refused although the first is valid
    assert L.batq_quant_act_grouped(ctypes.addressof(q), 2, None) == _lib.BATQ_ERR_SHAPE
    q[1].N, q[1].layout = 256, 7
    assert L.batq_quant_act_grouped(ctypes.addressof(q), 2, None) == _lib.BATQ_ERR_INVALID_ARG
    g = (BQ._GemmArgs * 2)()
    g[0] = BQ._GemmArgs(FAKE, FAKE, FAKE, FAKE, 16, 128, 256, 0, FAKE, 128)
    g[1] = BQ._GemmArgs(FAKE, FAKE, FAKE, FAKE, 16, 120, 256, 0, FAKE, 128)  # M % 16 != 0
    assert L.batq_gemm_mxfp4_grouped(ctypes.addressof(g), 0, None) == _lib.BATQ_ERR_INVALID_ARG
    assert L.batq_gemm_mxfp4_grouped(ctypes.addressof(g), 2, None) == _lib.BATQ_ERR_SHAPE
    g[1].M, g[1].a_codes = 128, 0
    assert L.batq_gemm_mxfp4_grouped(ctypes.addressof(g), 2, None) == _lib.BATQ_ERR_INVALID_ARG


def test_prepare_checks(L):
    A = np.eye(8, dtype=np.float32)
    B = np.tile(np.eye(4, dtype=np.float32), (8, 1, 1))
    st = L.batq_prepare_weights(FAKE, 0, 128, 256, 256, A.ctypes.data, B.ctypes.data, FAKE, FAKE, 1, FAKE, 1, None)
    assert st == _lib.BATQ_ERR_WORKSPACE


def test_variant_buffer_and_workspace_sizes(L):
    cb, sb, b = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    # MXFP8: one byte per element, the MXFP4 scale layouts
    assert L.batq_mxfp8_buffer_sizes(200, 320, 1, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert cb.value == 200 * 320 and sb.value == O.mma_layout_bytes(200, 10)
    # NVFP4: packed codes, one scale per 16 elements (N/16 columns, a multiple of 4)
    assert L.batq_nvfp4_buffer_sizes(200, 320, 1, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert cb.value == 200 * 160 and sb.value == 256 * 20 == O.mma_layout_bytes(200, 20)
    assert L.batq_nvfp4_buffer_sizes(200, 320, 0, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert sb.value == 200 * 20
    assert L.batq_nvfp4_buffer_sizes(200, 100, 0, ctypes.byref(cb), ctypes.byref(sb)) == _lib.BATQ_ERR_SHAPE
    base = ctypes.c_size_t()
    assert L.batq_prepare_workspace_size(4096, ctypes.byref(base)) == 0
    assert L.batq_prepare_weights_nvfp4_workspace_size(4096, ctypes.byref(b)) == 0 and b.value == base.value + 256
    assert L.batq_prepare_weights_kron_workspace_size(4096, ctypes.byref(b)) == 0
    assert b.value == base.value + 128 * 64 * 4
    assert L.batq_linear_nvfp4_workspace_size(2048, 4096, ctypes.byref(b)) == 0
    assert b.value == 2048 * 2048 + 2048 * 256
    assert L.batq_linear_w4a8_workspace_size(2048, 4096, ctypes.byref(b)) == 0
    assert b.value == 2048 * 4096 + 2048 * 128
    assert L.batq_prepare_weights_w4a8_workspace_size(4096, 4096, ctypes.byref(b)) == 0
    assert b.value == base.value + 4096 * 2048


def test_variant_argument_checks_fail_before_any_launch(L):
    A = np.eye(8, dtype=np.float32)
    B = np.tile(np.eye(4, dtype=np.float32), (8, 1, 1))
    err = _lib
    # NVFP4: misaligned per-tensor scale pointers, missing gs output
    assert L.batq_quant_act_nvfp4(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, None, FAKE + 2, FAKE, FAKE, 1, None,
                                  None) == err.BATQ_ERR_ALIGNMENT
    assert L.batq_gemm_nvfp4(FAKE, FAKE, FAKE + 1, FAKE, FAKE, None, 16, 128, 256, 0, FAKE, 128,
                             None) == err.BATQ_ERR_ALIGNMENT
    assert L.batq_prepare_weights_nvfp4(FAKE, 0, 128, 256, 256, A.ctypes.data, B.ctypes.data, FAKE, FAKE, 1, None,
                                        FAKE, 1 << 20, None) == err.BATQ_ERR_INVALID_ARG
    assert L.batq_linear_nvfp4(FAKE, 1, 16, 256, 256, A.ctypes.data, FAKE, None, None, FAKE, FAKE, None, 128, FAKE, 16,
                               0, FAKE, 128, None) == err.BATQ_ERR_WORKSPACE
    # KV cache: slot mapping, slot count, format, alignment
    kv = L.batq_quant_kv_cache
    assert kv(FAKE, 1, 16, 1024, 1024, A.ctypes.data, FAKE, None, None, 100, 0, FAKE, FAKE,
              None) == err.BATQ_ERR_INVALID_ARG
    assert kv(FAKE, 1, 16, 1024, 1024, A.ctypes.data, FAKE, None, FAKE, 0, 0, FAKE, FAKE,
              None) == err.BATQ_ERR_INVALID_ARG
    assert kv(FAKE, 1, 16, 1024, 1024, A.ctypes.data, FAKE, None, FAKE, 100, 2, FAKE, FAKE,
              None) == err.BATQ_ERR_INVALID_ARG
    assert kv(FAKE, 1, 16, 1024, 1024, A.ctypes.data, FAKE, None, FAKE + 2, 100, 1, FAKE, FAKE,
              None) == err.BATQ_ERR_ALIGNMENT
    assert kv(FAKE, 1, 16, 1000, 1024, A.ctypes.data, FAKE, None, FAKE, 100, 1, FAKE, FAKE,
              None) == err.BATQ_ERR_SHAPE
    # naive Kronecker: per-block factors required and 16-byte aligned; workspaces checked
    assert L.batq_quant_act_kron(FAKE, 1, 16, 256, 256, None, FAKE, None, FAKE, FAKE, 1, None,
                                 None) == err.BATQ_ERR_INVALID_ARG
    assert L.batq_quant_act_kron(FAKE, 1, 16, 256, 256, FAKE + 4, FAKE, None, FAKE, FAKE, 1, None,
                                 None) == err.BATQ_ERR_ALIGNMENT
    Ak = np.tile(np.eye(8, dtype=np.float32), (8, 1, 1))
    assert L.batq_prepare_weights_kron(FAKE, 0, 128, 256, 256, Ak.ctypes.data, B.ctypes.data, FAKE, FAKE, 1, FAKE,
                                       64, None) == err.BATQ_ERR_WORKSPACE
    assert L.batq_linear_kron(FAKE, 1, 16, 256, 256, FAKE, FAKE, None, FAKE, FAKE, 128, FAKE, 16, 0, FAKE, 128,
                              None) == err.BATQ_ERR_WORKSPACE


def test_rmsnorm_sizes_and_argument_checks_fail_before_any_launch(L):
    """The fused RMSNorm calls: workspace sizes, and every argument error reported on the host
    before anything is launched (no GPU needed)."""
    v = ctypes.c_size_t()
    assert L.batq_rmsnorm_workspace_size(1000, ctypes.byref(v)) == 0 and v.value == 4096
    assert L.batq_rmsnorm_workspace_size(0, ctypes.byref(v)) == _lib.BATQ_ERR_SHAPE
    lin = ctypes.c_size_t()
    assert L.batq_linear_workspace_size(2048, 4096, ctypes.byref(lin)) == 0
    assert L.batq_rmsnorm_linear_workspace_size(2048, 4096, ctypes.byref(v)) == 0
    assert v.value == -(-lin.value // 256) * 256 + 8192
    A = np.eye(8, dtype=np.float32)
    q = L.batq_rmsnorm_quant_act
    # null gamma, negative or non-finite eps, null workspace
    assert q(FAKE, 1, 16, 256, 256, None, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 256, None,
             None) == _lib.BATQ_ERR_INVALID_ARG
    assert q(FAKE, 1, 16, 256, 256, FAKE, -1.0, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 256, None,
             None) == _lib.BATQ_ERR_INVALID_ARG
    assert q(FAKE, 1, 16, 256, 256, FAKE, float("nan"), A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 256, None,
             None) == _lib.BATQ_ERR_INVALID_ARG
    assert q(FAKE, 1, 16, 256, 256, FAKE, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None, 256, None,
             None) == _lib.BATQ_ERR_INVALID_ARG
    # misaligned gamma, short workspace, bad shape
    assert q(FAKE, 1, 16, 256, 256, FAKE + 4, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 256, None,
             None) == _lib.BATQ_ERR_ALIGNMENT
    assert q(FAKE, 1, 16, 256, 256, FAKE, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 16, None,
             None) == _lib.BATQ_ERR_WORKSPACE
    assert q(FAKE, 1, 16, 100, 256, FAKE, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, FAKE, 256, None,
             None) == _lib.BATQ_ERR_SHAPE
    lr = L.batq_rmsnorm_linear
    assert lr(FAKE, 1, 16, 256, 256, FAKE, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 128, FAKE, 64, 0, FAKE, 128,
              None) == _lib.BATQ_ERR_WORKSPACE
    assert lr(FAKE, 1, 16, 256, 256, None, 1e-6, A.ctypes.data, FAKE, None, FAKE, FAKE, 128, FAKE, 1 << 20, 0, FAKE,
              128, None) == _lib.BATQ_ERR_INVALID_ARG


def test_sizes_beyond_the_32_bit_index_range_are_rejected(L):
    """rows x N/32 must stay below 2^31 (the kernels' tile indices and scale offsets are 32-bit)."""
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.batq_act_buffer_sizes((1 << 31) // 128 - 1, 4096, 1, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert L.batq_act_buffer_sizes((1 << 31) // 128, 4096, 1, ctypes.byref(cb), ctypes.byref(sb)) == _lib.BATQ_ERR_SHAPE
    A = np.eye(8, dtype=np.float32)
    assert L.batq_quant_act(FAKE, 1, 1 << 24, 4096, 4096, A.ctypes.data, FAKE, None, FAKE, FAKE, 1, None,
                            None) == _lib.BATQ_ERR_SHAPE


def test_no_alloc_scratch_limit_edge(L):
    """The fixed scratch of batq_linear_no_alloc holds exactly the workspace of 7704 tokens at
    N = 4096 (codes 7704 x 2048 bytes plus MMA-layout scales 7808 x 128 bytes = 16 MiB); one token
    more is refused with BATQ_ERR_SCRATCH_LIMIT before any CUDA call, so this runs without a GPU."""
    ws = ctypes.c_size_t()
    assert L.batq_linear_workspace_size(7704, 4096, ctypes.byref(ws)) == 0
    assert ws.value == _lib.NO_ALLOC_SCRATCH_BYTES
    assert L.batq_linear_workspace_size(7705, 4096, ctypes.byref(ws)) == 0
    assert ws.value > _lib.NO_ALLOC_SCRATCH_BYTES
    A = np.eye(8, dtype=np.float32)
    buf = (ctypes.c_uint8 * 256)()
    p = (ctypes.addressof(buf) + 15) // 16 * 16  # never dereferenced: the size check comes first
    st = L.batq_linear_no_alloc(p, _lib.BATQ_BF16, 7705, 4096, 4096, A.ctypes.data, p, p, p, p, 4096,
                                _lib.BATQ_F32, p, 4096, None)
    assert st == _lib.BATQ_ERR_SCRATCH_LIMIT
    assert b"scratch" in L.batq_status_string(st)
