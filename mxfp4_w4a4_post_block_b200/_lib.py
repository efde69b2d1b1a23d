"""ctypes loader for libbatq.so (argument types only; no logic)."""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbatq.so")

BATQ_OK = 0
BATQ_ERR_INVALID_ARG = 1
BATQ_ERR_SHAPE = 2
BATQ_ERR_ALIGNMENT = 3
BATQ_ERR_SINGULAR = 4
BATQ_ERR_ARCH = 5
BATQ_ERR_CUDA = 6
BATQ_ERR_TIMEOUT = 7
BATQ_ERR_WORKSPACE = 8
BATQ_ERR_SCRATCH_LIMIT = 9
NO_ALLOC_SCRATCH_BYTES = 16 * 1024 * 1024

BATQ_F32 = 0
BATQ_BF16 = 1
BATQ_SCALES_LINEAR = 0
BATQ_SCALES_MMA = 1
BATQ_KV_MXFP4 = 0
BATQ_KV_MXFP8 = 1

_c_int, _c_size_p, _vp, _fp = ctypes.c_int, ctypes.POINTER(ctypes.c_size_t), ctypes.c_void_p, ctypes.c_void_p

# name -> (restype, argtypes); one entry per function declared in include/batq.h
SIGNATURES = {
    "batq_status_string": (ctypes.c_char_p, [_c_int]),
    "batq_version": (_c_int, []),
    "batq_act_buffer_sizes": (_c_int, [_c_int, _c_int, _c_int, _c_size_p, _c_size_p]),
    "batq_clip_ratios": (_c_int, [_vp, _vp, _c_int, _vp]),
    "batq_quant_act": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]),
    "batq_prepare_workspace_size": (_c_int, [_c_int, _c_size_p]),
    "batq_prepare_weights": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp,
                                      ctypes.c_size_t, _vp]),
    "batq_gemm_mxfp4": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp]),
    "batq_linear_workspace_size": (_c_int, [_c_int, _c_int, _c_size_p]),
    "batq_linear": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                             ctypes.c_size_t, _c_int, _vp, _c_int, _vp]),
    "batq_linear_grouped_workspace_size": (_c_int, [_vp, _c_int, _c_size_p]),
    "batq_linear_grouped": (_c_int, [_vp, _c_int, _vp, ctypes.c_size_t, _vp]),
    "batq_quant_act_grouped": (_c_int, [_vp, _c_int, _vp]),
    "batq_gemm_mxfp4_grouped": (_c_int, [_vp, _c_int, _vp]),
    "batq_linear_no_alloc": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int,
                                      _c_int, _vp, _c_int, _vp]),
    "batq_mxfp8_buffer_sizes": (_c_int, [_c_int, _c_int, _c_int, _c_size_p, _c_size_p]),
    "batq_quant_act_mxfp8": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                                      _vp]),
    "batq_prepare_weights_w4a8_workspace_size": (_c_int, [_c_int, _c_int, _c_size_p]),
    "batq_prepare_weights_w4a8": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp,
                                           ctypes.c_size_t, _vp]),
    "batq_gemm_w4a8": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp]),
    "batq_linear_w4a8_workspace_size": (_c_int, [_c_int, _c_int, _c_size_p]),
    "batq_linear_w4a8": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                                  ctypes.c_size_t, _c_int, _vp, _c_int, _vp]),
    "batq_nvfp4_buffer_sizes": (_c_int, [_c_int, _c_int, _c_int, _c_size_p, _c_size_p]),
    "batq_quant_act_nvfp4": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                                      _vp, _vp]),
    "batq_prepare_weights_nvfp4_workspace_size": (_c_int, [_c_int, _c_size_p]),
    "batq_prepare_weights_nvfp4": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp,
                                            _vp, ctypes.c_size_t, _vp]),
    "batq_gemm_nvfp4": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp]),
    "batq_linear_nvfp4_workspace_size": (_c_int, [_c_int, _c_int, _c_size_p]),
    "batq_linear_nvfp4": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                                   _vp, ctypes.c_size_t, _c_int, _vp, _c_int, _vp]),
    "batq_quant_act_kron": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                                     _vp]),
    "batq_prepare_weights_kron_workspace_size": (_c_int, [_c_int, _c_size_p]),
    "batq_prepare_weights_kron": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp,
                                           ctypes.c_size_t, _vp]),
    "batq_linear_kron": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                                  ctypes.c_size_t, _c_int, _vp, _c_int, _vp]),
    "batq_quant_kv_cache": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _c_int, _vp,
                                     _vp, _vp]),
    "batq_rmsnorm_workspace_size": (_c_int, [_c_int, _c_size_p]),
    "batq_rmsnorm_quant_act": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, ctypes.c_float, _vp, _vp, _vp,
                                        _vp, _vp, _c_int, _vp, ctypes.c_size_t, _vp, _vp]),
    "batq_rmsnorm_linear_workspace_size": (_c_int, [_c_int, _c_int, _c_size_p]),
    "batq_rmsnorm_linear": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, ctypes.c_float, _vp, _vp, _vp, _vp,
                                     _vp, _c_int, _vp, ctypes.c_size_t, _c_int, _vp, _c_int, _vp]),
    "batq_selftest_wait_timeout": (_c_int, [ctypes.c_uint, _vp]),
    "batq_device_error": (_c_int, [_vp, ctypes.POINTER(ctypes.c_uint)]),
}

_LIB = None


def load() -> ctypes.CDLL:
    """Load libbatq.so once; raise if it has not been built (there is no fallback)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mxfp4_w4a4_post_block_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB
