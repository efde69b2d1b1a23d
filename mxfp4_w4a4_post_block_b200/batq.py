"""Python binding of libbatq with the C-ABI's call names (argument marshalling only).

Device buffers are torch CUDA tensors (PyTorch supplies memory and streams);
every step of the path runs in libbatq's kernels.  A non-OK status raises
``BatqError``.  Host-side parameters (A, B for weight preparation, alpha for the
clip ratios) may be numpy arrays or CPU tensors.
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import _lib
from ._lib import (BATQ_BF16, BATQ_F32, BATQ_KV_MXFP4, BATQ_KV_MXFP8, BATQ_OK, BATQ_SCALES_LINEAR,  # noqa: F401
                   BATQ_SCALES_MMA)


class BatqError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        msg = _lib.load().batq_status_string(status).decode()
        super().__init__(f"{call}: {msg} (status {status})")


def _check(status: int, call: str):
    if status != BATQ_OK:
        raise BatqError(status, call)


def _torch():
    import torch
    return torch


def _dev_ptr(t, name):
    """Raw pointer of a CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not getattr(t, "is_cuda", False):
        raise TypeError(f"{name} must be a CUDA tensor (libbatq has no CPU path)")
    return ctypes.c_void_p(t.data_ptr())


def _host_f32(a, count, name):
    arr = np.ascontiguousarray(np.asarray(a.cpu() if hasattr(a, "cpu") else a, dtype=np.float32)).reshape(-1)
    if arr.size != count:
        raise ValueError(f"{name} must hold {count} floats, got {arr.size}")
    return arr


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BATQ_BF16
    if t.dtype == torch.float32:
        return BATQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32")


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ----------------------------------------------------------------- host calls

def batq_version() -> int:
    return _lib.load().batq_version()


def batq_act_buffer_sizes(rows: int, N: int, layout: int = BATQ_SCALES_MMA):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.load().batq_act_buffer_sizes(rows, N, layout, ctypes.byref(cb), ctypes.byref(sb)),
           "batq_act_buffer_sizes")
    return cb.value, sb.value


def batq_clip_ratios(alpha_min, alpha_max) -> np.ndarray:
    amin = np.ascontiguousarray(alpha_min, dtype=np.float32)
    amax = np.ascontiguousarray(alpha_max, dtype=np.float32)
    out = np.empty(2 * amin.size, dtype=np.float32)
    _check(_lib.load().batq_clip_ratios(amin.ctypes.data, amax.ctypes.data, amin.size, out.ctypes.data),
           "batq_clip_ratios")
    return out


def batq_prepare_workspace_size(N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_prepare_workspace_size(N, ctypes.byref(b)), "batq_prepare_workspace_size")
    return b.value


def batq_linear_workspace_size(S: int, N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_linear_workspace_size(S, N, ctypes.byref(b)), "batq_linear_workspace_size")
    return b.value


# -------------------------------------------------------------- device calls

def batq_quant_act(X, A, B, ratios, codes, scales, layout=BATQ_SCALES_MMA, y_debug=None, stream=None):
    """Online activation path: transform + clip + MXFP4 of X (S x N) into codes / scales."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_quant_act(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                      _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"), _dev_ptr(codes, "codes"),
                                      _dev_ptr(scales, "scales"), layout, _dev_ptr(y_debug, "y_debug"),
                                      _stream(stream)), "batq_quant_act")


def batq_prepare_weights(W, A, B_host, w_codes, w_scales, workspace, layout=BATQ_SCALES_MMA, stream=None):
    """Offline: fuse W P^-T and quantize to MXFP4 along K."""
    M, N = W.shape
    a = _host_f32(A, 64, "A")
    b = _host_f32(B_host, (N // 32) * 16, "B")
    _check(_lib.load().batq_prepare_weights(_dev_ptr(W, "W"), _dtype_code(W), M, N, W.stride(0), a.ctypes.data,
                                            b.ctypes.data, _dev_ptr(w_codes, "w_codes"),
                                            _dev_ptr(w_scales, "w_scales"), layout,
                                            _dev_ptr(workspace, "workspace"),
                                            workspace.numel() * workspace.element_size(), _stream(stream)),
           "batq_prepare_weights")


def batq_gemm_mxfp4(a_codes, a_scales, w_codes, w_scales, S, M, N, out, stream=None):
    """out (S x M, fp32 or bf16) = deq(a) deq(w)^T on the tensor cores."""
    _check(_lib.load().batq_gemm_mxfp4(_dev_ptr(a_codes, "a_codes"), _dev_ptr(a_scales, "a_scales"),
                                       _dev_ptr(w_codes, "w_codes"), _dev_ptr(w_scales, "w_scales"), S, M, N,
                                       _dtype_code(out), _dev_ptr(out, "out"), out.stride(0), _stream(stream)),
           "batq_gemm_mxfp4")


def batq_linear(X, A, B, ratios, w_codes, w_scales, M, workspace, out, stream=None):
    """Whole W4A4 linear: quantize X online, then the block-scaled GEMM against prepared weights."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_linear(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                   _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"), _dev_ptr(w_codes, "w_codes"),
                                   _dev_ptr(w_scales, "w_scales"), M, _dev_ptr(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), _dtype_code(out),
                                   _dev_ptr(out, "out"), out.stride(0), _stream(stream)), "batq_linear")


class _LinearArgs(ctypes.Structure):
    """batq_linear_args of include/batq.h."""
    _fields_ = [("X", ctypes.c_void_p), ("x_dtype", ctypes.c_int), ("S", ctypes.c_int), ("N", ctypes.c_int),
                ("ldx", ctypes.c_int), ("A_host", ctypes.c_void_p), ("B_dev", ctypes.c_void_p),
                ("ratios_dev", ctypes.c_void_p), ("w_codes", ctypes.c_void_p), ("w_scales", ctypes.c_void_p),
                ("M", ctypes.c_int), ("out_dtype", ctypes.c_int), ("out", ctypes.c_void_p), ("ldo", ctypes.c_int)]


def _linear_args(linears):
    """ctypes array of batq_linear_args from dicts with X, A, B, ratios, w_codes, w_scales, M, out; also
    returns the host copies of A that must stay alive during the call."""
    arr = (_LinearArgs * len(linears))()
    keep = []
    for i, l in enumerate(linears):
        X, out = l["X"], l["out"]
        a = _host_f32(l["A"], 64, "A")
        keep.append(a)
        arr[i] = _LinearArgs(_dev_ptr(X, "X"), _dtype_code(X), X.shape[0], X.shape[1], X.stride(0), a.ctypes.data,
                             _dev_ptr(l["B"], "B"), _dev_ptr(l["ratios"], "ratios"), _dev_ptr(l["w_codes"], "w_codes"),
                             _dev_ptr(l["w_scales"], "w_scales"), int(l["M"]), _dtype_code(out), _dev_ptr(out, "out"),
                             out.stride(0))
    return arr, keep


def batq_linear_grouped_workspace_size(shapes):
    """Workspace bytes for linears of the given (S, N) shapes."""
    arr = (_LinearArgs * len(shapes))()
    for i, (S, N) in enumerate(shapes):
        arr[i].S, arr[i].N = S, N
    n = ctypes.c_size_t()
    _check(_lib.load().batq_linear_grouped_workspace_size(ctypes.addressof(arr), len(shapes), ctypes.byref(n)),
           "batq_linear_grouped_workspace_size")
    return n.value


def batq_linear_grouped(linears, workspace, stream=None):
    """Independent linears (dicts with X, A, B, ratios, w_codes, w_scales, M, out) in one quantiser launch and one
    GEMM launch where the shapes allow (see include/batq.h)."""
    arr, keep = _linear_args(linears)
    _check(_lib.load().batq_linear_grouped(ctypes.addressof(arr), len(linears), _dev_ptr(workspace, "workspace"),
                                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "batq_linear_grouped")
    del keep


class _QuantArgs(ctypes.Structure):
    """batq_quant_args of include/batq.h."""
    _fields_ = [("X", ctypes.c_void_p), ("x_dtype", ctypes.c_int), ("S", ctypes.c_int), ("N", ctypes.c_int),
                ("ldx", ctypes.c_int), ("A_host", ctypes.c_void_p), ("B_dev", ctypes.c_void_p),
                ("ratios_dev", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("layout", ctypes.c_int)]


class _GemmArgs(ctypes.Structure):
    """batq_gemm_args of include/batq.h."""
    _fields_ = [("a_codes", ctypes.c_void_p), ("a_scales", ctypes.c_void_p), ("w_codes", ctypes.c_void_p),
                ("w_scales", ctypes.c_void_p), ("S", ctypes.c_int), ("M", ctypes.c_int), ("N", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("out", ctypes.c_void_p), ("ldo", ctypes.c_int)]


def batq_quant_act_grouped(acts, layout=BATQ_SCALES_MMA, stream=None):
    """Independent batq_quant_act calls (dicts with X, A, B, ratios, codes, scales) in one launch of the
    tensor-core quantiser when every X is bf16 (see include/batq.h)."""
    arr = (_QuantArgs * len(acts))()
    keep = []
    for i, q in enumerate(acts):
        X = q["X"]
        a = _host_f32(q["A"], 64, "A")
        keep.append(a)
        arr[i] = _QuantArgs(_dev_ptr(X, "X"), _dtype_code(X), X.shape[0], X.shape[1], X.stride(0), a.ctypes.data,
                            _dev_ptr(q["B"], "B"), _dev_ptr(q["ratios"], "ratios"), _dev_ptr(q["codes"], "codes"),
                            _dev_ptr(q["scales"], "scales"), int(layout))
    _check(_lib.load().batq_quant_act_grouped(ctypes.addressof(arr), len(acts), _stream(stream)),
           "batq_quant_act_grouped")
    del keep


def batq_gemm_mxfp4_grouped(gemms, stream=None):
    """Independent batq_gemm_mxfp4 calls (dicts with a_codes, a_scales, w_codes, w_scales, S, M, N, out) in one
    launch of the CTA-pair GEMM when every S > 128 and the output types agree (see include/batq.h)."""
    arr = (_GemmArgs * len(gemms))()
    for i, g in enumerate(gemms):
        out = g["out"]
        arr[i] = _GemmArgs(_dev_ptr(g["a_codes"], "a_codes"), _dev_ptr(g["a_scales"], "a_scales"),
                           _dev_ptr(g["w_codes"], "w_codes"), _dev_ptr(g["w_scales"], "w_scales"), int(g["S"]),
                           int(g["M"]), int(g["N"]), _dtype_code(out), _dev_ptr(out, "out"), out.stride(0))
    _check(_lib.load().batq_gemm_mxfp4_grouped(ctypes.addressof(arr), len(gemms), _stream(stream)),
           "batq_gemm_mxfp4_grouped")


def prepare_linear_grouped(linears, workspace):
    """batq_linear_grouped with its arguments marshalled once: returns run(stream=None), which launches
    the same call with a single ctypes call (for decode-size steps, where building the argument array
    on every call would cost more host time than the kernels take)."""
    arr, keep = _linear_args(linears)
    lib = _lib.load()
    ws_ptr, ws_bytes, n = _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), len(linears)
    addr = ctypes.addressof(arr)

    def run(stream=None):
        _check(lib.batq_linear_grouped(addr, n, ws_ptr, ws_bytes, _stream(stream)), "batq_linear_grouped")

    run._keep = (arr, keep, linears, workspace)  # the marshalled arguments and the tensors stay alive
    return run


def prepare_quant_act_grouped(acts, layout=BATQ_SCALES_MMA):
    """batq_quant_act_grouped with its arguments marshalled once (see prepare_linear_grouped)."""
    arr = (_QuantArgs * len(acts))()
    keep = []
    for i, q in enumerate(acts):
        X = q["X"]
        a = _host_f32(q["A"], 64, "A")
        keep.append(a)
        arr[i] = _QuantArgs(_dev_ptr(X, "X"), _dtype_code(X), X.shape[0], X.shape[1], X.stride(0), a.ctypes.data,
                            _dev_ptr(q["B"], "B"), _dev_ptr(q["ratios"], "ratios"), _dev_ptr(q["codes"], "codes"),
                            _dev_ptr(q["scales"], "scales"), int(layout))
    lib, addr, n = _lib.load(), ctypes.addressof(arr), len(acts)

    def run(stream=None):
        _check(lib.batq_quant_act_grouped(addr, n, _stream(stream)), "batq_quant_act_grouped")

    run._keep = (arr, keep, acts)
    return run


def prepare_gemm_mxfp4_grouped(gemms):
    """batq_gemm_mxfp4_grouped with its arguments marshalled once (see prepare_linear_grouped)."""
    arr = (_GemmArgs * len(gemms))()
    for i, g in enumerate(gemms):
        out = g["out"]
        arr[i] = _GemmArgs(_dev_ptr(g["a_codes"], "a_codes"), _dev_ptr(g["a_scales"], "a_scales"),
                           _dev_ptr(g["w_codes"], "w_codes"), _dev_ptr(g["w_scales"], "w_scales"), int(g["S"]),
                           int(g["M"]), int(g["N"]), _dtype_code(out), _dev_ptr(out, "out"), out.stride(0))
    lib, addr, n = _lib.load(), ctypes.addressof(arr), len(gemms)

    def run(stream=None):
        _check(lib.batq_gemm_mxfp4_grouped(addr, n, _stream(stream)), "batq_gemm_mxfp4_grouped")

    run._keep = (arr, gemms)
    return run


def batq_linear_no_alloc(X, A, B, ratios, w_codes, w_scales, M, out, stream=None):
    """batq_linear for callers that cannot allocate device memory: the scratch for the
    quantised activations comes from a fixed array inside the library (see
    include/batq.h for its size, sharing and ordering rules)."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_linear_no_alloc(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                            _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"),
                                            _dev_ptr(w_codes, "w_codes"), _dev_ptr(w_scales, "w_scales"), M,
                                            _dtype_code(out), _dev_ptr(out, "out"), out.stride(0),
                                            _stream(stream)), "batq_linear_no_alloc")


# ------------------------------------------------------ W4A8 variant calls

def batq_mxfp8_buffer_sizes(rows: int, N: int, layout: int = BATQ_SCALES_MMA):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.load().batq_mxfp8_buffer_sizes(rows, N, layout, ctypes.byref(cb), ctypes.byref(sb)),
           "batq_mxfp8_buffer_sizes")
    return cb.value, sb.value


def batq_prepare_weights_w4a8_workspace_size(M: int, N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_prepare_weights_w4a8_workspace_size(M, N, ctypes.byref(b)),
           "batq_prepare_weights_w4a8_workspace_size")
    return b.value


def batq_linear_w4a8_workspace_size(S: int, N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_linear_w4a8_workspace_size(S, N, ctypes.byref(b)), "batq_linear_w4a8_workspace_size")
    return b.value


def batq_quant_act_mxfp8(X, A, B, ratios, codes, scales, layout=BATQ_SCALES_MMA, y_debug=None, stream=None):
    """W4A8 activation path: transform + clip + MXFP8 (E4M3) of X (S x N) into codes (S x N) / scales."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_quant_act_mxfp8(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                            _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"), _dev_ptr(codes, "codes"),
                                            _dev_ptr(scales, "scales"), layout, _dev_ptr(y_debug, "y_debug"),
                                            _stream(stream)), "batq_quant_act_mxfp8")


def batq_prepare_weights_w4a8(W, A, B_host, w_codes8, w_scales, workspace, layout=BATQ_SCALES_MMA, stream=None):
    """Offline: the MXFP4 weights of batq_prepare_weights, each code held in one E4M3 byte (M x N)."""
    M, N = W.shape
    a = _host_f32(A, 64, "A")
    b = _host_f32(B_host, (N // 32) * 16, "B")
    _check(_lib.load().batq_prepare_weights_w4a8(_dev_ptr(W, "W"), _dtype_code(W), M, N, W.stride(0),
                                                 a.ctypes.data, b.ctypes.data, _dev_ptr(w_codes8, "w_codes8"),
                                                 _dev_ptr(w_scales, "w_scales"), layout,
                                                 _dev_ptr(workspace, "workspace"),
                                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "batq_prepare_weights_w4a8")


def batq_gemm_w4a8(a_codes8, a_scales, w_codes8, w_scales, S, M, N, out, stream=None):
    """out (S x M) = deq(a) deq(w)^T with E4M3 codes on both sides."""
    _check(_lib.load().batq_gemm_w4a8(_dev_ptr(a_codes8, "a_codes8"), _dev_ptr(a_scales, "a_scales"),
                                      _dev_ptr(w_codes8, "w_codes8"), _dev_ptr(w_scales, "w_scales"), S, M, N,
                                      _dtype_code(out), _dev_ptr(out, "out"), out.stride(0), _stream(stream)),
           "batq_gemm_w4a8")


def batq_linear_w4a8(X, A, B, ratios, w_codes8, w_scales, M, workspace, out, stream=None):
    """Whole W4A8 linear: MXFP8 activations online, then the E4M3 x E4M3 block-scaled GEMM."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_linear_w4a8(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                        _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"),
                                        _dev_ptr(w_codes8, "w_codes8"), _dev_ptr(w_scales, "w_scales"), M,
                                        _dev_ptr(workspace, "workspace"),
                                        workspace.numel() * workspace.element_size(), _dtype_code(out),
                                        _dev_ptr(out, "out"), out.stride(0), _stream(stream)), "batq_linear_w4a8")


# ------------------------------------------------------ NVFP4 output calls

def batq_nvfp4_buffer_sizes(rows: int, N: int, layout: int = BATQ_SCALES_MMA):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.load().batq_nvfp4_buffer_sizes(rows, N, layout, ctypes.byref(cb), ctypes.byref(sb)),
           "batq_nvfp4_buffer_sizes")
    return cb.value, sb.value


def batq_prepare_weights_nvfp4_workspace_size(N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_prepare_weights_nvfp4_workspace_size(N, ctypes.byref(b)),
           "batq_prepare_weights_nvfp4_workspace_size")
    return b.value


def batq_linear_nvfp4_workspace_size(S: int, N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_linear_nvfp4_workspace_size(S, N, ctypes.byref(b)), "batq_linear_nvfp4_workspace_size")
    return b.value


def batq_quant_act_nvfp4(X, A, B, ratios, codes, scales, gs=None, layout=BATQ_SCALES_MMA, y_debug=None,
                         stream=None):
    """Transform + clip (32-blocks) + NVFP4 (E4M3 scale per 16) of X (S x N); gs: 1-element CUDA float or None."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_quant_act_nvfp4(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                            _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"), _dev_ptr(gs, "gs"),
                                            _dev_ptr(codes, "codes"), _dev_ptr(scales, "scales"), layout,
                                            _dev_ptr(y_debug, "y_debug"), _stream(stream)), "batq_quant_act_nvfp4")


def batq_prepare_weights_nvfp4(W, A, B_host, w_codes, w_scales, gs_out, workspace, layout=BATQ_SCALES_MMA,
                               stream=None):
    """Offline: fused weights measured for their amax, then NVFP4 with gs = 448*6/amax written to gs_out."""
    M, N = W.shape
    a = _host_f32(A, 64, "A")
    b = _host_f32(B_host, (N // 32) * 16, "B")
    _check(_lib.load().batq_prepare_weights_nvfp4(_dev_ptr(W, "W"), _dtype_code(W), M, N, W.stride(0),
                                                  a.ctypes.data, b.ctypes.data, _dev_ptr(w_codes, "w_codes"),
                                                  _dev_ptr(w_scales, "w_scales"), layout, _dev_ptr(gs_out, "gs_out"),
                                                  _dev_ptr(workspace, "workspace"),
                                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "batq_prepare_weights_nvfp4")


def batq_gemm_nvfp4(a_codes, a_scales, a_gs, w_codes, w_scales, w_gs, S, M, N, out, stream=None):
    """out (S x M) = fp32(1/(gs_a gs_w)) x deq(a) deq(w)^T for NVFP4 operands (gs tensors or None)."""
    _check(_lib.load().batq_gemm_nvfp4(_dev_ptr(a_codes, "a_codes"), _dev_ptr(a_scales, "a_scales"),
                                       _dev_ptr(a_gs, "a_gs"), _dev_ptr(w_codes, "w_codes"),
                                       _dev_ptr(w_scales, "w_scales"), _dev_ptr(w_gs, "w_gs"), S, M, N,
                                       _dtype_code(out), _dev_ptr(out, "out"), out.stride(0), _stream(stream)),
           "batq_gemm_nvfp4")


def batq_linear_nvfp4(X, A, B, ratios, a_gs, w_codes, w_scales, w_gs, M, workspace, out, stream=None):
    """Whole NVFP4 linear: NVFP4 activations online, then the kind::mxf4nvf4 block-scaled GEMM."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_linear_nvfp4(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                         _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"), _dev_ptr(a_gs, "a_gs"),
                                         _dev_ptr(w_codes, "w_codes"), _dev_ptr(w_scales, "w_scales"),
                                         _dev_ptr(w_gs, "w_gs"), M, _dev_ptr(workspace, "workspace"),
                                         workspace.numel() * workspace.element_size(), _dtype_code(out),
                                         _dev_ptr(out, "out"), out.stride(0), _stream(stream)), "batq_linear_nvfp4")


# ------------------------------------------------- naive Kronecker (per-block A_i)

def batq_prepare_weights_kron_workspace_size(N: int) -> int:
    b = ctypes.c_size_t()
    _check(_lib.load().batq_prepare_weights_kron_workspace_size(N, ctypes.byref(b)),
           "batq_prepare_weights_kron_workspace_size")
    return b.value


def batq_quant_act_kron(X, A_blocks, B, ratios, codes, scales, layout=BATQ_SCALES_MMA, y_debug=None, stream=None):
    """As batq_quant_act with one 8x8 A_i per block (A_blocks: CUDA float tensor, k x 64)."""
    S, N = X.shape
    _check(_lib.load().batq_quant_act_kron(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0),
                                           _dev_ptr(A_blocks, "A_blocks"), _dev_ptr(B, "B"),
                                           _dev_ptr(ratios, "ratios"), _dev_ptr(codes, "codes"),
                                           _dev_ptr(scales, "scales"), layout, _dev_ptr(y_debug, "y_debug"),
                                           _stream(stream)), "batq_quant_act_kron")


def batq_prepare_weights_kron(W, A_blocks_host, B_host, w_codes, w_scales, workspace, layout=BATQ_SCALES_MMA,
                              stream=None):
    """Offline weight side with one A_i per block (host arrays: A_blocks k x 8 x 8, B k x 4 x 4)."""
    M, N = W.shape
    k = N // 32
    a = _host_f32(A_blocks_host, k * 64, "A_blocks")
    b = _host_f32(B_host, k * 16, "B")
    _check(_lib.load().batq_prepare_weights_kron(_dev_ptr(W, "W"), _dtype_code(W), M, N, W.stride(0),
                                                 a.ctypes.data, b.ctypes.data, _dev_ptr(w_codes, "w_codes"),
                                                 _dev_ptr(w_scales, "w_scales"), layout,
                                                 _dev_ptr(workspace, "workspace"),
                                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "batq_prepare_weights_kron")


def batq_linear_kron(X, A_blocks, B, ratios, w_codes, w_scales, M, workspace, out, stream=None):
    """Whole W4A4 linear with one A_i per block (A_blocks: CUDA float tensor, k x 64)."""
    S, N = X.shape
    _check(_lib.load().batq_linear_kron(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0),
                                        _dev_ptr(A_blocks, "A_blocks"), _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"),
                                        _dev_ptr(w_codes, "w_codes"), _dev_ptr(w_scales, "w_scales"), M,
                                        _dev_ptr(workspace, "workspace"),
                                        workspace.numel() * workspace.element_size(), _dtype_code(out),
                                        _dev_ptr(out, "out"), out.stride(0), _stream(stream)), "batq_linear_kron")


# -------------------------------------------------------------- KV cache

def batq_quant_kv_cache(X, A, B, ratios, slot_mapping, cache_codes, cache_scales, kv_format=BATQ_KV_MXFP4,
                        stream=None):
    """Transform + clip + MXFP4 / MXFP8 of new K or V rows X (S x N) into cache rows slot_mapping (int32 CUDA)."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    num_slots = cache_codes.shape[0]
    _check(_lib.load().batq_quant_kv_cache(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0), a.ctypes.data,
                                           _dev_ptr(B, "B"), _dev_ptr(ratios, "ratios"),
                                           _dev_ptr(slot_mapping, "slot_mapping"), num_slots, kv_format,
                                           _dev_ptr(cache_codes, "cache_codes"), _dev_ptr(cache_scales, "cache_scales"),
                                           _stream(stream)), "batq_quant_kv_cache")


# ------------------------------------------------- RMSNorm ahead of the transform

def batq_rmsnorm_workspace_size(S: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.load().batq_rmsnorm_workspace_size(S, ctypes.byref(v)), "batq_rmsnorm_workspace_size")
    return v.value


def batq_rmsnorm_linear_workspace_size(S: int, N: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.load().batq_rmsnorm_linear_workspace_size(S, N, ctypes.byref(v)), "batq_rmsnorm_linear_workspace_size")
    return v.value


def batq_rmsnorm_quant_act(X, gamma, eps, A, B, ratios, codes, scales, workspace, layout=BATQ_SCALES_MMA,
                           y_debug=None, stream=None):
    """RMSNorm (gamma: CUDA float tensor of N, eps) fused ahead of the transform, clip and MXFP4 of X."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_rmsnorm_quant_act(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0),
                                              _dev_ptr(gamma, "gamma"), float(eps), a.ctypes.data, _dev_ptr(B, "B"),
                                              _dev_ptr(ratios, "ratios"), _dev_ptr(codes, "codes"),
                                              _dev_ptr(scales, "scales"), layout, _dev_ptr(workspace, "workspace"),
                                              workspace.numel() * workspace.element_size(),
                                              _dev_ptr(y_debug, "y_debug"), _stream(stream)), "batq_rmsnorm_quant_act")


def batq_rmsnorm_linear(X, gamma, eps, A, B, ratios, w_codes, w_scales, M, workspace, out, stream=None):
    """Whole W4A4 linear with the RMSNorm fused ahead of the online quantisation."""
    S, N = X.shape
    a = _host_f32(A, 64, "A")
    _check(_lib.load().batq_rmsnorm_linear(_dev_ptr(X, "X"), _dtype_code(X), S, N, X.stride(0),
                                           _dev_ptr(gamma, "gamma"), float(eps), a.ctypes.data, _dev_ptr(B, "B"),
                                           _dev_ptr(ratios, "ratios"), _dev_ptr(w_codes, "w_codes"),
                                           _dev_ptr(w_scales, "w_scales"), M, _dev_ptr(workspace, "workspace"),
                                           workspace.numel() * workspace.element_size(), _dtype_code(out),
                                           _dev_ptr(out, "out"), out.stride(0), _stream(stream)), "batq_rmsnorm_linear")


def batq_selftest_wait_timeout(limit_us: int, stream=None):
    """Launch the bounded-wait self-test kernel (its wait always expires)."""
    _check(_lib.load().batq_selftest_wait_timeout(limit_us, _stream(stream)), "batq_selftest_wait_timeout")


def batq_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    v = ctypes.c_uint(0)
    st = _lib.load().batq_device_error(_stream(stream), ctypes.byref(v))
    if st not in (BATQ_OK, _lib.BATQ_ERR_TIMEOUT):
        raise BatqError(st, "batq_device_error")
    return v.value


# ------------------------------------------------------- allocation helpers

def empty_act_buffers(rows: int, N: int, layout=BATQ_SCALES_MMA, device="cuda"):
    """(codes, scales) uint8 CUDA tensors sized for a rows x N matrix."""
    torch = _torch()
    cb, sb = batq_act_buffer_sizes(rows, N, layout)
    codes = torch.empty((rows, N // 2), dtype=torch.uint8, device=device)
    scales = torch.empty(sb, dtype=torch.uint8, device=device)
    return codes, scales


def empty_mxfp8_buffers(rows: int, N: int, layout=BATQ_SCALES_MMA, device="cuda"):
    """(codes, scales) uint8 CUDA tensors for MXFP8 (one byte per element) of a rows x N matrix."""
    torch = _torch()
    cb, sb = batq_mxfp8_buffer_sizes(rows, N, layout)
    codes = torch.empty((rows, N), dtype=torch.uint8, device=device)
    scales = torch.empty(sb, dtype=torch.uint8, device=device)
    return codes, scales


def empty_nvfp4_buffers(rows: int, N: int, layout=BATQ_SCALES_MMA, device="cuda"):
    """(codes, scales) uint8 CUDA tensors for NVFP4 (packed E2M1, one scale per 16) of a rows x N matrix."""
    torch = _torch()
    cb, sb = batq_nvfp4_buffer_sizes(rows, N, layout)
    codes = torch.empty((rows, N // 2), dtype=torch.uint8, device=device)
    scales = torch.empty(sb, dtype=torch.uint8, device=device)
    return codes, scales
