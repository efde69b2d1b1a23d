"""Failure detection on the GPU without a fault: a barrier wait that runs out.

Every libbatq kernel waits on its pipeline barriers with a bounded wait; when a
wait expires the kernel records a bit in a per-device error word and returns,
so a lost stage turns into BATQ_ERR_TIMEOUT on the host instead of a hang.
batq_selftest_wait_timeout runs that same wait on a barrier nothing arrives on.
"""

import time

import numpy as np
import pytest
import torch

from mxfp4_w4a4_post_block_b200 import _lib
from mxfp4_w4a4_post_block_b200 import batq as BQ
from mxfp4_w4a4_post_block_b200 import workloads as WL
import gpu_util as GU

pytestmark = pytest.mark.gpu


def test_expired_wait_sets_error_word_and_context_stays_usable():
    assert BQ.batq_device_error() == 0
    t0 = time.perf_counter()
    BQ.batq_selftest_wait_timeout(2000)  # 2 ms
    flags = BQ.batq_device_error()
    assert flags & 1, flags
    assert time.perf_counter() - t0 < 5.0
    # the word was cleared and the context still runs the real kernels
    assert BQ.batq_device_error() == 0
    w = WL.tiny(with_w=False)
    codes, scales, _, _ = GU.gpu_quant(w, BQ.BATQ_SCALES_LINEAR, y_debug=False)
    assert codes.shape == (w.S, w.N // 2)


def test_device_error_status_code():
    L = _lib.load()
    BQ.batq_selftest_wait_timeout(500)
    import ctypes
    v = ctypes.c_uint(0)
    st = L.batq_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(v))
    assert st == _lib.BATQ_ERR_TIMEOUT and v.value & 1


def test_selftest_argument_check():
    with pytest.raises(BQ.BatqError):
        BQ.batq_selftest_wait_timeout(0)
