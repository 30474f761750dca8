"""Failure detection without faulting the GPU.

The library is rebuilt for these tests with -DSWA_TEST_FAULTS and a bounded
wait limit of about a millisecond (instead of about two seconds).  The checked
build adds two switches:

* a device flag (passed through swa_debug_set_trace) that makes softmax warp 0
  withhold its P-ready arrival on the last key tile of its first item.  The
  MMA warp's bounded wait on that arrival runs out, the kernel records
  SWA_ERR_TIMEOUT in the status word, every role leaves through the normal
  teardown (its issued copies awaited, tensor memory freed) and the call
  returns.  No copy is withheld and nothing traps;
* a host flag (swa_debug_fail_encode) that makes the TMA descriptor encoding
  fail as if the driver had refused it: the call must return SWA_ERR_CUDA
  before anything is enqueued.

After each fault the same GPU context must still run the tiny workload of the
normal library correctly.
"""
import ctypes
import math
import os

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from sliding_window_gqa_chunk_b200.csrc import build as swa_build
from swa_workloads import random_case
from tests.gpu_helpers import assert_close, dev_i32, gpu_chunked_prefill

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda"


@pytest.fixture(scope="module")
def faults_lib():
    so = swa_build.build(force=True, defines=["SWA_TEST_FAULTS", "SWA_WAIT_LIMIT_CYCLES=2000000LL"],
                         out=os.path.join(HERE, "_build", "libswa_faults.so"))
    lib = ctypes.CDLL(so)
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    D = ctypes.POINTER(swa._CDims)
    lib.swa_prefill_chunk.argtypes = [D, P, P, P, P, I32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.swa_prefill_chunk.restype = ctypes.c_int
    lib.swa_prefill_workspace_size.argtypes = [D, I32]
    lib.swa_prefill_workspace_size.restype = ctypes.c_size_t
    lib.swa_device_status.argtypes = [P]
    lib.swa_device_status.restype = ctypes.c_int
    lib.swa_last_error.restype = ctypes.c_char_p
    lib.swa_debug_set_trace.argtypes = [P]
    lib.swa_debug_set_trace.restype = None
    lib.swa_debug_fail_encode.argtypes = [ctypes.c_int]
    lib.swa_debug_fail_encode.restype = None
    return lib


def _case():
    B, L, W, Hq, Hkv, d = 1, 256, 256, 4, 2, 64
    q, k, v = random_case(31, B, L, Hq, Hkv, d)
    dims = swa.Dims(B, Hq, Hkv, d, W, 1.0 / math.sqrt(d), "f32")
    return dims, q, k, v


def _call(lib, dims, q, k, v, out, kc, vc, ws=None):
    cd = dims.c()
    T = q.shape[1]
    sp, nt = dev_i32([0]), dev_i32([T])
    ws_ptr = None if ws is None else ws.data_ptr()
    ws_bytes = 0 if ws is None else ws.numel()
    return lib.swa_prefill_chunk(ctypes.byref(cd), out.data_ptr(), q.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), T, kc.data_ptr(), vc.data_ptr(), sp.data_ptr(),
                                 nt.data_ptr(), ws_ptr, ws_bytes, None)


def _normal_library_still_works():
    """The tiny prefill through the normal library, against the oracle."""
    B, L, W, Hq, Hkv, d = 1, 12, 4, 4, 2, 16
    q, k, v = random_case(5, B, L, Hq, Hkv, d)
    dims = swa.Dims(B, Hq, Hkv, d, W, 0.25, "f32")
    got, _, _ = gpu_chunked_prefill(dims, q, k, v, [L], 4)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, 4, 0.25)
    assert_close(got, ref, "normal library after a fault")


@pytest.mark.parametrize("persistent", [False, True], ids=["grid", "persistent"])
def test_withheld_arrival_times_out_and_the_gpu_stays_usable(faults_lib, persistent):
    dims, q, k, v = _case()
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    kc, vc = swa.new_cache(dims, DEV)
    out = torch.zeros(q.shape, dtype=torch.float32, device=DEV)
    ws = None
    if persistent:
        ws = torch.zeros(faults_lib.swa_prefill_workspace_size(ctypes.byref(dims.c()), q.shape[1]),
                         dtype=torch.uint8, device=DEV)
    flag = torch.ones(1, dtype=torch.int32, device=DEV)
    faults_lib.swa_debug_set_trace(ctypes.c_void_p(flag.data_ptr()))
    try:
        assert _call(faults_lib, dims, qd, kd, vd, out, kc, vc, ws) == swa.SWA_OK
        torch.cuda.synchronize()
        assert faults_lib.swa_device_status(None) == swa.SWA_ERR_TIMEOUT
        assert b"status 5" in faults_lib.swa_last_error()
        assert faults_lib.swa_device_status(None) == swa.SWA_OK     # read and cleared
        # switch off: the checked build itself computes the chunk correctly
        flag.zero_()
        if ws is not None:
            ws.zero_()      # a timed-out call may leave its counters behind
        out.zero_()
        assert _call(faults_lib, dims, qd, kd, vd, out, kc, vc, ws) == swa.SWA_OK
        torch.cuda.synchronize()
        assert faults_lib.swa_device_status(None) == swa.SWA_OK
    finally:
        faults_lib.swa_debug_set_trace(None)
    ref, _ = oracle.run_chunked_prefill(q, k, v, dims.window, q.shape[1], dims.scale)
    assert_close(out.double().cpu().numpy(), ref, "checked build after the timeout")
    _normal_library_still_works()


def test_descriptor_encode_failure_enqueues_nothing(faults_lib):
    dims, q, k, v = _case()
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    kc, vc = swa.new_cache(dims, DEV)
    out = torch.full(q.shape, 7.0, dtype=torch.float32, device=DEV)
    faults_lib.swa_debug_fail_encode(1)
    try:
        rc = _call(faults_lib, dims, qd, kd, vd, out, kc, vc)
    finally:
        faults_lib.swa_debug_fail_encode(0)
    assert rc == swa.SWA_ERR_CUDA
    assert b"injected" in faults_lib.swa_last_error()
    torch.cuda.synchronize()
    assert faults_lib.swa_device_status(None) == swa.SWA_OK
    assert bool((out == 7.0).all())                       # nothing ran
    assert float(kc.abs().sum()) == 0.0
    _normal_library_still_works()
