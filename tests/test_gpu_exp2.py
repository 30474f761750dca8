"""The prefill softmax computes part of its 2^x on the FMA pipe (range reduction
plus a cubic fitted for the library, see csrc/swa_exp2.cuh).  Check it on the
device against CUDA's exp2f and float64 over the argument range the softmax
produces: finite values in [-126, 8] (clamped below -126)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
BUILD = os.path.join(HERE, "_build")


def _lib():
    os.makedirs(BUILD, exist_ok=True)
    so = os.path.join(BUILD, "libexp2_check.so")
    src = os.path.join(HERE, "csrc", "exp2_check.cu")
    csrc = os.path.join(ROOT, "sliding_window_gqa_chunk_b200", "csrc")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
                    "-I", csrc, src, "-o", so], check=True)
    lib = ctypes.CDLL(so)
    lib.exp2_check.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int]
    return lib


def test_fma_pipe_exp2_error_bound():
    lib = _lib()
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 21), torch.arange(-125.0, 9.0),
                   torch.tensor([0.0, -0.5, 0.5, -126.0, -125.5, 7.99, -1e-7, 1e-7])])
    if x.numel() % 2:
        x = torch.cat([x, torch.zeros(1)])
    xd = x.cuda()
    outs = [torch.empty_like(xd) for _ in range(3)]
    assert lib.exp2_check(xd.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                          outs[2].data_ptr(), xd.numel()) == 0
    fma_pipe, sfu, ref = (o.double().cpu().numpy() for o in outs)
    exact = np.exp2(x.double().numpy())
    rel = np.abs(fma_pipe - exact) / exact
    assert rel.max() < 1.1e-4, rel.max()
    # and against CUDA's exp2f
    rel_cuda = np.abs(fma_pipe - ref) / ref
    assert rel_cuda.max() < 1.2e-4
    # exact powers of two at integer arguments
    ints = (x.numpy() == np.round(x.numpy())) & (x.numpy() > -126)
    assert ints.sum() >= 100
    np.testing.assert_array_equal(fma_pipe[ints], exact[ints])
    # the SFU path stays within its own documented few-ulp error
    assert (np.abs(sfu - exact) / exact).max() < 1e-6


def test_fma_pipe_exp2_is_exactly_zero_for_masked_keys():
    # A masked key enters the softmax as -inf; it must contribute exactly 0,
    # as the SFU's exp2(-inf) does.  So must anything below the clamp.
    lib = _lib()
    x = torch.tensor([-float("inf"), -1e30, -200.0, -126.5, -127.0, -126.0, 0.0, 1.0])
    xd = x.cuda()
    outs = [torch.empty_like(xd) for _ in range(3)]
    assert lib.exp2_check(xd.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                          outs[2].data_ptr(), xd.numel()) == 0
    got = outs[0].cpu().numpy()
    assert (got[:5] == 0.0).all(), got
    assert got[5] == 2.0 ** -126 and got[6] == 1.0 and got[7] == 2.0
    assert (outs[1].cpu().numpy()[:1] == 0.0).all()
