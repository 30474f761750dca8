"""swa_decode_static: the decode step for callers that cannot allocate device
memory (an engine with a fixed, pre-planned arena, or code that only receives
tensor pointers).  It takes no workspace; its scratch is an array built into
the library.  These tests check it against swa_decode (which takes a caller
workspace) on the same inputs, over two calls in a row, and check that dims
needing more scratch than the built-in array holds are refused.

This file is named so that pytest collects it last.
"""
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_chunk_b200 as swa
from tests.gpu_helpers import assert_close, dev_i32

pytestmark = pytest.mark.gpu
DEV = "cuda"
STATIC_SCRATCH_BYTES = 4 << 20


def _case(B=4, W=1024, Hq=32, Hkv=8, d=128, seed=123):
    g = torch.Generator().manual_seed(seed)
    dims = swa.Dims(B, Hq, Hkv, d, W, 1.0 / math.sqrt(d), "f32")
    kc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    pos0 = torch.randint(W, 8 * W, (B,), generator=g).tolist()
    steps = []
    for _ in range(2):
        steps.append(tuple(torch.randn(B, h, d, generator=g).to(torch.bfloat16).to(DEV)
                           for h in (Hq, Hkv, Hkv)))
    return dims, kc, vc, pos0, steps


def test_static_decode_matches_workspace_decode_on_two_calls():
    dims, kc, vc, pos0, steps = _case()
    need = swa.decode_workspace_size(dims)
    assert 16 < need <= STATIC_SCRATCH_BYTES  # the split path, so the scratch is used
    kc_a, vc_a = kc.to(DEV), vc.to(DEV)       # swa_decode with a workspace
    kc_b, vc_b = kc.to(DEV), vc.to(DEV)       # swa_decode_static
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    for i, (q, k, v) in enumerate(steps):
        pos = dev_i32([p + i for p in pos0])
        out_a = torch.zeros((dims.batch, dims.n_q_heads, dims.head_dim), dtype=torch.float32,
                            device=DEV)
        out_b = torch.full_like(out_a, float("nan"))
        swa.decode(dims, out_a, q, k, v, kc_a, vc_a, pos, ws)
        swa.decode_static(dims, out_b, q, k, v, kc_b, vc_b, pos)
        torch.cuda.synchronize()
        assert_close(out_b.double().cpu().numpy(), out_a.double().cpu().numpy(),
                     f"static vs workspace decode, call {i}")
        assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)
    swa.device_status()


def test_static_decode_refuses_dims_beyond_its_scratch():
    # 64 sequences x 64 query heads x 2 splits of fp32 partials > 4 MiB
    dims = swa.Dims(64, 64, 8, 128, 4096, 1.0 / math.sqrt(128), "f32")
    assert swa.decode_workspace_size(dims) > STATIC_SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.bfloat16, device=DEV)
    pos = dev_i32([0])
    with pytest.raises(swa.SwaError) as e:
        swa.decode_static(dims, t, t, t, t, t, t, pos)
    assert e.value.code == swa.SWA_ERR_WORKSPACE_TOO_SMALL
    assert "built-in scratch" in e.value.message
    swa.device_status()
