"""swa_decode_static: the decode step for callers that cannot allocate device
memory (an engine with a fixed, pre-planned arena, or code that only receives
tensor pointers).  It takes no workspace; its scratch is an array built into
the library.

The dims here take the path that really uses that scratch: enough (sequence,
kv head) pairs (more than the SMs) that the splits of the cache sweep are
merged through memory by a second kernel (swa_decode_launch_info reports two
launches).  Two calls
in a row are checked against swa_decode with a caller workspace and against
the float64 oracle; then calls with other dims (another split count and batch,
so another partial layout over the same scratch) show that nothing stale from
the earlier calls leaks in.  Dims that need more scratch than the array holds
are refused.

This file is named so that pytest collects it last.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from tests.gpu_helpers import assert_close, dev_i32

pytestmark = pytest.mark.gpu
DEV = "cuda"
STATIC_SCRATCH_BYTES = 4 << 20


def _run_case(B, W, Hq, Hkv, d, expect_splits, seed):
    dims = swa.Dims(B, Hq, Hkv, d, W, 1.0 / math.sqrt(d), "f32")
    n_splits, n_launches = swa.decode_launch_info(dims)
    assert (n_splits, n_launches) == (expect_splits, 2)        # merged through the scratch
    assert B * Hq * n_splits * (d + 2) * 4 <= STATIC_SCRATCH_BYTES
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    pos0 = torch.randint(W, 8 * W, (B,), generator=g).tolist()
    ref = oracle.RollingCache(B, Hkv, W, d)
    k64, v64 = kc.double().numpy(), vc.double().numpy()
    for b in range(B):
        for p in range(pos0[b] - W, pos0[b]):
            ref.write(b, p, k64[b, :, p % W], v64[b, :, p % W])
    kc_a, vc_a = kc.to(DEV), vc.to(DEV)       # swa_decode with a workspace
    kc_b, vc_b = kc.to(DEV), vc.to(DEV)       # swa_decode_static
    ws = swa.decode_workspace(dims, DEV)
    for i in range(2):
        q, k, v = (torch.randn(B, h, d, generator=g).to(torch.bfloat16) for h in (Hq, Hkv, Hkv))
        pos = [p + i for p in pos0]
        out_a = torch.zeros((B, Hq, d), dtype=torch.float32, device=DEV)
        out_b = torch.full_like(out_a, float("nan"))
        qd, kd, vd, posd = q.to(DEV), k.to(DEV), v.to(DEV), dev_i32(pos)
        swa.decode(dims, out_a, qd, kd, vd, kc_a, vc_a, posd, ws)
        swa.decode_static(dims, out_b, qd, kd, vd, kc_b, vc_b, posd)
        torch.cuda.synchronize()
        expect = oracle.decode(ref, q, k, v, pos, dims.scale)
        got_b = out_b.double().cpu().numpy()
        assert_close(got_b, expect, f"static decode B={B} W={W} call {i} vs oracle")
        assert_close(got_b, out_a.double().cpu().numpy(),
                     f"static decode B={B} W={W} call {i} vs workspace decode")
        assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)
        np.testing.assert_array_equal(kc_b.double().cpu().numpy(), ref.k)
    swa.device_status()


def test_static_decode_uses_its_scratch_and_matches_on_two_calls():
    # 24 x 8 = 192 (sequence, kv head) pairs: 3 splits of 1408 slots each,
    # merged by the combine kernel through 1.2 MB of the built-in scratch
    _run_case(B=24, W=4096, Hq=32, Hkv=8, d=128, expect_splits=3, seed=123)


def test_static_decode_after_other_dims_sees_no_stale_scratch():
    # run after the case above: 256 pairs, 2 splits, another layout of partials
    # over the same scratch bytes, then the first dims again
    _run_case(B=32, W=4096, Hq=32, Hkv=8, d=128, expect_splits=2, seed=7)
    _run_case(B=24, W=4096, Hq=32, Hkv=8, d=128, expect_splits=3, seed=8)


def test_static_decode_refuses_dims_beyond_its_scratch():
    # 32 sequences x 128 query heads x 2 splits of fp32 partials: 4.26 MB > 4 MiB
    dims = swa.Dims(32, 128, 8, 128, 4096, 1.0 / math.sqrt(128), "f32")
    assert swa.decode_launch_info(dims) == (2, 2)
    t = torch.zeros(16, dtype=torch.bfloat16, device=DEV)
    pos = dev_i32([0])
    with pytest.raises(swa.SwaError) as e:
        swa.decode_static(dims, t, t, t, t, t, t, pos)
    assert e.value.code == swa.SWA_ERR_WORKSPACE_TOO_SMALL
    assert "built-in scratch" in e.value.message
    swa.device_status()
