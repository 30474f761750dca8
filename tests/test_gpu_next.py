"""GPU checks of two uses of the boundary beyond the single-path workloads.

* Mixed prefill and decode in one launch (continuous batching): a decode token
  is a one-token chunk that attends to the cache before its own append plus
  itself, which is the decode step's key set (Mistral 7B, section 2, Rolling
  Buffer Cache and Pre-fill and Chunking paragraphs).  So one
  swa_prefill_chunk call serves sequences that prefill chunks of different
  lengths next to sequences that decode one token, each at its own position.
* Receptive field of stacked layers (section 2, Sliding Window Attention and
  Figure 1): with Q = 0 every visible key gets the same weight, so with
  positive values a change at token t reaches exactly positions
  t .. t + k(W - 1) after k layers.  Every chained layer is also compared with
  the oracle's full-KV windowed attention of its input.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from swa_workloads import random_case
from tests.gpu_helpers import assert_close, cache_as_f64, dev_i32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gather(x, starts, counts, T):
    """Rows starts[b] .. starts[b] + counts[b] of x [B, L, H, d] into [B, T, H, d]."""
    B = x.shape[0]
    out = torch.zeros((B, T) + tuple(x.shape[2:]), dtype=x.dtype)
    for b in range(B):
        n = counts[b]
        out[b, :n] = x[b, starts[b]:starts[b] + n]
    return out


def test_mixed_prefill_and_decode_in_one_launch():
    B, W, Hq, Hkv, d = 4, 256, 8, 2, 64
    q, k, v = random_case(77, B, 576, Hq, Hkv, d)
    dims = swa.Dims(B, Hq, Hkv, d, W, 1.0 / 8.0, "f32")
    kc, vc = swa.new_cache(dims, DEV)
    ref = oracle.RollingCache(B, Hkv, W, d)
    # histories: seq 0 none, seq 1 positions 0..299, seq 2 0..511, seq 3 0..4
    calls = [([0, 0, 0, 0], [0, 256, 256, 5]), ([0, 256, 256, 5], [0, 44, 256, 0])]
    # then one launch: seq 0 prefills 200 tokens from 0, seq 1 decodes at 300,
    # seq 2 prefills 64 tokens from 512 (full, wrapped cache), seq 3 decodes at 5
    calls.append(([0, 300, 512, 5], [200, 1, 64, 1]))
    for ci, (starts, counts) in enumerate(calls):
        T = max(max(counts), 1)
        qc, kcn, vcn = (_gather(x, starts, counts, T) for x in (q, k, v))
        o = torch.zeros((B, T, Hq, d), dtype=torch.float32, device=DEV)
        sp, nt = dev_i32(starts), dev_i32(counts)
        kg, vg = kcn.to(DEV), vcn.to(DEV)
        swa.prefill_chunk(dims, o, qc.to(DEV), kg, vg, kc, vc, sp, nt,
                          workspace=swa.prefill_workspace(dims, T, DEV))
        swa.cache_append(dims, kc, vc, kg, vg, sp, nt)
        expect = oracle.prefill_chunk(ref, qc, kcn, vcn, starts, counts, dims.scale)
        oracle.cache_append(ref, kcn, vcn, starts, counts)
        if ci == len(calls) - 1:
            got = o.double().cpu().numpy()
            for b in range(B):
                n = counts[b]
                assert_close(got[b, :n], expect[b, :n], f"mixed launch, sequence {b} (n={n})")
            # the two one-token rows are exactly the oracle's decode steps
            for b in (1, 3):
                dec_ref = oracle.RollingCache(1, Hkv, W, d)
                for p in range(max(0, starts[b] - W + 1), starts[b]):
                    dec_ref.write(0, p, k[b, p], v[b, p])
                dec = oracle.decode(dec_ref, q[b:b + 1, starts[b]], k[b:b + 1, starts[b]],
                                    v[b:b + 1, starts[b]], [starts[b]], dims.scale)
                assert_close(got[b, 0][None], dec, f"decode row of sequence {b}")
    np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
    np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    swa.device_status()


def _layer(x, W, k_layers_cache=None):
    """One attention layer on the GPU with Q = 0: x [1, L, 1, d] bf16 values
    (keys are x too; they do not matter when Q = 0).  Chunks of W tokens."""
    L, d = x.shape[1], x.shape[3]
    dims = swa.Dims(1, 1, 1, d, W, 1.0, "f32")
    kc, vc = swa.new_cache(dims, DEV)
    xd = x.to(DEV)
    qz = torch.zeros_like(xd)
    out = torch.zeros((1, L, 1, d), dtype=torch.float32, device=DEV)
    for s in range(0, L, W):
        n = min(W, L - s)
        sp, nt = dev_i32([s]), dev_i32([n])
        swa.prefill_chunk(dims, out[:, s:s + n], qz[:, s:s + n], xd[:, s:s + n], xd[:, s:s + n],
                          kc, vc, sp, nt)
        swa.cache_append(dims, kc, vc, xd[:, s:s + n], xd[:, s:s + n], sp, nt)
    return out.cpu()


@pytest.mark.parametrize("k_layers", [1, 2, 3])
def test_receptive_field_of_stacked_layers(k_layers):
    W, L, d, t = 4, 24, 16, 5
    base = torch.ones((1, L, 1, d), dtype=torch.bfloat16)
    pert = base.clone()
    pert[0, t] = 2.0
    xb, xp = base, pert
    for layer in range(k_layers):
        # each chained GPU layer against the oracle's full-KV windowed attention
        # of that layer's (bf16) input, with Q = 0 as on the GPU
        for name, x in (("base", xb), ("perturbed", xp)):
            got = _layer(x, W)
            ref = oracle.full_kv_banded(torch.zeros_like(x), x, x, W, 1.0)
            assert_close(got.double().numpy(), ref, f"stacked layer {layer + 1} ({name})")
            if name == "base":
                xb_next = got.to(torch.bfloat16)
            else:
                xp_next = got.to(torch.bfloat16)
        xb, xp = xb_next, xp_next
    diff = (xp.float() - xb.float()).abs().amax(dim=(0, 2, 3)).numpy()
    changed = set(np.nonzero(diff > 1e-3)[0].tolist())
    reach = k_layers * (W - 1)
    assert changed == set(range(t, min(L, t + reach + 1))), (k_layers, sorted(changed))
    swa.device_status()
