"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (bf16 outputs), on sampled outputs the oracle computes one by one.

* 16K prefill (W = chunk = 4096, 32q/8kv, d = 128): every chunk, sampled query
  rows of every head, plus the final cache bytes.
* Decode, batch 64, positions in [4096, 32768): two steps, a subset of the
  sequences checked against the oracle's literal rolling cache.
* Variable-length batched prefill (8 prompts of 1024..32768 tokens): sampled
  rows of every chunk of every sequence.
* 32-layer decode: one step through all 32 layers at batch 1, and the first and
  last layer at batch 16 (each layer has its own cache and inputs).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from swa_workloads import (DECODE_B64, PREFILL_16K, decode_32l_workload, decode_cache,
                           decode_positions, decode_step_inputs, prefill_inputs, varlen_workload)
from tests.gpu_helpers import assert_close, dev_i32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def sampled_rows_reference(q, k, v, b, rows, W, scale):
    """Oracle output of query rows `rows` of sequence b (positions = row index),
    straight from the definition over the full key history (no cache)."""
    outs = []
    for t in rows:
        lo = max(0, t - W + 1)
        pos = np.arange(lo, t + 1)
        o = oracle.attend(q[b, t:t + 1], [t], k[b, lo:t + 1], v[b, lo:t + 1], pos, W, scale)
        outs.append(o[0])
    return np.stack(outs)


def test_prefill_16k_full_size_sampled():
    wl = PREFILL_16K
    s = wl.shape
    q, k, v = prefill_inputs(wl, "cpu")
    L, W, C = wl.lengths[0], s.window, wl.chunk
    dims = swa.Dims(1, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, "bf16")
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out = torch.empty((1, L, s.n_q_heads, s.head_dim), dtype=torch.bfloat16, device=DEV)
    kc, vc = swa.new_cache(dims, DEV)
    for c in range(L // C):
        a, b = c * C, (c + 1) * C
        sp, nt = dev_i32([a]), dev_i32([C])
        swa.prefill_chunk(dims, out[:, a:b], qd[:, a:b], kd[:, a:b], vd[:, a:b], kc, vc, sp, nt)
        swa.cache_append(dims, kc, vc, kd[:, a:b], vd[:, a:b], sp, nt)
    torch.cuda.synchronize()
    swa.device_status()
    g = np.random.default_rng(2)
    rows = []
    for c in range(L // C):
        rows += sorted(g.choice(np.arange(c * C, (c + 1) * C), 12, replace=False).tolist())
    rows += [0, 1, C - 1, C, L - 1]
    ref = sampled_rows_reference(q, k, v, 0, rows, W, wl.scale)
    got = out[0, rows].double().cpu().numpy()
    assert_close(got, ref, "16k prefill sampled rows", bf16_out=True)
    # final cache: positions 12288..16383 in slots p mod 4096
    np.testing.assert_array_equal(kc[0].cpu().transpose(0, 1).float().numpy(),
                                  k[0, L - W:].float().numpy())
    np.testing.assert_array_equal(vc[0].cpu().transpose(0, 1).float().numpy(),
                                  v[0, L - W:].float().numpy())


def test_decode_b64_full_size_subset():
    wl = DECODE_B64
    s = wl.shape
    W = s.window
    kc, vc = decode_cache(wl, 0, "cpu")
    pos0 = decode_positions(wl, "cpu").tolist()
    dims = swa.Dims(wl.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, "bf16")
    check = [0, 1, 17, 31, 46, 63]
    ref = oracle.RollingCache(len(check), s.n_kv_heads, W, s.head_dim)
    for j, b in enumerate(check):
        for p in range(pos0[b] - W, pos0[b]):
            ref.write(j, p, kc[b, :, p % W], vc[b, :, p % W])
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    ws = torch.empty(swa.decode_workspace_size(dims), dtype=torch.uint8, device=DEV)
    for step in range(2):
        q, k, v = decode_step_inputs(wl, step, 0, "cpu")
        pos = [p + step for p in pos0]
        out = torch.empty((wl.batch, s.n_q_heads, s.head_dim), dtype=torch.bfloat16, device=DEV)
        swa.decode(dims, out, q.to(DEV), k.to(DEV), v.to(DEV), kcd, vcd, dev_i32(pos), ws)
        expect = oracle.decode(ref, q[check], k[check], v[check], [pos[b] for b in check],
                               wl.scale)
        assert_close(out[check].double().cpu().numpy(), expect, f"decode b64 step {step}",
                     bf16_out=True)
        for j, b in enumerate(check):
            slot = pos[b] % W
            assert torch.equal(kcd[b, :, slot].cpu(), k[b])
            assert torch.equal(vcd[b, :, slot].cpu(), v[b])
    swa.device_status()


def test_varlen_prefill_full_size_sampled():
    wl = varlen_workload()
    s = wl.shape
    q, k, v = prefill_inputs(wl, "cpu")
    B, L = q.shape[0], q.shape[1]
    W, C = s.window, wl.chunk
    dims = swa.Dims(B, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, "bf16")
    kc, vc = swa.new_cache(dims, DEV)
    out = torch.zeros((B, L, s.n_q_heads, s.head_dim), dtype=torch.bfloat16)
    n_calls = max((n + C - 1) // C for n in wl.lengths)
    for c in range(n_calls):
        a = c * C
        counts = [max(0, min(C, n - a)) for n in wl.lengths]
        hi = min(L, a + C)
        qc = torch.zeros((B, C, s.n_q_heads, s.head_dim), dtype=torch.bfloat16)
        kcn = torch.zeros((B, C, s.n_kv_heads, s.head_dim), dtype=torch.bfloat16)
        vcn = torch.zeros_like(kcn)
        qc[:, : hi - a] = q[:, a:hi]
        kcn[:, : hi - a] = k[:, a:hi]
        vcn[:, : hi - a] = v[:, a:hi]
        od = torch.zeros((B, C, s.n_q_heads, s.head_dim), dtype=torch.bfloat16, device=DEV)
        sp, nt = dev_i32([a] * B), dev_i32(counts)
        kg, vg = kcn.to(DEV), vcn.to(DEV)
        swa.prefill_chunk(dims, od, qc.to(DEV), kg, vg, kc, vc, sp, nt)
        swa.cache_append(dims, kc, vc, kg, vg, sp, nt)
        out[:, a:hi] = od[:, : hi - a].cpu()
    torch.cuda.synchronize()
    swa.device_status()
    g = np.random.default_rng(4)
    for b, n in enumerate(wl.lengths):
        rows = sorted(set(g.choice(n, 6, replace=False).tolist() + [0, n - 1]))
        ref = sampled_rows_reference(q, k, v, b, rows, W, wl.scale)
        assert_close(out[b, rows].double().numpy(), ref, f"varlen seq {b} (L={n})", bf16_out=True)
        # rows past the prompt were never written
        if n < L:
            assert float(out[b, n:].abs().max()) == 0.0


@pytest.mark.parametrize("batch", [1, 16])
def test_decode_32_layers_one_step(batch):
    wl = decode_32l_workload(batch)
    s = wl.shape
    W = s.window
    dims = swa.Dims(batch, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, "bf16")
    pos = decode_positions(wl, "cpu").tolist()
    ws = torch.empty(swa.decode_workspace_size(dims), dtype=torch.uint8, device=DEV)
    check = list(range(batch)) if batch <= 2 else [0, batch // 2, batch - 1]
    layers = range(wl.layers) if batch == 1 else [0, wl.layers - 1]
    for layer in layers:
        kc, vc = decode_cache(wl, layer, "cpu")
        q, k, v = decode_step_inputs(wl, 0, layer, "cpu")
        ref = oracle.RollingCache(len(check), s.n_kv_heads, W, s.head_dim)
        for j, b in enumerate(check):
            for p in range(pos[b] - W, pos[b]):
                ref.write(j, p, kc[b, :, p % W], vc[b, :, p % W])
        kcd, vcd = kc.to(DEV), vc.to(DEV)
        out = torch.empty((batch, s.n_q_heads, s.head_dim), dtype=torch.bfloat16, device=DEV)
        swa.decode(dims, out, q.to(DEV), k.to(DEV), v.to(DEV), kcd, vcd, dev_i32(pos), ws)
        expect = oracle.decode(ref, q[check], k[check], v[check], [pos[b] for b in check],
                               wl.scale)
        assert_close(out[check].double().cpu().numpy(), expect, f"layer {layer}",
                     bf16_out=True)
    swa.device_status()
