"""GPU parity at the workloads' full sizes, on sampled outputs the oracle
computes one by one.

Every workload runs twice: with fp32 outputs, held to the pass bar for
attention outputs from bf16 inputs with fp32 accumulation (max-abs 1e-2,
normalised L1 2e-3), and with bf16 outputs, the launch configuration bench.py
times (one more output rounding; 1e-2 / 4e-3).

* 16K prefill (W = chunk = 4096, 32q/8kv, d = 128): all four chunks, 256
  random query rows per chunk plus the rows at both edges of every 128-row
  tile boundary the chunk starts with and ends with, all 32 heads, plus the
  final cache bytes.
* Dense causal comparator: the same inputs as one 16384-token chunk with
  W = 16384 (the vanilla attention of the pages' 2x claim), sampled rows of
  every query tile including the last one.
* Decode, batch 64, positions in [4096, 32768): all 64 sequences for two steps
  against the oracle's literal rolling cache.
* Variable-length batched prefill (8 prompts of 1024..32768 tokens): sampled
  rows of every chunk of every sequence.
* 32-layer decode: one step through all 32 layers at batch 1, and 8 layers at
  batch 16 (each layer has its own cache and inputs).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from swa_workloads import (DECODE_B64, DENSE_16K, PREFILL_16K, decode_32l_workload, decode_cache,
                           decode_positions, decode_step_inputs, prefill_inputs, varlen_workload)
from tests.gpu_helpers import assert_close, dev_i32

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"
OUT_DTYPES = ["f32", "bf16"]


def sampled_rows_reference(q, k, v, b, rows, W, scale):
    """Oracle output of query rows `rows` of sequence b (positions = row index),
    straight from the definition over the full key history (no cache)."""
    # widen sequence b once; each row then passes contiguous float64 slices
    q, k, v = (x[b:b + 1].double().numpy() for x in (q, k, v))
    b = 0
    outs = []
    for t in rows:
        lo = max(0, t - W + 1)
        pos = np.arange(lo, t + 1)
        o = oracle.attend(q[b, t:t + 1], [t], k[b, lo:t + 1], v[b, lo:t + 1], pos, W, scale)
        outs.append(o[0])
    return np.stack(outs)


def chunk_rows(g, a, b, n_random):
    """Random rows of [a, b) plus both edges of the first and last 128-row tiles."""
    edge = [a, a + 127, a + 128, b - 129, b - 128, b - 1]
    pick = g.choice(np.arange(a, b), n_random, replace=False).tolist()
    return sorted(set(x for x in edge + pick if a <= x < b))


def fill_reference_cache(ref, j, kc, vc, b, pos, W):
    """Oracle cache row j holds positions [pos - W, pos) of sequence b, taken
    from the slots p mod W of the input cache (every slot is written)."""
    k64 = kc[b].double().numpy()
    v64 = vc[b].double().numpy()
    for p in range(max(0, pos - W), pos):
        ref.write(j, p, k64[:, p % W], v64[:, p % W])


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_prefill_16k_full_size(out_dtype):
    wl = PREFILL_16K
    s = wl.shape
    q, k, v = prefill_inputs(wl, "cpu")
    L, W, C = wl.lengths[0], s.window, wl.chunk
    dims = swa.Dims(1, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, out_dtype)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out = torch.empty((1, L, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype, device=DEV)
    kc, vc = swa.new_cache(dims, DEV)
    ws = swa.prefill_workspace(dims, C, DEV)
    for c in range(L // C):
        a, b = c * C, (c + 1) * C
        sp, nt = dev_i32([a]), dev_i32([C])
        swa.prefill_chunk(dims, out[:, a:b], qd[:, a:b], kd[:, a:b], vd[:, a:b], kc, vc, sp, nt,
                          workspace=ws)
        swa.cache_append(dims, kc, vc, kd[:, a:b], vd[:, a:b], sp, nt)
    torch.cuda.synchronize()
    swa.device_status()
    g = np.random.default_rng(2)
    bf = out_dtype == "bf16"
    for c in range(L // C):
        rows = chunk_rows(g, c * C, (c + 1) * C, 256 if not bf else 32)
        ref = sampled_rows_reference(q, k, v, 0, rows, W, wl.scale)
        got = out[0, rows].double().cpu().numpy()
        assert_close(got, ref, f"16k prefill {out_dtype} chunk {c} ({len(rows)} rows)",
                     bf16_out=bf)
    # final cache: positions 12288..16383 in slots p mod 4096
    np.testing.assert_array_equal(kc[0].cpu().transpose(0, 1).float().numpy(),
                                  k[0, L - W:].float().numpy())
    np.testing.assert_array_equal(vc[0].cpu().transpose(0, 1).float().numpy(),
                                  v[0, L - W:].float().numpy())


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_dense_causal_16k_comparator(out_dtype):
    """The call bench.py times as vanilla attention: one chunk of 16384 with
    W = 16384, i.e. causal attention over the whole prompt (128 query tiles,
    up to 128 key tiles per CTA)."""
    wl = DENSE_16K
    s = wl.shape
    q, k, v = prefill_inputs(wl, "cpu")
    L = wl.lengths[0]
    dims = swa.Dims(1, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, wl.scale, out_dtype)
    kc, vc = swa.new_cache(dims, DEV)
    out = torch.empty((1, L, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype, device=DEV)
    ws = swa.prefill_workspace(dims, L, DEV)
    swa.prefill_chunk(dims, out, q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, dev_i32([0]),
                      dev_i32([L]), workspace=ws)
    torch.cuda.synchronize()
    swa.device_status()
    g = np.random.default_rng(16)
    per_tile = 1 if out_dtype == "f32" else 0
    rows = [0, 1, 127, 128, L - 129, L - 128, L - 64, L - 1]
    for qt in range(L // 128):
        rows += (qt * 128 + g.choice(128, per_tile, replace=False)).tolist()
    rows = sorted(set(rows))
    ref = sampled_rows_reference(q, k, v, 0, rows, L, wl.scale)
    got = out[0, rows].double().cpu().numpy()
    assert_close(got, ref, f"dense causal 16k {out_dtype} ({len(rows)} rows)",
                 bf16_out=out_dtype == "bf16")


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_decode_b64_full_size(out_dtype):
    wl = DECODE_B64
    s = wl.shape
    W = s.window
    kc, vc = decode_cache(wl, 0, "cpu")
    pos0 = decode_positions(wl, "cpu").tolist()
    dims = swa.Dims(wl.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, out_dtype)
    check = list(range(wl.batch)) if out_dtype == "f32" else [0, 17, 46, 63]
    ref = oracle.RollingCache(len(check), s.n_kv_heads, W, s.head_dim)
    for j, b in enumerate(check):
        fill_reference_cache(ref, j, kc, vc, b, pos0[b], W)
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    ws = swa.decode_workspace(dims, DEV)
    for step in range(2):
        q, k, v = decode_step_inputs(wl, step, 0, "cpu")
        pos = [p + step for p in pos0]
        out = torch.empty((wl.batch, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype,
                          device=DEV)
        swa.decode(dims, out, q.to(DEV), k.to(DEV), v.to(DEV), kcd, vcd, dev_i32(pos), ws)
        expect = oracle.decode(ref, q[check], k[check], v[check], [pos[b] for b in check],
                               wl.scale)
        assert_close(out[check].double().cpu().numpy(), expect,
                     f"decode b64 {out_dtype} step {step} ({len(check)} sequences)",
                     bf16_out=out_dtype == "bf16")
        for b in check:
            slot = pos[b] % W
            assert torch.equal(kcd[b, :, slot].cpu(), k[b])
            assert torch.equal(vcd[b, :, slot].cpu(), v[b])
    swa.device_status()


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_varlen_prefill_full_size(out_dtype):
    wl = varlen_workload()
    s = wl.shape
    q, k, v = prefill_inputs(wl, "cpu")
    B, L = q.shape[0], q.shape[1]
    W, C = s.window, wl.chunk
    dims = swa.Dims(B, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, out_dtype)
    kc, vc = swa.new_cache(dims, DEV)
    ws = swa.prefill_workspace(dims, C, DEV)
    out = torch.zeros((B, L, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype)
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
        od = torch.zeros((B, C, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype, device=DEV)
        sp, nt = dev_i32([a] * B), dev_i32(counts)
        kg, vg = kcn.to(DEV), vcn.to(DEV)
        swa.prefill_chunk(dims, od, qc.to(DEV), kg, vg, kc, vc, sp, nt, workspace=ws)
        swa.cache_append(dims, kc, vc, kg, vg, sp, nt)
        out[:, a:hi] = od[:, : hi - a].cpu()
    torch.cuda.synchronize()
    swa.device_status()
    g = np.random.default_rng(4)
    per_chunk = 12 if out_dtype == "f32" else 3
    for b, n in enumerate(wl.lengths):
        rows = []
        for a in range(0, n, C):
            hi = min(n, a + C)
            rows += [a, hi - 1] + g.choice(np.arange(a, hi), min(per_chunk, hi - a),
                                           replace=False).tolist()
        rows = sorted(set(rows))
        ref = sampled_rows_reference(q, k, v, b, rows, W, wl.scale)
        assert_close(out[b, rows].double().numpy(), ref,
                     f"varlen {out_dtype} seq {b} (L={n}, {len(rows)} rows)",
                     bf16_out=out_dtype == "bf16")
        # rows past the prompt were never written
        if n < L:
            assert float(out[b, n:].abs().max()) == 0.0


@pytest.mark.parametrize("batch,out_dtype", [(1, "f32"), (1, "bf16"), (16, "f32")])
def test_decode_32_layers_one_step(batch, out_dtype):
    wl = decode_32l_workload(batch)
    s = wl.shape
    W = s.window
    dims = swa.Dims(batch, s.n_q_heads, s.n_kv_heads, s.head_dim, W, wl.scale, out_dtype)
    pos = decode_positions(wl, "cpu").tolist()
    ws = swa.decode_workspace(dims, DEV)
    check = list(range(batch))
    layers = range(wl.layers) if batch == 1 else range(0, wl.layers, 4)
    for layer in layers:
        kc, vc = decode_cache(wl, layer, "cpu")
        q, k, v = decode_step_inputs(wl, 0, layer, "cpu")
        ref = oracle.RollingCache(len(check), s.n_kv_heads, W, s.head_dim)
        for j, b in enumerate(check):
            fill_reference_cache(ref, j, kc, vc, b, pos[b], W)
        kcd, vcd = kc.to(DEV), vc.to(DEV)
        out = torch.empty((batch, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype,
                          device=DEV)
        swa.decode(dims, out, q.to(DEV), k.to(DEV), v.to(DEV), kcd, vcd, dev_i32(pos), ws)
        expect = oracle.decode(ref, q[check], k[check], v[check], [pos[b] for b in check],
                               wl.scale)
        assert_close(out[check].double().cpu().numpy(), expect,
                     f"32-layer decode b{batch} {out_dtype} layer {layer}",
                     bf16_out=out_dtype == "bf16")
    swa.device_status()
