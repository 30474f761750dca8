"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Bit-exact: cache slot placement (the cache bytes after every append / decode)
and the mask (zero-Q / one-hot-V probe).  Within tolerance (tests/gpu_helpers):
attention outputs.  Shapes span several 128-row tiles, ragged tails, windows
that are not multiples of 128 or smaller than one tile, chunks shorter than
the window (so cache tiles wrap), GQA group sizes 1, 2, 3, 4 and 8, and head
dims 16, 64 and 128.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from swa_workloads import random_case, tiny_inputs, TINY_PREFILL, TINY_SHAPE
from tests.gpu_helpers import (MEASURED, REL_L1, assert_close, cache_as_f64, dev_i32,
                               gpu_chunked_prefill, rel_l1)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def mk_dims(B, Hq, Hkv, d, W, scale=None, out="f32"):
    return swa.Dims(B, Hq, Hkv, d, W, scale if scale is not None else 1.0 / math.sqrt(d), out)


# ----------------------------------------------------------------------------
# Cache append: slot placement is bit-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("d", [16, 64, 128])
def test_append_slot_placement_bit_exact(d):
    B, Hkv, W, T = 3, 2, 64, 40
    dims = mk_dims(B, 4, Hkv, d, W)
    kc, vc = swa.new_cache(dims, DEV)
    ref = oracle.RollingCache(B, Hkv, W, d)
    g = torch.Generator().manual_seed(d)
    calls = [([0, 10, 50], [40, 7, 30]), ([40, 17, 80], [24, 40, 0]), ([64, 57, 80], [1, 33, 39])]
    for starts, counts in calls:
        k = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
        v = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
        swa.cache_append(dims, kc, vc, k.to(DEV), v.to(DEV), dev_i32(starts), dev_i32(counts))
        oracle.cache_append(ref, k, v, starts, counts)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
        np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    swa.device_status()


# ----------------------------------------------------------------------------
# Config 1: 3 chunks of 4 with W = 4, then 4 decode steps
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_tiny_workload_prefill_then_decode(out_dtype):
    s = TINY_SHAPE
    dims = swa.Dims(1, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, TINY_PREFILL.scale,
                    out_dtype)
    chunks, steps = tiny_inputs()
    kc, vc = swa.new_cache(dims, DEV)
    ref = oracle.RollingCache(1, s.n_kv_heads, s.window, s.head_dim)
    bf = out_dtype == "bf16"
    pws = swa.prefill_workspace(dims, 4, DEV)
    for c, (q, k, v) in enumerate(chunks):
        st = 4 * c
        o = torch.zeros((1, 4, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype, device=DEV)
        sp, nt = dev_i32([st]), dev_i32([4])
        swa.prefill_chunk(dims, o, q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, sp, nt, workspace=pws)
        swa.cache_append(dims, kc, vc, k.to(DEV), v.to(DEV), sp, nt)
        expect = oracle.prefill_chunk(ref, q, k, v, [st], [4], dims.scale)
        oracle.cache_append(ref, k, v, [st], [4])
        assert_close(o.double().cpu().numpy(), expect, f"chunk {c}", bf16_out=bf)
        np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
        np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    ws = swa.decode_workspace(dims, DEV)
    for i, (q, k, v) in enumerate(steps):
        p = 12 + i
        o = torch.zeros((1, s.n_q_heads, s.head_dim), dtype=dims.torch_out_dtype, device=DEV)
        swa.decode(dims, o, q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, dev_i32([p]), ws)
        expect = oracle.decode(ref, q, k, v, [p], dims.scale)
        assert_close(o.double().cpu().numpy(), expect, f"step {i}", bf16_out=bf)
        np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
        np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    # positions 12..15 went to slots 0..3
    np.testing.assert_array_equal(ref.pos[0], [12, 13, 14, 15])
    swa.device_status()


# ----------------------------------------------------------------------------
# Mask structure: zero-Q / one-hot-V probe, bit-exact support
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("W,chunk,L,d,Hq,Hkv", [(4, 4, 12, 16, 4, 2), (8, 8, 24, 64, 4, 1),
                                               (8, 5, 23, 64, 2, 2), (16, 16, 120, 128, 8, 2)])
def test_mask_probe_support_bit_exact(W, chunk, L, d, Hq, Hkv):
    """Q = 0 gives equal weights on the visible keys, V = one-hot(position mod d)
    marks them: the set of non-zero output columns is the visible set."""
    g = torch.Generator().manual_seed(W * 100 + L)
    q = torch.zeros(1, L, Hq, d, dtype=torch.bfloat16)
    k = torch.randn(1, L, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.zeros(1, L, Hkv, d, dtype=torch.bfloat16)
    for p in range(L):
        v[0, p, :, p % d] = 1.0
    dims = mk_dims(1, Hq, Hkv, d, W, scale=1.0)
    got, _, _ = gpu_chunked_prefill(dims, q, k, v, [L], chunk)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, chunk, 1.0)
    np.testing.assert_array_equal(got != 0, ref != 0)
    # and each row sees min(i + 1, W) keys when positions are distinct mod d
    if L <= d:
        counts = (got[0, :, 0] != 0).sum(-1)
        np.testing.assert_array_equal(counts, np.minimum(np.arange(L) + 1, W))


# ----------------------------------------------------------------------------
# Prefill against the oracle on random inputs
# ----------------------------------------------------------------------------

PREFILL_CASES = [
    # B, lengths,     W,   chunk, Hq, Hkv, d
    (1, [300],        128, 128,   4,  2,   128),
    (2, [700, 333],   256, 256,   8,  2,   64),
    (1, [520],        512, 512,   2,  2,   128),   # G = 1
    (2, [390, 129],   200, 200,   6,  2,   64),    # G = 3, W not a multiple of 128
    (1, [64],         32,  32,    8,  1,   16),    # G = 8, W below one tile
    (2, [600, 411],   256, 100,   4,  2,   128),   # chunk < W: wrapping cache tiles
    (3, [257, 1, 130], 384, 384,  4,  1,   128),   # ragged, a 1-token prompt
]


@pytest.mark.parametrize("workspace", [True, False], ids=["persistent", "grid"])
@pytest.mark.parametrize("B,lengths,W,chunk,Hq,Hkv,d", PREFILL_CASES)
def test_prefill_matches_oracle(B, lengths, W, chunk, Hq, Hkv, d, workspace):
    L = max(lengths)
    q, k, v = random_case(1000 + W + chunk + d, B, L, Hq, Hkv, d, lengths=lengths)
    dims = mk_dims(B, Hq, Hkv, d, W)
    got, kc, vc = gpu_chunked_prefill(dims, q, k, v, lengths, chunk, workspace=workspace)
    ref, rcache = oracle.run_chunked_prefill(q, k, v, W, chunk, dims.scale, lengths=lengths)
    assert_close(got, ref, f"prefill B={B} L={lengths} W={W} chunk={chunk}")
    np.testing.assert_array_equal(cache_as_f64(kc), rcache.k)
    np.testing.assert_array_equal(cache_as_f64(vc), rcache.v)


# Shapes with few units per call, so the persistent schedule cuts every unit
# that sees at least 8 key tiles into 2-4 pieces of its key range and merges
# them (the path a 4096-token chunk takes for its last wave of units).
SPLIT_CASES = [
    # B, lengths,      W,    chunk, Hq, Hkv, d
    (1, [2304],        2048, 256,   4,  2,   128),   # 4 units per call: 4 pieces each
    (2, [3000, 2100],  2048, 512,   8,  2,   64),    # ragged batch, G = 4
    (1, [1500],        1024, 500,   3,  3,   128),   # G = 1 (one head per CTA), chunk < W
    (1, [700],         1024, 350,   2,  1,   16),    # d = 16
]


@pytest.mark.parametrize("B,lengths,W,chunk,Hq,Hkv,d", SPLIT_CASES)
def test_prefill_split_pieces_match_oracle(B, lengths, W, chunk, Hq, Hkv, d):
    L = max(lengths)
    q, k, v = random_case(2000 + W + chunk + d, B, L, Hq, Hkv, d, lengths=lengths)
    dims = mk_dims(B, Hq, Hkv, d, W)
    got, kc, vc = gpu_chunked_prefill(dims, q, k, v, lengths, chunk, workspace=True)
    ref, rcache = oracle.run_chunked_prefill(q, k, v, W, chunk, dims.scale, lengths=lengths)
    assert_close(got, ref, f"split pieces B={B} L={lengths} W={W} chunk={chunk}")
    np.testing.assert_array_equal(cache_as_f64(kc), rcache.k)


# Score spikes: key kappa is set to alpha times the query of row r (first head of
# its kv group), so that row's score for kappa exceeds everything it has seen by
# about 16 * alpha in log2 units.  Spikes of 4 land far above the 2^32 bound of
# the optimistic exponentials: the tile is redone against the new max, so the
# spike's p is exactly 1.  Spikes of 1.5 stay below it: the row keeps its stale
# max and the spike's p (about 2^19) is rounded to bf16 before the P V product
# while the row sum holds it in fp32.  For a row that one key dominates, that
# rounding moves the output by up to half a bf16 ulp of p relative, i.e.
# 2^-8 |v| -- the same size as rounding the output itself to bf16.  Held to
# that bound (plus 1e-3) element by element and to 2e-3 in the normalised L1.
SPIKES = [  # (row, key, alpha)
    (700, 600, 4.0), (900, 530, 4.0), (1000, 390, 4.0), (610, 230, 4.0),
    (300, 200, 1.5), (1010, 140, 1.5), (820, 700, 1.5),
]


@pytest.mark.parametrize("workspace", [True, False], ids=["persistent", "grid"])
def test_prefill_score_spikes_match_oracle(workspace):
    B, L, W, chunk, Hq, Hkv, d = 1, 1024, 1024, 512, 4, 2, 128
    q, k, v = random_case(4242, B, L, Hq, Hkv, d)
    G = Hq // Hkv
    for r, kappa, alpha in SPIKES:
        assert kappa < r
        for kvh in range(Hkv):
            k[0, kappa, kvh] = (alpha * q[0, r, kvh * G].float()).to(torch.bfloat16)
    dims = mk_dims(B, Hq, Hkv, d, W)
    got, _, _ = gpu_chunked_prefill(dims, q, k, v, [L], chunk, workspace=workspace)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, chunk, dims.scale)
    what = f"score spikes ({'persistent' if workspace else 'grid'})"
    err = np.abs(got - ref)
    rl = rel_l1(got, ref)
    vmax = float(v.abs().max())
    max_bar = 2.0 ** -8 * vmax + 1e-3
    MEASURED.append((what, float(err.max()), rl, REL_L1, f"{max_bar:.2e}"))
    assert np.isfinite(got).all()
    assert float(err.max()) <= max_bar, f"{what}: max_abs={err.max():.3e}"
    assert rl <= REL_L1, f"{what}: rel_l1={rl:.3e}"
    # the rows redone against their spike attend almost only to that key
    for r, kappa, alpha in SPIKES:
        if alpha >= 4.0:
            np.testing.assert_allclose(got[0, r, 0], v[0, kappa, 0].double().numpy(), atol=1e-3)


def test_prefill_bf16_output():
    B, L, W, Hq, Hkv, d = 2, 300, 128, 8, 2, 128
    q, k, v = random_case(77, B, L, Hq, Hkv, d)
    dims = mk_dims(B, Hq, Hkv, d, W, out="bf16")
    got, _, _ = gpu_chunked_prefill(dims, q, k, v, [L, L], W)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, W, dims.scale)
    assert_close(got, ref, "bf16 out", bf16_out=True)


# bf16 output at d = 128: whole 128-row tiles leave through the shared-memory
# staging tile and TMA stores, ragged tiles and merged split pieces from
# registers.  One head per CTA (odd group sizes) and many units per persistent
# CTA exercise the staging tile's hand-over between items.
TMA_STORE_CASES = [
    # B, lengths,                  W,    chunk, Hq, Hkv, workspace
    (4, [2048, 2000, 1500, 777],   1024, 1024,  8,  8,  True),    # G = 1, up to 2 units per CTA
    (4, [2048, 2000, 1500, 777],   1024, 1024,  8,  8,  False),   # the same, one CTA per unit
    (2, [1100, 1300],              1024, 512,   6,  2,  True),    # G = 3, split pieces
    (3, [640, 129, 1024],          256,  256,   8,  2,  True),    # G = 4, two heads per CTA
]


@pytest.mark.parametrize("B,lengths,W,chunk,Hq,Hkv,workspace", TMA_STORE_CASES)
def test_prefill_bf16_output_staged_stores(B, lengths, W, chunk, Hq, Hkv, workspace):
    d = 128
    L = max(lengths)
    q, k, v = random_case(5000 + W + chunk + Hq, B, L, Hq, Hkv, d, lengths=lengths)
    dims = mk_dims(B, Hq, Hkv, d, W, out="bf16")
    got, _, _ = gpu_chunked_prefill(dims, q, k, v, lengths, chunk, workspace=workspace)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, chunk, dims.scale, lengths=lengths)
    assert_close(got, ref, f"bf16 staged stores B={B} L={lengths} W={W} chunk={chunk} G={Hq // Hkv}",
                 bf16_out=True)


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_output_16_byte_aligned(out_dtype, d):
    """The epilogue stores 32 bytes per instruction when the output base is
    32-byte aligned, 16 otherwise: an output 16 bytes past a 32-byte boundary
    gets the same values, bit for bit."""
    B, L, W, Hq, Hkv = 2, 256, 256, 8, 2
    q, k, v = random_case(4242 + d, B, L, Hq, Hkv, d)
    dims = mk_dims(B, Hq, Hkv, d, W, out=out_dtype)
    kc_a, vc_a = swa.new_cache(dims, DEV)
    kc_b, vc_b = swa.new_cache(dims, DEV)
    qg, kg, vg = q.to(DEV), k.to(DEV), v.to(DEV)
    sp, nt = dev_i32([0] * B), dev_i32([L] * B)
    n = B * L * Hq * d
    shift = 16 // torch.empty((), dtype=dims.torch_out_dtype).element_size()
    buf = torch.full((n + 64,), float("nan"), dtype=dims.torch_out_dtype, device=DEV)
    base = (-buf.data_ptr() % 32) // buf.element_size()       # first 32-byte-aligned element
    out_a = buf[base:base + n].view(B, L, Hq, d)
    buf_b = torch.full((n + 64,), float("nan"), dtype=dims.torch_out_dtype, device=DEV)
    off = (-buf_b.data_ptr() % 32) // buf_b.element_size() + shift
    out_b = buf_b[off:off + n].view(B, L, Hq, d)
    assert out_a.data_ptr() % 32 == 0 and out_b.data_ptr() % 32 == 16
    swa.prefill_chunk(dims, out_a, qg, kg, vg, kc_a, vc_a, sp, nt)
    swa.prefill_chunk(dims, out_b, qg, kg, vg, kc_b, vc_b, sp, nt)
    torch.cuda.synchronize()
    swa.device_status()
    assert torch.equal(out_a, out_b)
    ref, _ = oracle.run_chunked_prefill(q, k, v, W, L, dims.scale)
    assert_close(out_b.double().cpu().numpy(), ref, f"16-byte aligned out {out_dtype} d={d}",
                 bf16_out=out_dtype == "bf16")


def test_prefill_chunk_after_decode_steps():
    """A chunk that starts at a position that is not a multiple of 128, after a
    few decode steps, with a cache that is not full yet (unwritten slots are zero)."""
    B, W, Hq, Hkv, d = 2, 256, 4, 2, 128
    first, T = 37, 200
    L = first + T
    q, k, v = random_case(55, B, L, Hq, Hkv, d)
    dims = mk_dims(B, Hq, Hkv, d, W)
    kc, vc = swa.new_cache(dims, DEV)
    ref = oracle.RollingCache(B, Hkv, W, d)
    ws = swa.decode_workspace(dims, DEV)
    for p in range(first):
        o = torch.zeros((B, Hq, d), dtype=torch.float32, device=DEV)
        swa.decode(dims, o, q[:, p].contiguous().to(DEV), k[:, p].contiguous().to(DEV),
                   v[:, p].contiguous().to(DEV), kc, vc, dev_i32([p] * B), ws)
        expect = oracle.decode(ref, q[:, p], k[:, p], v[:, p], [p] * B, dims.scale)
        assert_close(o.double().cpu().numpy(), expect, f"decode {p}")
    o = torch.zeros((B, T, Hq, d), dtype=torch.float32, device=DEV)
    qc, kcn, vcn = (x[:, first:].contiguous() for x in (q, k, v))
    sp, nt = dev_i32([first] * B), dev_i32([T, T - 50])
    swa.prefill_chunk(dims, o, qc.to(DEV), kcn.to(DEV), vcn.to(DEV), kc, vc, sp, nt,
                      workspace=swa.prefill_workspace(dims, T, DEV))
    swa.cache_append(dims, kc, vc, kcn.to(DEV), vcn.to(DEV), sp, nt)
    expect = oracle.prefill_chunk(ref, qc, kcn, vcn, [first] * B, [T, T - 50], dims.scale)
    oracle.cache_append(ref, kcn, vcn, [first] * B, [T, T - 50])
    assert_close(o.double().cpu().numpy(), expect, "chunk after decode")
    np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
    swa.device_status()


def test_positions_near_the_int32_limit():
    """Positions are int32: a cache filled up to just below 2^31 - 1000, a chunk
    there, then decode steps, all against the oracle (slot = position mod W
    with positions near 2^31; no signed 32-bit overflow in any kernel)."""
    B, W, Hq, Hkv, d = 2, 256, 4, 2, 128
    S = [2 ** 31 - 1000, 2 ** 31 - 700]          # chunk starts
    T, n = 200, [200, 150]
    g = torch.Generator().manual_seed(31)
    dims = mk_dims(B, Hq, Hkv, d, W)
    kc, vc = swa.new_cache(dims, DEV)
    ref = oracle.RollingCache(B, Hkv, W, d)
    # the W positions before each chunk, appended in one call
    kf = torch.randn(B, W, Hkv, d, generator=g).to(torch.bfloat16)
    vf = torch.randn(B, W, Hkv, d, generator=g).to(torch.bfloat16)
    starts = [s - W for s in S]
    swa.cache_append(dims, kc, vc, kf.to(DEV), vf.to(DEV), dev_i32(starts), dev_i32([W] * B))
    oracle.cache_append(ref, kf, vf, starts, [W] * B)
    q = torch.randn(B, T, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    o = torch.zeros((B, T, Hq, d), dtype=torch.float32, device=DEV)
    sp, nt = dev_i32(S), dev_i32(n)
    swa.prefill_chunk(dims, o, q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, sp, nt,
                      workspace=swa.prefill_workspace(dims, T, DEV))
    swa.cache_append(dims, kc, vc, k.to(DEV), v.to(DEV), sp, nt)
    expect = oracle.prefill_chunk(ref, q, k, v, S, n, dims.scale)
    oracle.cache_append(ref, k, v, S, n)
    got = o.double().cpu().numpy()
    for b in range(B):   # rows past n_tokens are not written
        assert_close(got[b, : n[b]], expect[b, : n[b]], f"chunk near 2^31, sequence {b}")
    np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
    ws = swa.decode_workspace(dims, DEV)
    for step in range(3):
        pos = [s + m + step for s, m in zip(S, n)]
        qd = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
        kd = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
        vd = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
        od = torch.zeros((B, Hq, d), dtype=torch.float32, device=DEV)
        swa.decode(dims, od, qd.to(DEV), kd.to(DEV), vd.to(DEV), kc, vc, dev_i32(pos), ws)
        expect = oracle.decode(ref, qd, kd, vd, pos, dims.scale)
        assert_close(od.double().cpu().numpy(), expect, f"decode near 2^31, step {step}")
    np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
    np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    swa.device_status()


def test_prefill_chunks_replayed_from_a_cuda_graph():
    """The prefill and append kernels are launched with programmatic dependent
    launch: a CUDA graph of a whole prompt (chunk, append, chunk, append, ...)
    replayed twice gives the eager result bit for bit, and the oracle's."""
    B, L, W, Hq, Hkv, d = 2, 768, 256, 8, 2, 128
    q, k, v = random_case(909, B, L, Hq, Hkv, d)
    dims = mk_dims(B, Hq, Hkv, d, W)
    n = L // W
    qs = [q[:, c * W:(c + 1) * W].contiguous().to(DEV) for c in range(n)]
    ks = [k[:, c * W:(c + 1) * W].contiguous().to(DEV) for c in range(n)]
    vs = [v[:, c * W:(c + 1) * W].contiguous().to(DEV) for c in range(n)]
    sps = [dev_i32([c * W] * B) for c in range(n)]
    nt = dev_i32([W] * B)
    ws = swa.prefill_workspace(dims, W, DEV)

    def prompt(kc, vc, outs):
        for c in range(n):
            swa.prefill_chunk(dims, outs[c], qs[c], ks[c], vs[c], kc, vc, sps[c], nt, workspace=ws)
            swa.cache_append(dims, kc, vc, ks[c], vs[c], sps[c], nt)

    kc_e, vc_e = swa.new_cache(dims, DEV)
    outs_e = [torch.zeros((B, W, Hq, d), dtype=torch.float32, device=DEV) for _ in range(n)]
    prompt(kc_e, vc_e, outs_e)
    torch.cuda.synchronize()
    swa.device_status()

    kc_g, vc_g = swa.new_cache(dims, DEV)
    outs_g = [torch.full((B, W, Hq, d), float("nan"), dtype=torch.float32, device=DEV) for _ in range(n)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            prompt(kc_g, vc_g, outs_g)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        kc_g.zero_()
        vc_g.zero_()
        graph.replay()
        torch.cuda.synchronize()
        swa.device_status()
        for c in range(n):
            assert torch.equal(outs_g[c], outs_e[c]), f"chunk {c}"
        assert torch.equal(kc_g, kc_e) and torch.equal(vc_g, vc_e)
    ref, rcache = oracle.run_chunked_prefill(q, k, v, W, W, dims.scale)
    got = torch.cat([o.double().cpu() for o in outs_g], dim=1).numpy()
    assert_close(got, ref, "prefill from a CUDA graph")
    np.testing.assert_array_equal(cache_as_f64(kc_g), rcache.k)
    del graph


# ----------------------------------------------------------------------------
# Decode against the oracle
# ----------------------------------------------------------------------------

DECODE_CASES = [
    # B, W,    Hq, Hkv, d,   first positions, steps
    (4, 4096, 32, 8, 128, [4096, 5000, 9999, 31000], 3),
    (2, 300, 8, 2, 64, [0, 298], 4),          # empty cache / fills exactly at W-1
    (3, 100, 12, 4, 128, [5, 99, 100000], 3),  # G = 3, far position
    (1, 16, 16, 1, 16, [3], 20),               # G = 16, wraps several times
    (5, 1000, 4, 4, 64, [0, 1, 2, 999, 1000], 2),  # G = 1
    (2, 4096, 64, 8, 128, [70000, 4095], 2),   # G = 8
    # 80 pairs: one streaming CTA per pair, 11 chunks with a partial last one,
    # caches from empty to wrapped
    (10, 700, 16, 8, 64, [0, 5, 699, 700, 1500, 33, 2000, 64, 65, 128], 2),
    (6, 2048, 32, 8, 128, [9000, 2047, 2048, 100, 3000, 4100], 2),  # 48 pairs: clusters of 2
    # clusters sized so that every pair's cluster is resident at once: 16 pairs
    # take clusters of 6 (688 slots per CTA, 656 in the last), 24 pairs of 5
    (2, 4096, 32, 8, 128, [50000, 4097], 2),
    (3, 4096, 32, 8, 128, [4096, 12345, 700], 2),
    # 64 pairs: clusters of 2 (2048 slots each)
    (8, 4096, 32, 8, 128, [4096, 9000, 100, 4095, 20000, 7000, 1, 5000], 2),
    # 8 pairs: clusters of 8 (512 slots per CTA); then a cache holding 101
    # positions, so 7 of the 8 CTAs of each cluster see no slot
    (1, 4096, 32, 8, 128, [40000], 3),
    (1, 4096, 32, 8, 128, [100], 2),
    # 4 pairs: clusters of 8, G = 4
    (1, 4096, 16, 4, 128, [4096], 2),
    # G = 16 (two n-tiles of heads per warp) at d = 128: 8 pairs in clusters of 8
    (4, 4096, 32, 2, 128, [9000, 4096, 100, 20000], 2),
]


@pytest.mark.parametrize("B,W,Hq,Hkv,d,pos0,steps", DECODE_CASES)
def test_decode_matches_oracle(B, W, Hq, Hkv, d, pos0, steps):
    g = torch.Generator().manual_seed(B * 1000 + W + d)
    dims = mk_dims(B, Hq, Hkv, d, W)
    # start from a cache holding positions [max(0, p - W), p) for each sequence
    kc = torch.zeros(B, Hkv, W, d, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    ref = oracle.RollingCache(B, Hkv, W, d)
    for b, p0 in enumerate(pos0):
        for p in range(max(0, p0 - W), p0):
            kr = torch.randn(Hkv, d, generator=g).to(torch.bfloat16)
            vr = torch.randn(Hkv, d, generator=g).to(torch.bfloat16)
            kc[b, :, p % W] = kr
            vc[b, :, p % W] = vr
            ref.write(b, p, kr, vr)
    kc, vc = kc.to(DEV), vc.to(DEV)
    ws = swa.decode_workspace(dims, DEV)
    for s in range(steps):
        pos = [p + s for p in pos0]
        q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
        k = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
        v = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
        o = torch.zeros((B, Hq, d), dtype=torch.float32, device=DEV)
        swa.decode(dims, o, q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, dev_i32(pos), ws)
        expect = oracle.decode(ref, q, k, v, pos, dims.scale)
        assert_close(o.double().cpu().numpy(), expect, f"decode step {s}")
        np.testing.assert_array_equal(cache_as_f64(kc), ref.k)
        np.testing.assert_array_equal(cache_as_f64(vc), ref.v)
    swa.device_status()


def test_decode_bf16_output():
    B, W, Hq, Hkv, d = 3, 512, 32, 8, 128
    g = torch.Generator().manual_seed(9)
    dims = mk_dims(B, Hq, Hkv, d, W, out="bf16")
    kc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, W, d, generator=g).to(torch.bfloat16)
    ref = oracle.RollingCache(B, Hkv, W, d)
    pos = [600, 1023, 5000]
    for b in range(B):
        for p in range(pos[b] - W, pos[b]):
            ref.write(b, p, kc[b, :, p % W], vc[b, :, p % W])
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    kcd, vcd = kc.to(DEV), vc.to(DEV)
    ws = swa.decode_workspace(dims, DEV)
    o = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    swa.decode(dims, o, q.to(DEV), k.to(DEV), v.to(DEV), kcd, vcd, dev_i32(pos), ws)
    expect = oracle.decode(ref, q, k, v, pos, dims.scale)
    assert_close(o.double().cpu().numpy(), expect, "decode bf16", bf16_out=True)


def test_device_status_reports_bad_device_arguments():
    dims = mk_dims(1, 4, 2, 64, 64)
    kc, vc = swa.new_cache(dims, DEV)
    k = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16, device=DEV)
    swa.cache_append(dims, kc, vc, k, k, dev_i32([-5]), dev_i32([8]))
    with pytest.raises(swa.SwaError) as e:
        swa.device_status()
    assert e.value.code == swa.SWA_ERR_DEVICE_ARG
    swa.device_status()  # cleared
    swa.cache_append(dims, kc, vc, k, k, dev_i32([0]), dev_i32([9]))  # n_tokens > max_tokens
    with pytest.raises(swa.SwaError):
        swa.device_status()
    assert float(kc.abs().sum()) == 0.0
