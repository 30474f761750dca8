"""Pins for the float64 oracle: it is checked against things other than itself.

* the worked examples of Mistral 7B section 2 (Figures 1, 2 and 3, written out
  as text fixtures under tests/golden/),
* textbook attention (torch scaled_dot_product_attention in float64) where the
  window covers the whole sequence, and with an explicit band mask,
* the invariant that rolling-cache attention equals full-KV windowed attention,
* a pure-Python brute force on tiny inputs,
* the stacked-layer receptive field of the Figure 1 caption and the closed forms
  of section 2 (8x cache memory at 32k tokens, ~131K span with W = 4096).

A planted-mistake test at the end checks that each plausible mistake in the
oracle's arithmetic (window off by one, wrong head grouping, a dropped term, the
wrong call order, a lost scale) fails at least one of these pins.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from tests.golden_io import read_table

RTOL = 1e-12


def probe_inputs(L, d, Hq=2, Hkv=1, seed=0):
    """Q = 0 (uniform weights over the visible keys), V = one-hot(position)."""
    assert d >= L
    g = torch.Generator().manual_seed(seed)
    q = torch.zeros(1, L, Hq, d, dtype=torch.float64)
    k = torch.randn(1, L, Hkv, d, generator=g, dtype=torch.float64)
    v = torch.zeros(1, L, Hkv, d, dtype=torch.float64)
    for p in range(L):
        v[0, p, :, p] = 1.0
    return q, k, v


def support(out_row):
    return (np.abs(out_row) > 0).astype(np.int64)


def sdpa_reference(q, k, v, mask, scale):
    """torch SDPA in float64 with K/V heads repeated for their query-head group."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    qt = q.permute(0, 2, 1, 3)
    kt = k.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = v.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def band_mask(L, W):
    full = torch.ones(L, L, dtype=torch.bool)
    return torch.tril(full) & ~torch.tril(full, diagonal=-W)


def rand_case(seed, B, L, Hq, Hkv, d):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, L, Hq, d, generator=g, dtype=torch.float64),
            torch.randn(B, L, Hkv, d, generator=g, dtype=torch.float64),
            torch.randn(B, L, Hkv, d, generator=g, dtype=torch.float64))


# ----------------------------------------------------------------------------
# Figures 1-3
# ----------------------------------------------------------------------------

def test_fig1_window_w3_full_kv():
    meta, table = read_table("fig1_window_w3.txt")
    W, L = meta["W"], meta["L"]
    q, k, v = probe_inputs(L, d=L)
    out = oracle.full_kv_banded(q, k, v, W, scale=1.0)
    for h in range(q.shape[2]):
        got = np.stack([support(out[0, i, h]) for i in range(L)])
        np.testing.assert_array_equal(got, table)


def test_fig1_window_w3_through_rolling_cache():
    meta, table = read_table("fig1_window_w3.txt")
    W, L = meta["W"], meta["L"]
    q, k, v = probe_inputs(L, d=L)
    out, _ = oracle.run_chunked_prefill(q, k, v, W, chunk=W, scale=1.0)
    got = np.stack([support(out[0, i, 0]) for i in range(L)])
    np.testing.assert_array_equal(got, table)


def test_fig2_rolling_cache_slots():
    meta, table = read_table("fig2_rolling_cache_w4.txt")
    W = meta["W"]
    cache = oracle.RollingCache(1, 1, W, 2)
    q = np.zeros((1, 1, 2))
    for row in table:
        p, slot, held = int(row[0]), int(row[1]), row[2:]
        assert cache.slot(p) == slot
        oracle.decode(cache, q, np.full((1, 1, 2), p), np.full((1, 1, 2), p), [p], 1.0)
        np.testing.assert_array_equal(cache.pos[0], held)
        # the slot's content is the value written for that position
        assert cache.k[0, 0, slot, 0] == p


def test_fig3_third_chunk_mask():
    meta, table = read_table("fig3_chunk_mask_w4.txt")
    W, C = meta["W"], meta["chunk"]
    L = 3 * C
    q, k, v = probe_inputs(L, d=16)
    cache = oracle.RollingCache(1, 1, W, 16)
    for c in range(3):
        st = c * C
        if c == 2:
            # before the third chunk the cache holds positions 4..7 in slots 0..3
            np.testing.assert_array_equal(cache.pos[0], [4, 5, 6, 7])
        out = oracle.prefill_chunk(cache, q[:, st:st + C], k[:, st:st + C], v[:, st:st + C],
                                   [st], [C], 1.0)
        oracle.cache_append(cache, k[:, st:st + C], v[:, st:st + C], [st], [C])
    got = np.stack([support(out[0, r, 0, :L]) for r in range(C)])
    np.testing.assert_array_equal(got, table)
    # each query of the chunk sees exactly W keys
    assert (table.sum(axis=1) == W).all()


# ----------------------------------------------------------------------------
# Textbook attention
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (6, 1), (8, 2)])
def test_causal_equals_sdpa_when_window_covers_sequence(Hq, Hkv):
    q, k, v = rand_case(11 + Hq + Hkv, 2, 37, Hq, Hkv, 16)
    scale = 1.0 / math.sqrt(16)
    ref = sdpa_reference(q, k, v, band_mask(37, 37), scale)
    causal = torch.nn.functional.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1),
        v.permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1), is_causal=True,
        scale=scale).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(ref, causal, rtol=0, atol=1e-13)
    got = oracle.full_kv_banded(q, k, v, window=64, scale=scale)
    np.testing.assert_allclose(got, causal, rtol=RTOL, atol=1e-12)


@pytest.mark.parametrize("W", [1, 2, 5, 16, 29])
def test_window_equals_sdpa_with_band_mask(W):
    q, k, v = rand_case(100 + W, 2, 41, 8, 2, 8)
    scale = 0.37
    ref = sdpa_reference(q, k, v, band_mask(41, W), scale)
    got = oracle.full_kv_banded(q, k, v, W, scale)
    np.testing.assert_allclose(got, ref, rtol=RTOL, atol=1e-12)


def test_window_one_is_identity_on_values():
    q, k, v = rand_case(5, 1, 9, 4, 2, 8)
    got = oracle.full_kv_banded(q, k, v, window=1, scale=1.0)
    expect = v.numpy().repeat(2, axis=2)
    np.testing.assert_array_equal(got, expect)


def test_first_position_returns_its_value_exactly():
    q, k, v = rand_case(6, 1, 5, 4, 2, 8)
    out, _ = oracle.run_chunked_prefill(q, k, v, window=4, chunk=4, scale=0.5)
    np.testing.assert_array_equal(out[0, 0], v[0, 0].numpy().repeat(2, axis=0))


def test_zero_query_gives_window_mean():
    L, W = 20, 6
    _, k, v = rand_case(7, 1, L, 2, 1, 4)
    q = torch.zeros(1, L, 2, 4, dtype=torch.float64)
    got = oracle.full_kv_banded(q, k, v, W, 1.0)
    for i in range(L):
        lo = max(0, i - W + 1)
        np.testing.assert_allclose(got[0, i, 0], v[0, lo:i + 1, 0].numpy().mean(0),
                                   rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------
# Rolling cache == full KV under the window
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("W,chunk,lengths", [
    (4, 4, [12]), (8, 8, [30, 17, 8, 1]), (16, 16, [50, 33]), (16, 5, [40, 7]),
    (7, 7, [23, 22]), (32, 32, [20]),
])
def test_chunked_rolling_cache_equals_full_kv(W, chunk, lengths):
    L = max(lengths)
    q, k, v = rand_case(200 + W + chunk, len(lengths), L, 4, 2, 8)
    scale = 0.25
    got, _ = oracle.run_chunked_prefill(q, k, v, W, chunk, scale, lengths=lengths)
    ref = oracle.full_kv_banded(q, k, v, W, scale, lengths=lengths)
    np.testing.assert_allclose(got, ref, rtol=RTOL, atol=1e-12)


@pytest.mark.parametrize("W,prompt", [(8, 3), (8, 7), (8, 8), (8, 21), (5, 12)])
def test_decode_equals_last_row_of_full_kv(W, prompt):
    steps = 11
    L = prompt + steps
    q, k, v = rand_case(300 + W + prompt, 2, L, 4, 2, 8)
    scale = 0.3
    _, cache = oracle.run_chunked_prefill(q[:, :prompt], k[:, :prompt], v[:, :prompt],
                                          W, W, scale)
    ref = oracle.full_kv_banded(q, k, v, W, scale)
    for s in range(steps):
        p = prompt + s
        got = oracle.decode(cache, q[:, p], k[:, p], v[:, p], [p, p], scale)
        np.testing.assert_allclose(got, ref[:, p], rtol=RTOL, atol=1e-12)
        # the cache never holds more than W positions, and holds the last min(p+1, W)
        held = sorted(cache.pos[0][cache.pos[0] >= 0].tolist())
        assert held == list(range(max(0, p - W + 1), p + 1))


# ----------------------------------------------------------------------------
# Brute force
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("W,L,Hq,Hkv", [(3, 8, 2, 1), (4, 12, 4, 2), (5, 9, 3, 3)])
def test_brute_force_tiny(W, L, Hq, Hkv):
    q, k, v = rand_case(400 + W, 1, L, Hq, Hkv, 4)
    scale = 0.7
    bf = np.array(brute.attention(q[0].tolist(), k[0].tolist(), v[0].tolist(), W, scale))
    got, _ = oracle.run_chunked_prefill(q, k, v, W, W, scale)
    np.testing.assert_allclose(got[0], bf, rtol=1e-12, atol=1e-13)


def test_brute_force_tiny_workload_bf16_values():
    """Config 1 shape (W=4, Hq=4, Hkv=2, d=16) on its own bf16-rounded draws."""
    from swa_workloads import tiny_inputs, TINY_PREFILL
    chunks, steps = tiny_inputs()
    q = torch.cat([c[0] for c in chunks], 1).double()
    k = torch.cat([c[1] for c in chunks], 1).double()
    v = torch.cat([c[2] for c in chunks], 1).double()
    q = torch.cat([q, torch.stack([s[0] for s in steps], 1).double()], 1)
    k = torch.cat([k, torch.stack([s[1] for s in steps], 1).double()], 1)
    v = torch.cat([v, torch.stack([s[2] for s in steps], 1).double()], 1)
    scale = TINY_PREFILL.scale
    bf = np.array(brute.attention(q[0].tolist(), k[0].tolist(), v[0].tolist(), 4, scale))
    out, cache = oracle.run_chunked_prefill(q[:, :12], k[:, :12], v[:, :12], 4, 4, scale)
    np.testing.assert_allclose(out[0], bf[:12], rtol=1e-12, atol=1e-13)
    for s in range(4):
        p = 12 + s
        o = oracle.decode(cache, q[:, p], k[:, p], v[:, p], [p], scale)
        np.testing.assert_allclose(o[0], bf[p], rtol=1e-12, atol=1e-13)
    # slots of positions 12..15 are 0,1,2,3
    np.testing.assert_array_equal(cache.pos[0], [12, 13, 14, 15])


# ----------------------------------------------------------------------------
# Receptive field and closed forms
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("W,layers,t", [(3, 1, 4), (3, 2, 4), (3, 4, 2), (5, 3, 7)])
def test_receptive_field_of_stacked_layers(W, layers, t):
    """Figure 1 caption: after k layers information moves forward by up to k x W.

    Q = 0 makes each layer a window average; V > 0 chains through the layers.
    Perturbing token t changes exactly positions t .. t + k(W-1), which lies
    inside [t, t + kW]."""
    L = 40
    g = torch.Generator().manual_seed(W * 10 + layers)
    v0 = 1.0 + torch.rand(1, L, 1, 1, generator=g, dtype=torch.float64)
    k = torch.zeros(1, L, 1, 1, dtype=torch.float64)
    q = torch.zeros(1, L, 1, 1, dtype=torch.float64)

    def stack(v):
        x = v
        for _ in range(layers):
            x = torch.from_numpy(oracle.full_kv_banded(q, k, x, W, 1.0))
        return x.numpy()[0, :, 0, 0]

    base = stack(v0)
    v1 = v0.clone()
    v1[0, t] += 0.5
    changed = np.nonzero(stack(v1) != base)[0].tolist()
    reach = layers * (W - 1)
    assert changed == list(range(t, min(L, t + reach + 1)))
    assert max(changed) - t <= layers * W


def test_closed_forms_cache_memory_and_span():
    W, seq = 4096, 32768
    # rolling cache holds W slots whatever the sequence length: 8x less than 32k
    cache_slots = oracle.RollingCache(1, 1, W, 1).k.shape[2]
    assert seq / cache_slots == 8
    # theoretical span at the last of 32 layers: 32 x 4096 ~ 131K tokens
    assert 32 * W == 131072


# ----------------------------------------------------------------------------
# Planted mistakes must fail a pin
# ----------------------------------------------------------------------------

def _mutant_window_plus_one(q, k, v, W, scale):
    return oracle.full_kv_banded(q, k, v, W + 1, scale)


def _mutant_head_modulo(q, k, v, W, scale):
    # kv head h % Hkv instead of h // G: permute query heads around the call
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    perm = [(h % Hkv) * G + (h // Hkv) for h in range(Hq)]
    out = oracle.full_kv_banded(q[:, :, perm], k, v, W, scale)
    inv = np.argsort(perm)
    return out[:, :, inv]


def _mutant_scale_dropped(q, k, v, W, scale):
    return oracle.full_kv_banded(q, k, v, W, 1.0)


def _mutant_k_v_swapped(q, k, v, W, scale):
    return oracle.full_kv_banded(q, v, k, W, scale)


@pytest.mark.parametrize("mutant", [_mutant_window_plus_one, _mutant_head_modulo,
                                    _mutant_scale_dropped, _mutant_k_v_swapped])
def test_planted_mistakes_fail_the_sdpa_pin(mutant):
    q, k, v = rand_case(500, 1, 24, 4, 2, 8)
    W, scale = 5, 0.4
    ref = sdpa_reference(q, k, v, band_mask(24, W), scale)
    got = mutant(q, k, v, W, scale)
    assert np.abs(got - ref).max() > 1e-3


def test_planted_window_mistake_fails_fig1():
    meta, table = read_table("fig1_window_w3.txt")
    q, k, v = probe_inputs(meta["L"], d=meta["L"])
    out = _mutant_window_plus_one(q, k, v, meta["W"], 1.0)
    got = np.stack([support(out[0, i, 0]) for i in range(meta["L"])])
    assert (got != table).any()


def test_planted_cache_mistakes_fail_the_invariant():
    """Dropping the cache, or appending the chunk before attending, breaks
    rolling == full KV (chunk = W, as in the Pre-fill and Chunking paragraph)."""
    W = 8
    q, k, v = rand_case(600, 1, 24, 4, 2, 8)
    ref = oracle.full_kv_banded(q, k, v, W, 0.3)

    def chunked(drop_cache, append_first):
        cache = oracle.RollingCache(1, 2, W, 8)
        out = np.zeros_like(ref)
        for st in range(0, 24, W):
            qc, kc, vc = q[:, st:st + W], k[:, st:st + W], v[:, st:st + W]
            if append_first:
                oracle.cache_append(cache, kc, vc, [st], [W])
            use = oracle.RollingCache(1, 2, W, 8) if drop_cache else cache
            out[:, st:st + W] = oracle.prefill_chunk(use, qc, kc, vc, [st], [W], 0.3)
            if not append_first:
                oracle.cache_append(cache, kc, vc, [st], [W])
        return out

    np.testing.assert_allclose(chunked(False, False), ref, rtol=RTOL, atol=1e-12)
    assert np.abs(chunked(True, False) - ref).max() > 1e-3
    assert np.abs(chunked(False, True) - ref).max() > 1e-3


def test_one_token_chunk_is_a_decode_step():
    # a chunk of one token attends to the cache before its append plus itself:
    # the same keys as a decode step, which appends first (section 2)
    g = np.random.default_rng(9)
    W, Hkv, Hq, d, pos = 8, 2, 4, 16, 13
    q = g.standard_normal((1, 1, Hq, d))
    k = g.standard_normal((1, 1, Hkv, d))
    v = g.standard_normal((1, 1, Hkv, d))
    a = oracle.RollingCache(1, Hkv, W, d)
    for p in range(pos - W + 1, pos):
        a.write(0, p, g.standard_normal((Hkv, d)), g.standard_normal((Hkv, d)))
    b = a.copy()
    pre = oracle.prefill_chunk(a, q, k, v, [pos], [1], 0.25)[0, 0]
    dec = oracle.decode(b, q[:, 0], k[:, 0], v[:, 0], [pos], 0.25)[0]
    np.testing.assert_allclose(pre, dec, rtol=0, atol=1e-14)
