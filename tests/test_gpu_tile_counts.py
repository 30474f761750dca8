"""Checked-mode pin of the prefill's tile handling: the key tiles a CTA loads,
and which (warp, tile) pairs carry masked keys, against counts derived by
brute force from the visibility rule i - W < j <= i (Mistral 7B, section 2,
Sliding Window Attention and Figure 1) and the rolling cache's contents
(Rolling Buffer Cache paragraph, Figure 2) for a chunk that attends to the
cache before its append plus causally to itself (Pre-fill and Chunking,
Figure 3).

The library is rebuilt for this test with -DSWA_TILE_COUNTERS, which makes the
prefill kernel count (0) key tiles loaded, (1) softmax (warp, tile) pairs with
at least one masked key in the warp's rows, (2) pairs with none.  Tiles that
no row can see must never be loaded; a tile is "full" for a warp only if all
32 rows see all 128 of its keys.
"""
import ctypes
import math
import os

import numpy as np
import pytest
import torch

import sliding_window_gqa_chunk_b200 as swa
from sliding_window_gqa_chunk_b200.csrc import build as swa_build

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda"
ROWS = KEYS = 128


@pytest.fixture(scope="module")
def counting_lib():
    so = swa_build.build(force=True, defines=["SWA_TILE_COUNTERS"],
                         out=os.path.join(HERE, "_build", "libswa_tile_counters.so"))
    lib = ctypes.CDLL(so)
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    D = ctypes.POINTER(swa._CDims)
    lib.swa_prefill_chunk.argtypes = [D, P, P, P, P, I32, P, P, P, P, P, ctypes.c_size_t, P]
    lib.swa_prefill_chunk.restype = ctypes.c_int
    lib.swa_device_status.argtypes = [P]
    lib.swa_device_status.restype = ctypes.c_int
    lib.swa_debug_set_trace.argtypes = [P]
    lib.swa_debug_set_trace.restype = None
    return lib


def expected_counts(s, n, T, W, Hq, Hkv):
    """Brute force over rows, keys and tiles of one sequence's chunk call."""
    G = Hq // Hkv
    hpc = 2 if G % 2 == 0 else 1
    groups = Hq // hpc                      # CTAs per query tile
    # rolling cache before the chunk: slot r holds position p(r) < s, or nothing
    slots = np.arange(((W + KEYS - 1) // KEYS) * KEYS)
    if s >= W:
        p_slot = s - W + np.mod(slots - s, W)
    else:
        p_slot = np.where(slots < s, slots, -1)
    p_slot = np.where(slots < W, p_slot, -1)   # tile padding past slot W-1 holds nothing
    loaded = masked = full = 0
    for qt in range((T + ROWS - 1) // ROWS):
        t_lo = qt * ROWS
        if t_lo >= n:
            continue
        t = np.arange(t_lo, t_lo + ROWS)
        i = s + t
        lo = np.maximum(0, i - W + 1)
        tiles = []
        # cache tiles: keys = slots, visible iff the slot's position is in [lo_i, s)
        for k0 in range(0, len(slots), KEYS):
            p = p_slot[k0:k0 + KEYS]
            vis = (p[None, :] >= 0) & (p[None, :] >= lo[:, None]) & (p[None, :] < s)
            if vis.any():
                tiles.append(vis)
        # chunk tiles 0..qt: key t' visible iff t' <= t (t - t' < T <= W)
        for k0 in range(0, (qt + 1) * KEYS, KEYS):
            tk = np.arange(k0, k0 + KEYS)
            tiles.append(tk[None, :] <= t[:, None])
        loaded += len(tiles) * groups
        for vis in tiles:
            for w in range(4):
                any_masked = not vis[32 * w:32 * w + 32].all()
                masked += any_masked * hpc * groups
                full += (not any_masked) * hpc * groups
    return loaded, masked, full


CASES = [
    # s,     n,   T,    W,    Hq, Hkv   (T = max_tokens of the call)
    (0, 256, 256, 256, 8, 2),        # first chunk: causal only
    (256, 256, 256, 256, 8, 2),      # full window, cache full
    (400, 200, 200, 200, 8, 2),      # W not a multiple of 128, wrapped slots
    (337, 100, 100, 256, 12, 4),     # chunk < W, start not a multiple of 128, G = 3
    (90, 50, 64, 256, 4, 2),         # cache not full yet, ragged chunk (n < T)
    (4096, 4096, 4096, 4096, 32, 8),  # the 16K workload's full-window chunk
]


@pytest.mark.parametrize("s,n,T,W,Hq,Hkv", CASES)
def test_tile_classes_match_brute_force(counting_lib, s, n, T, W, Hq, Hkv):
    d = 64
    dims = swa.Dims(1, Hq, Hkv, d, W, 1.0 / math.sqrt(d), "f32")
    g = torch.Generator().manual_seed(s + 7 * n)
    q = torch.randn((1, T, Hq, d), generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn((1, T, Hkv, d), generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn((1, T, Hkv, d), generator=g).to(torch.bfloat16).to(DEV)
    kc, vc = swa.new_cache(dims, DEV)
    out = torch.zeros((1, T, Hq, d), dtype=torch.float32, device=DEV)
    counters = torch.zeros(4, dtype=torch.int32, device=DEV)
    sp = torch.tensor([s], dtype=torch.int32, device=DEV)
    nt = torch.tensor([n], dtype=torch.int32, device=DEV)
    cd = dims.c()
    counting_lib.swa_debug_set_trace(ctypes.c_void_p(counters.data_ptr()))
    try:
        rc = counting_lib.swa_prefill_chunk(
            ctypes.byref(cd), out.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), T,
            kc.data_ptr(), vc.data_ptr(), sp.data_ptr(), nt.data_ptr(), None, 0, None)
        assert rc == 0
        torch.cuda.synchronize()
    finally:
        counting_lib.swa_debug_set_trace(None)
    assert counting_lib.swa_device_status(None) == 0
    got = tuple(int(x) for x in counters[:3].cpu())
    assert got == expected_counts(s, n, T, W, Hq, Hkv)
