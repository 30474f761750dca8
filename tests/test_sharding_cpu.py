"""Kv-head sharding of a layer across ranks (sliding_window_gqa_chunk_b200.sharding):
the partition's invariants, and the output gather over 2 gloo ranks on CPU.

Grouped-query attention (Mistral 7B, section 1) makes every query head read
exactly one kv head (h // G), so contiguous kv-head ranges with their query
heads split the layer into pieces that need nothing from one another."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import sliding_window_gqa_chunk_b200 as swa
from sliding_window_gqa_chunk_b200 import sharding


@pytest.mark.parametrize("Hq,Hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 8), (12, 3, 2),
                                          (16, 16, 5), (8, 1, 1)])
def test_partition_covers_every_head_once(Hq, Hkv, world):
    dims = swa.Dims(3, Hq, Hkv, 128, 4096, 0.1, "bf16")
    shards = sharding.kv_head_shards(dims, world)
    G = Hq // Hkv
    assert [s.rank for s in shards] == list(range(world))
    assert shards[0].kv_lo == 0 and shards[-1].kv_hi == Hkv
    assert shards[0].q_lo == 0 and shards[-1].q_hi == Hq
    for a, b in zip(shards, shards[1:]):
        assert a.kv_hi == b.kv_lo and a.q_hi == b.q_lo       # contiguous, no overlap
    sizes = [s.n_kv_heads for s in shards]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    for s in shards:
        # each query head of the shard reads a kv head of the same shard
        for h in range(s.q_lo, s.q_hi):
            assert s.kv_lo <= h // G < s.kv_hi
        assert s.dims.n_q_heads == s.n_q_heads and s.dims.n_kv_heads == s.n_kv_heads
        assert s.dims.n_q_heads // s.dims.n_kv_heads == G
        assert (s.dims.batch, s.dims.head_dim, s.dims.window) == (3, 128, 4096)


def test_partition_rejects_impossible_splits():
    dims = swa.Dims(1, 8, 2, 64, 64, 0.1)
    with pytest.raises(ValueError):
        sharding.kv_head_shards(dims, 3)
    with pytest.raises(ValueError):
        sharding.kv_head_shards(dims, 0)


def test_head_slices_are_contiguous_copies():
    dims = swa.Dims(2, 12, 3, 16, 8, 0.1)
    s = sharding.kv_head_shards(dims, 2)[1]
    q = torch.arange(2 * 5 * 12 * 16, dtype=torch.float32).reshape(2, 5, 12, 16)
    qs = sharding.take_q_heads(q, s)
    assert qs.is_contiguous() and qs.shape == (2, 5, 4, 16)
    assert torch.equal(qs, q[:, :, 8:12])
    cache = torch.randn(2, 3, 8, 16)
    cs = sharding.take_cache_heads(cache, s)
    assert cs.is_contiguous() and torch.equal(cs, cache[:, 2:3])
    k = torch.randn(2, 5, 3, 16)
    assert torch.equal(sharding.take_kv_heads(k, s), k[:, :, 2:3])


def _free_port():
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def _rank_main(rank, world, port, out_dir, Hq, Hkv):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dims = swa.Dims(2, Hq, Hkv, 4, 16, 0.1)
        shards = sharding.kv_head_shards(dims, world)
        me = shards[rank]
        # this rank's "output": every element holds its global query head index
        out = torch.arange(me.q_lo, me.q_hi, dtype=torch.float32).view(1, -1, 1).expand(2, -1, 4)
        full = sharding.gather_heads(out.contiguous(), shards)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"heads": full[0, :, 0].tolist(), "shape": list(full.shape)}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (12, 3)])
def test_gather_heads_over_two_gloo_ranks(tmp_path, Hq, Hkv):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path), Hq, Hkv), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        with open(tmp_path / f"r{r}.json") as f:
            got = json.load(f)
        assert got["shape"] == [2, Hq, 4]
        assert got["heads"] == [float(h) for h in range(Hq)]
