"""Kv-head sharding of one attention layer across ranks (one process per GPU).

Grouped-query attention (Mistral 7B, section 1) ties every query head to one
kv head: query head h reads kv head h // G with G = Hq / Hkv.  So the layer
splits into independent pieces along the kv heads: rank r owns a contiguous
range of kv heads, their rolling caches (Rolling Buffer Cache paragraph of
section 2) and the G query heads of each.  No step of the attention needs data
from another rank; only the caller's output, if it wants all heads in one
place, is gathered (``gather_heads``, an all-gather over the process group,
NCCL on GPUs).

Everything here is bookkeeping: head ranges, per-rank ``Dims`` and contiguous
copies of the head slices.  The attention itself runs in the library's
kernels on each rank's own tensors.
"""
from __future__ import annotations

import dataclasses
from typing import List

import torch

from . import Dims


@dataclasses.dataclass(frozen=True)
class HeadShard:
    """The heads one rank owns: kv heads [kv_lo, kv_hi), query heads [q_lo, q_hi)."""

    rank: int
    world: int
    kv_lo: int
    kv_hi: int
    q_lo: int
    q_hi: int
    dims: Dims

    @property
    def n_kv_heads(self) -> int:
        return self.kv_hi - self.kv_lo

    @property
    def n_q_heads(self) -> int:
        return self.q_hi - self.q_lo


def kv_head_shards(dims: Dims, world: int) -> List[HeadShard]:
    """Contiguous, balanced kv-head ranges for `world` ranks (the first
    Hkv % world ranks take one extra kv head), with the query heads of each kv
    head.  Every rank needs at least one kv head."""
    Hkv, Hq = dims.n_kv_heads, dims.n_q_heads
    if world < 1 or world > Hkv:
        raise ValueError(f"cannot shard {Hkv} kv heads over {world} ranks")
    if Hq % Hkv != 0:
        raise ValueError(f"Hq={Hq} is not a multiple of Hkv={Hkv}")
    G = Hq // Hkv
    base, extra = divmod(Hkv, world)
    shards, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        sub = dataclasses.replace(dims, n_q_heads=(hi - lo) * G, n_kv_heads=hi - lo)
        shards.append(HeadShard(r, world, lo, hi, lo * G, hi * G, sub))
        lo = hi
    return shards


def take_q_heads(x: torch.Tensor, shard: HeadShard) -> torch.Tensor:
    """Query-head slice (q or out: [..., Hq, d]) of this shard, contiguous."""
    return x[..., shard.q_lo:shard.q_hi, :].contiguous()


def take_kv_heads(x: torch.Tensor, shard: HeadShard) -> torch.Tensor:
    """Kv-head slice of a chunk's or a decode step's k/v ([..., Hkv, d]), contiguous."""
    return x[..., shard.kv_lo:shard.kv_hi, :].contiguous()


def take_cache_heads(cache: torch.Tensor, shard: HeadShard) -> torch.Tensor:
    """Kv-head slice of a rolling cache ([B, Hkv, W, d]), contiguous."""
    return cache[:, shard.kv_lo:shard.kv_hi].contiguous()


def concat_heads(outs: List[torch.Tensor]) -> torch.Tensor:
    """Per-rank outputs ([..., Hq_r, d], in rank order) as one [..., Hq, d] tensor."""
    return torch.cat(outs, dim=-2)


def gather_heads(out: torch.Tensor, shards: List[HeadShard], group=None) -> torch.Tensor:
    """All-gather of every rank's output heads over the process group, then
    concat_heads.  Ranks may own different head counts, so each rank's tensor
    is padded to the largest shard for the collective and trimmed after."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if world != len(shards):
        raise ValueError("one shard per rank expected")
    width = max(s.n_q_heads for s in shards)
    pad_shape = list(out.shape)
    pad_shape[-2] = width
    padded = out.new_zeros(pad_shape)
    padded[..., :out.shape[-2], :] = out
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    return concat_heads([p[..., :s.n_q_heads, :] for p, s in zip(parts, shards)])
