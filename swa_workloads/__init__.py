"""Seeded synthetic inputs for the sliding-window GQA attention workloads.

This module is shared by the oracle-side tests and by the GPU path's tests and
benchmark.  It draws random numbers and lays them out; it holds none of the
attention arithmetic (no masks, no slot mapping, no softmax).

Values are drawn as float32 N(0, 1) with ``torch.Generator().manual_seed`` and
rounded to bfloat16 with round-to-nearest-even (``Tensor.to(torch.bfloat16)``).
Both the CUDA path and the oracle receive those same rounded values; the oracle
widens them to float64.

Workloads (Mistral 7B paper, section 2 "Architectural details", and the
Mistral-7B attention shape of 32 query heads, 8 kv heads, head_dim 128):

* ``TINY``        - one layer, batch 1, 12 tokens prefilled as 3 chunks of 4,
                    W=4, Hq=4, Hkv=2, d=16, then 4 decode steps (positions 12-15).
* ``PREFILL_16K`` - batch 1, 16384 tokens, W = chunk = 4096, Hq=32, Hkv=8,
                    d=128, Q drawn N(0,1) then divided by sqrt(128) (so the
                    kernel's scale is 1.0); also run as dense causal attention
                    (W = 16384, one chunk) on the same inputs.
* ``DECODE_B64``  - batch 64, positions uniform in [4096, 32768), cache of
                    W=4096 slots filled with N(0,1) keys/values, 256 steps.
* ``VARLEN``      - 8 prompts, lengths uniform in [1024, 32768], chunk = W = 4096.
* ``DECODE_32L``  - 32 layers of decode at W=4096, positions uniform in
                    [4096, 131072), batch 1, 16, 64 or 128.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import torch

BF16 = torch.bfloat16


@dataclasses.dataclass(frozen=True)
class Shape:
    """Attention shape shared by every call of one workload."""

    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    shape: Shape
    lengths: Tuple[int, ...]          # prompt length of each sequence
    chunk: int                        # tokens per prefill call (<= window)
    scale: float                      # multiplier applied to q.k
    q_prescale: float                 # Q is drawn N(0,1) * q_prescale
    seed: int

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    shape: Shape
    batch: int
    pos_lo: int                       # first positions drawn uniform in [pos_lo, pos_hi)
    pos_hi: int
    steps: int
    layers: int
    scale: float
    seed: int


MISTRAL = Shape(n_q_heads=32, n_kv_heads=8, head_dim=128, window=4096)

TINY_SHAPE = Shape(n_q_heads=4, n_kv_heads=2, head_dim=16, window=4)
TINY_PREFILL = PrefillWorkload("tiny_prefill", TINY_SHAPE, (12,), chunk=4,
                               scale=1.0 / math.sqrt(16), q_prescale=1.0, seed=1)
TINY_DECODE_STEPS = 4

PREFILL_16K = PrefillWorkload("prefill_16k_w4096", MISTRAL, (16384,), chunk=4096,
                              scale=1.0, q_prescale=1.0 / math.sqrt(128), seed=2)
# Same inputs, attention over the whole 16384-token sequence in one call.
DENSE_16K = PrefillWorkload("dense_causal_16k", Shape(32, 8, 128, 16384), (16384,),
                            chunk=16384, scale=1.0, q_prescale=1.0 / math.sqrt(128), seed=2)

DECODE_B64 = DecodeWorkload("decode_b64_w4096", MISTRAL, batch=64, pos_lo=4096,
                            pos_hi=32768, steps=256, layers=1,
                            scale=1.0 / math.sqrt(128), seed=3)

VARLEN_SEED = 4
VARLEN_N = 8
VARLEN_LO, VARLEN_HI = 1024, 32768


def varlen_workload(seed: int = VARLEN_SEED) -> PrefillWorkload:
    """Config 4: 8 prompt lengths uniform in [1024, 32768] (inclusive), chunk = W."""
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(VARLEN_LO, VARLEN_HI + 1, (VARLEN_N,), generator=g)
    return PrefillWorkload("varlen_prefill_8", MISTRAL, tuple(int(x) for x in lengths),
                           chunk=4096, scale=1.0 / math.sqrt(128), q_prescale=1.0,
                           seed=seed)


def decode_32l_workload(batch: int, seed: int = 5) -> DecodeWorkload:
    return DecodeWorkload(f"decode_32layer_b{batch}", MISTRAL, batch=batch, pos_lo=4096,
                          pos_hi=131072, steps=64, layers=32,
                          scale=1.0 / math.sqrt(128), seed=seed)


# ----------------------------------------------------------------------------
# Drawing helpers
# ----------------------------------------------------------------------------

def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape: Sequence[int], g: torch.Generator, device: str = "cpu",
               mul: float = 1.0) -> torch.Tensor:
    """N(0,1) float32 draw, optionally multiplied, rounded to bf16 (RNE)."""
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if mul != 1.0:
        x = x * mul
    return x.to(BF16)


def prefill_inputs(wl: PrefillWorkload, device: str = "cpu"):
    """Full-sequence q/k/v of a prefill workload, padded to the longest prompt.

    Returns (q [B, Lmax, Hq, d], k [B, Lmax, Hkv, d], v [B, Lmax, Hkv, d]) bf16.
    Rows past a sequence's length are zero.
    """
    s = wl.shape
    B, L = wl.batch, max(wl.lengths)
    g = _gen(wl.seed, device)
    q = randn_bf16((B, L, s.n_q_heads, s.head_dim), g, device, wl.q_prescale)
    k = randn_bf16((B, L, s.n_kv_heads, s.head_dim), g, device)
    v = randn_bf16((B, L, s.n_kv_heads, s.head_dim), g, device)
    for b, n in enumerate(wl.lengths):
        if n < L:
            q[b, n:] = 0
            k[b, n:] = 0
            v[b, n:] = 0
    return q, k, v


def tiny_inputs(seed: int = TINY_PREFILL.seed):
    """Config 1 draws: q,k,v for each of the 3 chunks, then q,k,v for each of 4 steps.

    Returns (chunks, steps): chunks is a list of (q [1,4,4,16], k [1,4,2,16],
    v [1,4,2,16]); steps is a list of (q [1,4,16], k [1,2,16], v [1,2,16]).
    """
    s = TINY_SHAPE
    g = _gen(seed)
    chunks = []
    for _ in range(3):
        q = randn_bf16((1, 4, s.n_q_heads, s.head_dim), g)
        k = randn_bf16((1, 4, s.n_kv_heads, s.head_dim), g)
        v = randn_bf16((1, 4, s.n_kv_heads, s.head_dim), g)
        chunks.append((q, k, v))
    steps = []
    for _ in range(TINY_DECODE_STEPS):
        q = randn_bf16((1, s.n_q_heads, s.head_dim), g)
        k = randn_bf16((1, s.n_kv_heads, s.head_dim), g)
        v = randn_bf16((1, s.n_kv_heads, s.head_dim), g)
        steps.append((q, k, v))
    return chunks, steps


def decode_positions(wl: DecodeWorkload, device: str = "cpu") -> torch.Tensor:
    g = _gen(wl.seed * 7919 + 1, "cpu")
    return torch.randint(wl.pos_lo, wl.pos_hi, (wl.batch,), generator=g,
                         dtype=torch.int64).to(torch.int32).to(device)


def decode_cache(wl: DecodeWorkload, layer: int = 0, device: str = "cpu",
                 batch_slice: Optional[slice] = None):
    """A full rolling cache (every slot written) for one layer.

    Returns (k_cache, v_cache), each [B, Hkv, W, d] bf16, N(0,1).  The slot
    that holds a given position is the caller's business; every slot holds a
    finite value.
    """
    s = wl.shape
    g = _gen(wl.seed * 1000003 + 17 * layer + 11, device)
    shape = (wl.batch, s.n_kv_heads, s.window, s.head_dim)
    kc = randn_bf16(shape, g, device)
    vc = randn_bf16(shape, g, device)
    if batch_slice is not None:
        kc, vc = kc[batch_slice].contiguous(), vc[batch_slice].contiguous()
    return kc, vc


def decode_step_inputs(wl: DecodeWorkload, step: int, layer: int = 0, device: str = "cpu"):
    """Fresh (q [B,Hq,d], k_new [B,Hkv,d], v_new [B,Hkv,d]) for one decode step."""
    s = wl.shape
    g = _gen(wl.seed * 1000003 + 104729 * (step + 1) + 31 * layer + 5, device)
    q = randn_bf16((wl.batch, s.n_q_heads, s.head_dim), g, device)
    k = randn_bf16((wl.batch, s.n_kv_heads, s.head_dim), g, device)
    v = randn_bf16((wl.batch, s.n_kv_heads, s.head_dim), g, device)
    return q, k, v


def random_case(seed: int, B: int, L: int, Hq: int, Hkv: int, d: int,
                device: str = "cpu", lengths: Optional[Sequence[int]] = None):
    """Generic small random prefill inputs for tests: q,k,v padded to L rows."""
    g = _gen(seed, device)
    q = randn_bf16((B, L, Hq, d), g, device)
    k = randn_bf16((B, L, Hkv, d), g, device)
    v = randn_bf16((B, L, Hkv, d), g, device)
    if lengths is not None:
        for b, n in enumerate(lengths):
            q[b, n:] = 0
            k[b, n:] = 0
            v[b, n:] = 0
    return q, k, v


