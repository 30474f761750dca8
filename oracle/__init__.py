"""Float64 CPU oracle for sliding-window GQA attention over a rolling KV cache.

TEST INFRASTRUCTURE ONLY.  The oracle is what the CUDA path is checked against.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  It shares no code with the CUDA library
(``sliding_window_gqa_chunk_b200``) and neither imports the other; the only
module both sides use is the seeded input generator ``swa_workloads``.

It follows Mistral 7B, section 2 "Architectural details":

* Sliding Window Attention (paragraph and Figure 1 caption): query position i
  sees key positions j with i - W < j <= i, at most W of them.  The arithmetic
  lives in ``swa_oracle.c`` (``swa_oracle_attend``).
* Rolling Buffer Cache (paragraph and Figure 2 caption): a cache of fixed size W;
  the keys and values of time step i are stored at position i mod W, and older
  values are overwritten.  ``RollingCache`` keeps the W slots literally,
  together with the position each slot holds.
* Pre-fill and Chunking (paragraph and Figure 3 caption): a long prompt is cut
  into chunks (chunk size = W); each chunk's attention is computed over the
  cache and over the chunk itself.  ``prefill_chunk`` reads the cache as it was
  before the chunk (the chunk's own keys come from the chunk), and
  ``cache_append`` then writes the chunk into the cache, the same order the
  library's calls use.
* Token-by-token generation: ``decode`` writes the new key/value at slot
  pos mod W and attends over the cache afterwards.

Where the pages are silent or ambiguous (window bounds, GQA grouping,
cache-before-append for chunks, append-before-attend for decode), this module
follows the readings stated above.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile swa_oracle.c into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            lib = ctypes.CDLL(path)
            lib.swa_oracle_attend.restype = ctypes.c_int64
            lib.swa_oracle_attend.argtypes = [
                ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                ctypes.c_double, ctypes.c_void_p, ctypes.c_int]
            lib.swa_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().swa_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Any tensor/array (bf16 torch tensors included) as contiguous float64 numpy."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def attend(q, q_pos, k, v, k_pos, window: int, scale: float,
           n_threads: int = 0) -> np.ndarray:
    """Sliding-window GQA attention of query rows against an explicit key set.

    q [n_q, Hq, d], q_pos [n_q]; k, v [n_k, Hkv, d], k_pos [n_k] (negative =
    empty slot).  Returns out [n_q, Hq, d] float64.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    q_pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64))
    k_pos = np.ascontiguousarray(np.asarray(k_pos, dtype=np.int64))
    n_q, Hq, d = q.shape
    n_k = k.shape[0]
    Hkv = k.shape[1] if n_k else 1
    if n_k:
        assert k.shape == (n_k, Hkv, d) and v.shape == k.shape
    assert Hq % Hkv == 0
    out = np.zeros((n_q, Hq, d), dtype=np.float64)
    if n_q == 0:
        return out
    if n_k == 0:
        k = np.zeros((1, Hkv, d))
        v = np.zeros((1, Hkv, d))
        k_pos = np.full((1,), -1, dtype=np.int64)
    _load().swa_oracle_attend(
        n_q, q.ctypes.data, q_pos.ctypes.data, max(n_k, 1) if n_k else 1,
        k.ctypes.data, v.ctypes.data, k_pos.ctypes.data, Hq, Hkv, d, int(window),
        float(scale), out.ctypes.data, int(n_threads))
    return out


class RollingCache:
    """The rolling buffer cache of Mistral 7B section 2 (Figure 2), kept literally.

    ``k``/``v`` are [B, Hkv, W, d] float64; ``pos`` is [B, W] int64, the absolute
    position each slot holds (-1: never written).  Position p is stored at slot
    p mod W, overwriting what was there.
    """

    def __init__(self, batch: int, n_kv_heads: int, window: int, head_dim: int):
        self.B, self.Hkv, self.W, self.d = batch, n_kv_heads, window, head_dim
        self.k = np.zeros((batch, n_kv_heads, window, head_dim), dtype=np.float64)
        self.v = np.zeros_like(self.k)
        self.pos = np.full((batch, window), -1, dtype=np.int64)

    def slot(self, p: int) -> int:
        return int(p) % self.W

    def write(self, b: int, p: int, k_row, v_row) -> None:
        """Store the [Hkv, d] key/value rows of position p of sequence b."""
        s = self.slot(p)
        self.k[b, :, s, :] = _f64(k_row)
        self.v[b, :, s, :] = _f64(v_row)
        self.pos[b, s] = int(p)

    def keys(self, b: int):
        """(k [W, Hkv, d], v [W, Hkv, d], pos [W]) of sequence b, all slots."""
        return (np.ascontiguousarray(self.k[b].transpose(1, 0, 2)),
                np.ascontiguousarray(self.v[b].transpose(1, 0, 2)),
                self.pos[b].copy())

    def copy(self) -> "RollingCache":
        c = RollingCache(self.B, self.Hkv, self.W, self.d)
        c.k[...] = self.k
        c.v[...] = self.v
        c.pos[...] = self.pos
        return c


def cache_append(cache: RollingCache, k, v, start_pos: Sequence[int],
                 n_tokens: Sequence[int]) -> None:
    """Write rows [0, n_tokens[b]) of k/v [B, T, Hkv, d] at positions start_pos[b]+t."""
    k = _f64(k)
    v = _f64(v)
    for b in range(cache.B):
        for t in range(int(n_tokens[b])):
            cache.write(b, int(start_pos[b]) + t, k[b, t], v[b, t])


def prefill_chunk(cache: RollingCache, q, k, v, start_pos: Sequence[int],
                  n_tokens: Sequence[int], scale: float, n_threads: int = 0) -> np.ndarray:
    """Attention of one prefill chunk over (cache before this chunk) + (the chunk).

    q [B, T, Hq, d], k/v [B, T, Hkv, d]; query row t of sequence b sits at
    position start_pos[b] + t.  Rows t >= n_tokens[b] are left zero.  The cache
    is not modified (``cache_append`` does that, after this call).
    Returns out [B, T, Hq, d] float64.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, T, Hq, d = q.shape
    out = np.zeros((B, T, Hq, d), dtype=np.float64)
    for b in range(B):
        n = int(n_tokens[b])
        if n == 0:
            continue
        s0 = int(start_pos[b])
        ck, cv, cpos = cache.keys(b)
        keys_k = np.concatenate([ck, k[b, :n]], axis=0)
        keys_v = np.concatenate([cv, v[b, :n]], axis=0)
        keys_p = np.concatenate([cpos, s0 + np.arange(n, dtype=np.int64)])
        out[b, :n] = attend(q[b, :n], s0 + np.arange(n, dtype=np.int64),
                            keys_k, keys_v, keys_p, cache.W, scale, n_threads)
    return out


def decode(cache: RollingCache, q, k_new, v_new, pos: Sequence[int], scale: float,
           n_threads: int = 0) -> np.ndarray:
    """One generated token per sequence: append (k_new, v_new) at slot pos mod W,
    then attend q [B, Hq, d] over the cache.  Returns out [B, Hq, d] float64."""
    q = _f64(q)
    k_new = _f64(k_new)
    v_new = _f64(v_new)
    B, Hq, d = q.shape
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        p = int(pos[b])
        cache.write(b, p, k_new[b], v_new[b])
        ck, cv, cpos = cache.keys(b)
        out[b] = attend(q[b][None], np.array([p], dtype=np.int64), ck, cv, cpos,
                        cache.W, scale, n_threads)[0]
    return out


def full_kv_banded(q, k, v, window: int, scale: float,
                   lengths: Optional[Sequence[int]] = None, n_threads: int = 0) -> np.ndarray:
    """Windowed attention straight over the whole sequence, no cache.

    q [B, L, Hq, d], k/v [B, L, Hkv, d]; token t sits at position t.  This is
    the "full KV under the window mask" side of the invariant that rolling-cache
    attention must equal.  Rows past lengths[b] are left zero.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, L, Hq, d = q.shape
    out = np.zeros((B, L, Hq, d), dtype=np.float64)
    for b in range(B):
        n = L if lengths is None else int(lengths[b])
        p = np.arange(n, dtype=np.int64)
        out[b, :n] = attend(q[b, :n], p, k[b, :n], v[b, :n], p, window, scale, n_threads)
    return out


def run_chunked_prefill(q, k, v, window: int, chunk: int, scale: float,
                        lengths: Optional[Sequence[int]] = None, n_threads: int = 0):
    """Prefill whole prompts chunk by chunk through a rolling cache.

    Issues, for c = 0, 1, ..., one prefill_chunk + cache_append over tokens
    [c*chunk, (c+1)*chunk) of every sequence.  Returns (out [B, L, Hq, d], cache).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if lengths is None:
        lengths = [L] * B
    cache = RollingCache(B, Hkv, window, d)
    out = np.zeros((B, L, Hq, d), dtype=np.float64)
    n_calls = max((int(n) + chunk - 1) // chunk for n in lengths)
    for c in range(n_calls):
        st = c * chunk
        starts = [st] * B
        counts = [max(0, min(chunk, int(n) - st)) for n in lengths]
        hi = min(L, st + chunk)
        T = chunk
        qc = np.zeros((B, T, Hq, d))
        kc = np.zeros((B, T, Hkv, d))
        vc = np.zeros((B, T, Hkv, d))
        qc[:, : hi - st] = q[:, st:hi]
        kc[:, : hi - st] = k[:, st:hi]
        vc[:, : hi - st] = v[:, st:hi]
        oc = prefill_chunk(cache, qc, kc, vc, starts, counts, scale, n_threads)
        out[:, st:hi] = oc[:, : hi - st]
        cache_append(cache, kc, vc, starts, counts)
    return out, cache
