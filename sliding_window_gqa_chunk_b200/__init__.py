"""Sliding-window GQA attention over a rolling KV cache on B200 (sm_100a).

Thin Python binding of ``libswa.so`` (C ABI in ``include/swa.h``).  Each
function takes torch tensors that already live on the GPU, passes their device
pointers and sizes to the C entry point of the same name, and raises
``SwaError`` on a non-zero status.  All computation happens in the library's
CUDA kernels; nothing here computes attention, and there is no CPU fallback:
if the library is missing the import of any entry point fails loudly.

Mistral 7B, section 2 "Architectural details": sliding-window attention with
window W, a rolling buffer cache of W slots (position i in slot i mod W), and
chunked prefill (chunk <= W) followed by token-by-token decoding; query head h
reads kv head h // (Hq // Hkv).

Typical use for one layer::

    dims = Dims(batch=B, n_q_heads=32, n_kv_heads=8, head_dim=128, window=4096,
                scale=128 ** -0.5)
    kc, vc = new_cache(dims)                       # zeroed [B, Hkv, W, d] bf16
    pws = prefill_workspace(dims, max_tokens=4096)  # zeroed, reused by every call
    for chunk ...:                                  # prompt, chunk by chunk
        prefill_chunk(dims, out, q, k, v, kc, vc, start_pos, n_tokens, workspace=pws)
        cache_append(dims, kc, vc, k, v, start_pos, n_tokens)
    ws = decode_workspace(dims)
    decode(dims, out1, q1, k1, v1, kc, vc, pos, ws)  # one token per sequence
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional

import torch

__all__ = [
    "Dims", "SwaError", "load_library", "library_path", "cache_append", "prefill_chunk",
    "decode", "decode_static", "decode_workspace_size", "decode_workspace", "decode_launch_info",
    "prefill_workspace_size", "prefill_workspace", "device_status", "new_cache", "abi_version",
    "SWA_OK", "SWA_ERR_INVALID_ARG", "SWA_ERR_UNSUPPORTED", "SWA_ERR_WORKSPACE_TOO_SMALL",
    "SWA_ERR_CUDA", "SWA_ERR_TIMEOUT", "SWA_ERR_DEVICE_ARG",
]

SWA_OK = 0
SWA_ERR_INVALID_ARG = 1
SWA_ERR_UNSUPPORTED = 2
SWA_ERR_WORKSPACE_TOO_SMALL = 3
SWA_ERR_CUDA = 4
SWA_ERR_TIMEOUT = 5
SWA_ERR_DEVICE_ARG = 6

_DTYPES = {"bf16": 0, "f32": 1}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libswa.so")
_lib = None
_lock = threading.Lock()


class SwaError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"libswa error {code}: {message}")
        self.code = code
        self.message = message


class _CDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("window", ctypes.c_int32), ("scale", ctypes.c_float),
                ("out_dtype", ctypes.c_int32)]


@dataclasses.dataclass(frozen=True)
class Dims:
    """Shape of one attention layer (mirrors ``swa_dims``)."""

    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int
    scale: float
    out_dtype: str = "f32"      # "bf16" or "f32"

    def c(self) -> _CDims:
        return _CDims(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.window,
                      float(self.scale), _DTYPES[self.out_dtype])

    @property
    def torch_out_dtype(self) -> torch.dtype:
        return torch.float32 if self.out_dtype == "f32" else torch.bfloat16


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libswa.so from the package directory (build it with
    ``python -m sliding_window_gqa_chunk_b200.csrc.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m sliding_window_gqa_chunk_b200.csrc.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I32 = ctypes.c_int32
        D = ctypes.POINTER(_CDims)
        lib.swa_cache_append.argtypes = [D, P, P, P, P, I32, P, P, P]
        lib.swa_cache_append.restype = ctypes.c_int
        lib.swa_prefill_workspace_size.argtypes = [D, I32]
        lib.swa_prefill_workspace_size.restype = ctypes.c_size_t
        lib.swa_prefill_chunk.argtypes = [D, P, P, P, P, I32, P, P, P, P, P, ctypes.c_size_t, P]
        lib.swa_prefill_chunk.restype = ctypes.c_int
        lib.swa_decode_workspace_size.argtypes = [D]
        lib.swa_decode_workspace_size.restype = ctypes.c_size_t
        lib.swa_decode_launch_info.argtypes = [D, ctypes.POINTER(I32), ctypes.POINTER(I32)]
        lib.swa_decode_launch_info.restype = ctypes.c_int
        lib.swa_decode.argtypes = [D, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.swa_decode.restype = ctypes.c_int
        lib.swa_decode_static.argtypes = [D, P, P, P, P, P, P, P, P]
        lib.swa_decode_static.restype = ctypes.c_int
        lib.swa_device_status.argtypes = [P]
        lib.swa_device_status.restype = ctypes.c_int
        lib.swa_last_error.argtypes = []
        lib.swa_last_error.restype = ctypes.c_char_p
        lib.swa_abi_version.argtypes = []
        lib.swa_abi_version.restype = ctypes.c_int
        _lib = lib
        return lib


def _check(rc: int) -> None:
    if rc != SWA_OK:
        msg = load_library().swa_last_error().decode(errors="replace")
        raise SwaError(rc, msg)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libswa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def abi_version() -> int:
    return int(load_library().swa_abi_version())


def new_cache(dims: Dims, device="cuda"):
    """Zeroed (k_cache, v_cache), each [B, Hkv, W, d] bf16 (zero = finite for unwritten slots)."""
    shape = (dims.batch, dims.n_kv_heads, dims.window, dims.head_dim)
    return (torch.zeros(shape, dtype=torch.bfloat16, device=device),
            torch.zeros(shape, dtype=torch.bfloat16, device=device))


def cache_append(dims: Dims, k_cache, v_cache, k, v, start_pos, n_tokens, stream=None) -> None:
    """swa_cache_append: k/v [B, T, Hkv, d] bf16 into the [B, Hkv, W, d] caches at slot p mod W."""
    cd = dims.c()
    _check(load_library().swa_cache_append(
        ctypes.byref(cd), _ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v), int(k.shape[1]),
        _ptr(start_pos), _ptr(n_tokens), _stream(stream)))


def prefill_workspace_size(dims: Dims, max_tokens: int) -> int:
    cd = dims.c()
    return int(load_library().swa_prefill_workspace_size(ctypes.byref(cd), int(max_tokens)))


def prefill_workspace(dims: Dims, max_tokens: int, device="cuda") -> torch.Tensor:
    """A zero-filled prefill workspace for these dims (reusable by every later
    call with the same dims on the same stream; calls leave it zero-filled)."""
    return torch.zeros(prefill_workspace_size(dims, max_tokens), dtype=torch.uint8, device=device)


def prefill_chunk(dims: Dims, out, q, k, v, k_cache, v_cache, start_pos, n_tokens,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """swa_prefill_chunk: out [B, T, Hq, d] = attention of chunk q over (cache + chunk k/v).

    ``workspace`` (from ``prefill_workspace``) lets the kernel run persistently
    and split the key ranges of its last query tiles across SMs; without it the
    call launches one CTA per query tile and head pair."""
    cd = dims.c()
    ws_bytes = 0 if workspace is None else int(workspace.numel() * workspace.element_size())
    _check(load_library().swa_prefill_chunk(
        ctypes.byref(cd), _ptr(out), _ptr(q), _ptr(k), _ptr(v), int(q.shape[1]),
        _ptr(k_cache), _ptr(v_cache), _ptr(start_pos), _ptr(n_tokens), _ptr(workspace),
        ws_bytes, _stream(stream)))


def decode_workspace_size(dims: Dims) -> int:
    cd = dims.c()
    return int(load_library().swa_decode_workspace_size(ctypes.byref(cd)))


def decode_workspace(dims: Dims, device="cuda") -> torch.Tensor:
    """A zero-filled decode workspace of decode_workspace_size(dims) bytes."""
    return torch.zeros(decode_workspace_size(dims), dtype=torch.uint8, device=device)


def decode_launch_info(dims: Dims):
    """(n_splits, n_launches) of swa_decode for these dims (host only)."""
    cd = dims.c()
    ns, nl = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load_library().swa_decode_launch_info(ctypes.byref(cd), ctypes.byref(ns), ctypes.byref(nl)))
    return int(ns.value), int(nl.value)


def decode(dims: Dims, out, q, k_new, v_new, k_cache, v_cache, pos, workspace,
           stream=None) -> None:
    """swa_decode: append (k_new, v_new) at slot pos mod W, then out [B, Hq, d] = attention."""
    cd = dims.c()
    _check(load_library().swa_decode(
        ctypes.byref(cd), _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
        _ptr(v_cache), _ptr(pos), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
        _stream(stream)))


def decode_static(dims: Dims, out, q, k_new, v_new, k_cache, v_cache, pos, stream=None) -> None:
    """swa_decode_static: the same decode step as ``decode`` with no workspace argument.

    For callers that cannot allocate device memory (an engine with a fixed,
    pre-planned arena, or code that only receives tensor pointers): the scratch
    comes from a 4 MiB array built into the library, shared by every call on a
    device.  Calls that may overlap on the GPU race on it; the first call on a
    device should come before any stream capture.
    """
    cd = dims.c()
    _check(load_library().swa_decode_static(
        ctypes.byref(cd), _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
        _ptr(v_cache), _ptr(pos), _stream(stream)))


def device_status(stream=None) -> None:
    """Synchronise and raise SwaError if a kernel flagged a timeout or a bad device argument."""
    _check(load_library().swa_device_status(_stream(stream)))
