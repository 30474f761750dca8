"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/swa.h, and rejects bad arguments on the host before it
touches CUDA (so these calls are safe without a device)."""
import ctypes
import os
import re

import pytest

import sliding_window_gqa_chunk_b200 as swa
from sliding_window_gqa_chunk_b200.csrc import build as swa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")

FAKE = 0x10000  # aligned, non-null; never dereferenced because validation fails first


@pytest.fixture(scope="module")
def lib():
    swa_build.build()
    return swa.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"swa_cache_append", "swa_prefill_chunk", "swa_prefill_workspace_size", "swa_decode",
            "swa_decode_workspace_size",
            "swa_last_error", "swa_device_status", "swa_abi_version"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_abi_version(lib):
    assert swa.abi_version() == 200


def test_prefill_workspace_checks(lib):
    d = dims()
    need = lib.swa_prefill_workspace_size(ctypes.byref(d), 128)
    assert need > 0
    assert lib.swa_prefill_workspace_size(ctypes.byref(d), 0) == 0
    assert lib.swa_prefill_workspace_size(ctypes.byref(d), 257) == 0
    p6 = [P()] * 6
    rc = lib.swa_prefill_chunk(ctypes.byref(d), *p6[:4], 128, *p6[4:], P(), P(), P(), need - 1, None)
    assert rc == swa.SWA_ERR_WORKSPACE_TOO_SMALL
    rc = lib.swa_prefill_chunk(ctypes.byref(d), *p6[:4], 128, *p6[4:], P(), P(), P(FAKE + 8), need,
                               None)
    assert rc == swa.SWA_ERR_INVALID_ARG and b"workspace" in lib.swa_last_error()
    rc = lib.swa_prefill_chunk(ctypes.byref(d), *p6[:4], 128, *p6[4:], P(), P(), None, 64, None)
    assert rc == swa.SWA_ERR_INVALID_ARG


def dims(**kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, window=256, scale=0.1,
                out_dtype="f32")
    base.update(kw)
    return swa.Dims(**base).c()


def P(x=FAKE):
    return ctypes.c_void_p(x)


def prefill(lib, d, max_tokens=128, ptrs=None):
    p = ptrs or [P()] * 6
    return lib.swa_prefill_chunk(ctypes.byref(d), p[0], p[1], p[2], p[3], max_tokens, p[4], p[5],
                                 P(), P(), None, 0, None)


@pytest.mark.parametrize("kw,code", [
    (dict(n_q_heads=6, n_kv_heads=4), swa.SWA_ERR_UNSUPPORTED),
    (dict(head_dim=32), swa.SWA_ERR_UNSUPPORTED),
    (dict(head_dim=256), swa.SWA_ERR_UNSUPPORTED),
    (dict(n_q_heads=64, n_kv_heads=2), swa.SWA_ERR_UNSUPPORTED),
    (dict(window=0), swa.SWA_ERR_INVALID_ARG),
    (dict(batch=0), swa.SWA_ERR_INVALID_ARG),
    (dict(scale=0.0), swa.SWA_ERR_INVALID_ARG),
    (dict(scale=-1.0), swa.SWA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), swa.SWA_ERR_INVALID_ARG),
])
def test_bad_dims_rejected_on_host(lib, kw, code):
    d = dims(**kw)
    assert prefill(lib, d) == code
    assert lib.swa_last_error()
    assert lib.swa_decode_workspace_size(ctypes.byref(d)) == 0


def test_bad_out_dtype(lib):
    d = dims()
    d.out_dtype = 7
    assert prefill(lib, d) == swa.SWA_ERR_INVALID_ARG


def test_null_and_misaligned_pointers(lib):
    d = dims()
    for i in range(6):
        ptrs = [P()] * 6
        ptrs[i] = None
        assert prefill(lib, d, ptrs=ptrs) == swa.SWA_ERR_INVALID_ARG
        assert b"NULL" in lib.swa_last_error()
        ptrs[i] = P(FAKE + 8)
        assert prefill(lib, d, ptrs=ptrs) == swa.SWA_ERR_INVALID_ARG
        assert b"aligned" in lib.swa_last_error()
    assert lib.swa_prefill_chunk(ctypes.byref(d), P(), P(), P(), P(), 16, P(), P(), None, P(),
                                 None, 0, None) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_prefill_chunk(None, P(), P(), P(), P(), 16, P(), P(), P(), P(),
                                 None, 0, None) == swa.SWA_ERR_INVALID_ARG


@pytest.mark.parametrize("max_tokens", [0, -3, 257])
def test_chunk_longer_than_window_rejected(lib, max_tokens):
    d = dims()
    assert prefill(lib, d, max_tokens=max_tokens) == swa.SWA_ERR_INVALID_ARG
    assert lib.swa_cache_append(ctypes.byref(d), P(), P(), P(), P(), max_tokens, P(), P(),
                                None) == swa.SWA_ERR_INVALID_ARG


def test_decode_workspace_checks(lib):
    d = dims(batch=1, n_kv_heads=8, n_q_heads=32, window=4096)
    need = lib.swa_decode_workspace_size(ctypes.byref(d))
    assert need > 0
    rc = lib.swa_decode(ctypes.byref(d), P(), P(), P(), P(), P(), P(), P(), P(), need - 1, None)
    assert rc == swa.SWA_ERR_WORKSPACE_TOO_SMALL
    rc = lib.swa_decode(ctypes.byref(d), P(), P(), P(), P(), P(), P(), None, P(), need, None)
    assert rc == swa.SWA_ERR_INVALID_ARG


@pytest.mark.parametrize("B,Hkv,W", [(1, 8, 4096), (64, 8, 4096), (128, 8, 4096), (1, 2, 4),
                                     (3, 1, 100), (16, 8, 4096)])
def test_decode_workspace_is_a_function_of_dims(lib, B, Hkv, W):
    d = dims(batch=B, n_kv_heads=Hkv, n_q_heads=4 * Hkv, window=W)
    a = lib.swa_decode_workspace_size(ctypes.byref(d))
    b = lib.swa_decode_workspace_size(ctypes.byref(d))
    assert a == b and a >= 16
    # at most one fp32 partial (d values + max + sum) per (sequence, head, 64-slot split)
    splits = -(-W // 64)
    assert a <= max(16, B * 4 * Hkv * splits * (128 + 2) * 4)


def test_python_binding_refuses_to_run_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(swa, "_lib", None)
    monkeypatch.setattr(swa, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        swa.load_library()


@pytest.mark.parametrize("B,Hq,Hkv,W,expect", [
    (1, 32, 8, 4096, (8, 1)),     # 8 pairs: a cluster of 8 streaming CTAs per pair, merged in-kernel
    (4, 32, 8, 4096, (4, 1)),     # 32 pairs: clusters of 4, so 128 CTAs run in one wave
    (2, 32, 8, 4096, (6, 1)),     # 16 pairs: a B200 holds 15 clusters of 8 or 7, 22 of 6
    (3, 32, 8, 4096, (5, 1)),     # 24 pairs: 22 clusters of 6 fit, 26 of 5
    (6, 32, 8, 4096, (2, 1)),     # 48 pairs: 45 clusters of 3 fit, 74 of 2
    (8, 32, 8, 4096, (2, 1)),     # 64 pairs: clusters of 2 (74 fit)
    (9, 32, 8, 4096, (2, 1)),     # 72 pairs: clusters of 2
    (10, 32, 8, 4096, (1, 1)),    # 80 pairs: no room for clusters of 2, one CTA per pair
    (16, 32, 8, 4096, (1, 1)),    # 128 pairs (< 148 SMs): one streaming CTA per pair
    (24, 32, 8, 4096, (3, 2)),    # 192 pairs: floor(592 / 192) = 3 splits + combine
    (32, 32, 8, 4096, (2, 2)),    # 256 pairs: 2 splits + combine
    (64, 32, 8, 4096, (1, 1)),    # 512 pairs: one split, no combine
    (128, 32, 8, 4096, (1, 1)),
    (2, 8, 2, 1000, (2, 1)),      # cluster of 2 CTAs (about 512 slots each)
    (2, 8, 2, 300, (1, 1)),       # one CTA covers the window
    (3, 12, 4, 100, (1, 1)),
])
def test_decode_launch_info_follows_the_split_rule(B, Hq, Hkv, W, expect):
    # Without a device the cluster sizes come from the resident-cluster counts
    # of a 148-SM B200 (on a GPU the library asks the device itself).
    d = swa.Dims(B, Hq, Hkv, 128, W, 0.1, "bf16")
    assert swa.decode_launch_info(d) == expect


def test_decode_launch_info_rejects_bad_dims(lib):
    d = dims(batch=1, n_kv_heads=3, n_q_heads=8, window=64)   # Hq % Hkv != 0
    rc = lib.swa_decode_launch_info(ctypes.byref(d), None, None)
    assert rc == swa.SWA_ERR_UNSUPPORTED
