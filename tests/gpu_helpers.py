"""Shared pieces of the GPU parity tests: running the CUDA path through the
Python binding of the C ABI, and the tolerance check against the oracle.

Tolerances (the same as the pass bar for attention outputs from bf16 inputs
with fp32 accumulation): max |gpu - ref| <= 1e-2 and
sum |gpu - ref| / sum |ref| <= 2e-3, with fp32 outputs.  bf16 outputs carry
one more rounding, of at most half a bf16 ulp of the value (2^-8 relative):
they are held to 4e-3 in the sum, and each element to 1e-2 beyond that
half ulp (an output near 4 alone can be off by 2^-7 after rounding).
"""
import numpy as np
import torch

import sliding_window_gqa_chunk_b200 as swa

MAX_ABS = 1e-2
REL_L1 = 2e-3
REL_L1_BF16_OUT = 4e-3

# (what, max_abs, rel_l1, rel_l1 bar, max_abs bar as text) of every comparison
# made in this session; the conftest prints them at the end of the run so the
# measured errors are on record next to the pass/fail verdict.
MEASURED = []


def rel_l1(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).sum() / max(np.abs(ref).sum(), 1e-300))


def assert_close(got, ref, what="", bf16_out=False):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    rl = rel_l1(got, ref)
    bar = REL_L1_BF16_OUT if bf16_out else REL_L1
    MEASURED.append((what, mx, rl, bar, "1e-2 + half ulp" if bf16_out else "1e-2"))
    excess = err
    if bf16_out and err.size:
        excess = err - bf16_half_ulp(ref)
    mx_excess = float(excess.max()) if err.size else 0.0
    assert mx_excess <= MAX_ABS and rl <= bar, f"{what}: max_abs={mx:.3e} rel_l1={rl:.3e}"
    return mx, rl


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    _, e = np.frexp(a)  # a in [2^(e-1), 2^e)
    return np.ldexp(1.0, e - 9)


def dev_i32(values, device="cuda"):
    return torch.tensor([int(x) for x in values], dtype=torch.int32, device=device)


def gpu_chunked_prefill(dims, q, k, v, lengths, chunk, device="cuda", workspace=True):
    """Prefill padded prompts q/k/v [B, L, H, d] (bf16, CPU) chunk by chunk on
    the GPU (with a prefill workspace, i.e. the persistent split schedule, or
    without one).  Returns (out [B, L, Hq, d] float64 numpy, k_cache, v_cache)."""
    B, L, Hq, d = q.shape
    kc, vc = swa.new_cache(dims, device)
    ws = swa.prefill_workspace(dims, chunk, device) if workspace else None
    out = torch.zeros((B, L, Hq, d), dtype=torch.float64)
    n_calls = max((n + chunk - 1) // chunk for n in lengths)
    for c in range(n_calls):
        st = c * chunk
        counts = [max(0, min(chunk, n - st)) for n in lengths]
        hi = min(L, st + chunk)
        T = chunk
        qc = torch.zeros((B, T, Hq, d), dtype=torch.bfloat16)
        kc_in = torch.zeros((B, T, k.shape[2], d), dtype=torch.bfloat16)
        vc_in = torch.zeros((B, T, k.shape[2], d), dtype=torch.bfloat16)
        qc[:, : hi - st] = q[:, st:hi]
        kc_in[:, : hi - st] = k[:, st:hi]
        vc_in[:, : hi - st] = v[:, st:hi]
        qg, kg, vg = qc.to(device), kc_in.to(device), vc_in.to(device)
        o = torch.zeros((B, T, Hq, d), dtype=dims.torch_out_dtype, device=device)
        sp = dev_i32([st] * B, device)
        nt = dev_i32(counts, device)
        swa.prefill_chunk(dims, o, qg, kg, vg, kc, vc, sp, nt, workspace=ws)
        swa.cache_append(dims, kc, vc, kg, vg, sp, nt)
        out[:, st:hi] = o[:, : hi - st].double().cpu()
    torch.cuda.synchronize()
    swa.device_status()
    return out.numpy(), kc, vc


def cache_as_f64(kc):
    return kc.double().cpu().numpy()
