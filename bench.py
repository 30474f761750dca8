"""Benchmark of the sliding-window GQA attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (the headline): single-layer Mistral-7B-shaped chunked prefill, batch
1, 16384 tokens, W = chunk = 4096, 32 query heads over 8 kv heads, head_dim
128, bf16 N(0,1) inputs with Q divided by sqrt(128) (scale 1.0).  One step =
the whole prompt: 4 x (swa_prefill_chunk + swa_cache_append), i.e. slot mapping,
cache append and chunk attention.  `value` is prompt tokens per second.

Alongside, in the same run and with the same step count:
  decode   - batch 64 at positions uniform in [4096, 32768), W = 4096 cache per
             sequence, one swa_decode call per step (tokens/s, HBM GB/s)
  dense    - the same 16384-token inputs as one causal chunk (W = 16384): the
             "vanilla attention" side of the pages' 2x SWA claim
Each reports its kernel's roofline fraction.  Timing: CUDA events on the
launching stream, L2 flushed before every timed step (a 256 MiB write, then a
256 MiB read of another buffer so that the write's dirty lines go back to HBM
before the step), max over ranks.  Under torchrun every rank runs its own replica of the workload (the
path needs no exchange between GPUs), so `value` is the sum over ranks.

--impl reference times the float64 CPU oracle on the same workload and prints
the same JSON line (a bounded sample of query rows per step).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from swa_workloads import (DECODE_B64, PREFILL_16K, decode_32l_workload, decode_cache,  # noqa: E402
                           decode_positions, decode_step_inputs, prefill_inputs, varlen_workload)

METRIC = ("prefill tokens/s & TFLOP/s (% bf16 peak); decode tokens/s & HBM GB/s (% peak)")

# DRAM bytes (read + write) per launch from one ncu capture of each kernel, valid only
# while the kernel source is the one that was profiled (source_key: sha256 prefix of the
# .cu file without comments); the summaries with the commands are under profiles/.
PROFILED_TRAFFIC = {
    "swa_prefill_kernel": {"file": "swa_prefill.cu", "sha": "9664eb26c2605ea5",
                           "bytes": 67_821_312 + 14_862_080,
                           "launch": "chunk 1 of 4 (every row sees 4096 keys)"},
    "swa_decode_kernel": {"file": "swa_decode.cu", "sha": "9924a131379beebb",
                          "bytes": 1_074_292_992 + 3_978_496, "launch": "one decode step"},
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
L2_NOTE = ("flushed before every timed step (outside the timed interval): a 256 MiB write, "
           "then a 256 MiB read of another buffer that writes the flush's dirty lines back")


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def prefill_pairs_per_head(L: int, W: int, chunk: int) -> int:
    """Visible (query, key) pairs of one head over a whole prompt: query i sees
    min(i + 1, W) keys, however the prompt is chunked."""
    return sum(min(i + 1, W) for i in range(L))


def chunk_pairs_per_head(start: int, T: int, W: int) -> int:
    return sum(min(start + t + 1, W) for t in range(T))


class ClockSampler:
    """SM clock and throttle reasons sampled every millisecond (NVML) while active.

    The timed regions last milliseconds, far below nvidia-smi's sampling
    period, so NVML is polled from a thread; nvidia-smi is the fallback.
    """

    NAMES = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
             ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4), ("hw_power_brake", 0x80))

    def __init__(self, gpu_index: int, period_s: float = 0.001):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.sm_max = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self._nvml = (pynvml, h)
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nvml = None
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                self._sample()
                time.sleep(self.period)

        self._sample()
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def _sample(self):
        if self._nvml is not None:
            pynvml, h = self._nvml
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                try:
                    reasons = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
                except Exception:
                    reasons = int(pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h))
                self.samples.append((sm, reasons))
            except Exception:
                pass
            return
        try:
            out = subprocess.run(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=clocks.sm,clocks.max.sm",
                 "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5).stdout
            sm, mx = (float(x) for x in out.strip().split(","))
            self.sm_max = mx
            self.samples.append((sm, 0))
        except Exception:
            pass

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)
        self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["unsampled"]}
        sms = [x[0] for x in self.samples]
        reasons = sorted({name for _, r in self.samples for name, bit in self.NAMES if r & bit})
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.sm_max, "reasons": reasons,
                "samples": len(self.samples), "source": "nvml" if self._nvml else "nvidia-smi"}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, world: int) -> float:
    """Maximum of a per-rank float over all ranks (identity when world == 1)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_key(path: str) -> str:
    """sha256 prefix of a CUDA source with its comments and blank space removed,
    so that an edit of comments alone keeps a profile's record valid."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)   # block comments
    text = re.sub(r"//[^\n]*", " ", text)                 # line comments
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def profiled_traffic(kernel: str):
    """ncu DRAM bytes per launch if the kernel source still matches the profiled one."""
    rec = PROFILED_TRAFFIC[kernel]
    path = os.path.join(ROOT, "sliding_window_gqa_chunk_b200", "csrc", rec["file"])
    try:
        key = source_key(path)
    except OSError:
        return None, None
    if key != rec["sha"]:
        return None, None
    return rec["bytes"], rec["launch"]


def headline_config(wl, world: int) -> dict:
    return {"workload": wl.name, "batch": 1, "seq_len": wl.lengths[0], "window": wl.shape.window,
            "chunk": wl.chunk, "n_q_heads": 32, "n_kv_heads": 8, "head_dim": 128,
            "out_dtype": "bf16", "l2": L2_NOTE,
            "parallelism": f"replicas x{world}"}


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------

class PrefillRun:
    """Chunked prefill of one 16384-token prompt through the C ABI."""

    def __init__(self, wl, out_dtype="bf16", device="cuda"):
        import sliding_window_gqa_chunk_b200 as swa
        self.swa = swa
        s = wl.shape
        self.wl = wl
        self.L = wl.lengths[0]
        self.chunk = wl.chunk
        self.dims = swa.Dims(1, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, wl.scale,
                             out_dtype)
        q, k, v = prefill_inputs(wl, device=device)
        self.q, self.k, self.v = q, k, v
        self.out = torch.empty((1, self.L, s.n_q_heads, s.head_dim), dtype=self.dims.torch_out_dtype,
                               device=device)
        self.kc, self.vc = swa.new_cache(self.dims, device)
        self.ws = swa.prefill_workspace(self.dims, self.chunk, device)
        n_calls = (self.L + self.chunk - 1) // self.chunk
        self.starts = [torch.tensor([c * self.chunk], dtype=torch.int32, device=device)
                       for c in range(n_calls)]
        self.counts = [torch.tensor([min(self.chunk, self.L - c * self.chunk)], dtype=torch.int32,
                                    device=device) for c in range(n_calls)]
        self.n_calls = n_calls
        # per-chunk views (contiguous: batch 1)
        self.views = []
        for c in range(n_calls):
            a, b = c * self.chunk, min(self.L, (c + 1) * self.chunk)
            self.views.append(tuple(x[:, a:b] for x in (self.q, self.k, self.v, self.out)))
        pairs = [chunk_pairs_per_head(c * self.chunk, min(self.chunk, self.L - c * self.chunk),
                                      s.window) for c in range(n_calls)]
        self.flops_per_call = [4.0 * s.head_dim * s.n_q_heads * p for p in pairs]
        self.launches_per_step = 2 * n_calls

    def run_chunk(self, c, events=None):
        """Chunk c: attention over the cache and the chunk, then its append."""
        q, k, v, o = self.views[c]
        if events is not None:
            events[c][0].record()
        self.swa.prefill_chunk(self.dims, o, q, k, v, self.kc, self.vc, self.starts[c], self.counts[c],
                               workspace=self.ws)
        if events is not None:
            events[c][1].record()
        self.swa.cache_append(self.dims, self.kc, self.vc, k, v, self.starts[c], self.counts[c])

    def step(self, events=None):
        # No cache reset between prompts: chunk 0 (start 0) reads nothing from
        # the cache, and chunk c > 0 reads only slots chunk c - 1 rewrote.
        for c in range(self.n_calls):
            self.run_chunk(c, events)


def run_prefill_e2e(run: PrefillRun, steps: int, warmup: int, flush):
    """Same workload through the public API with pinned host buffers: every step
    copies q/k/v host->device and the output device->host inside the timed
    region.  As a user streaming a prompt would, the copies run per chunk on
    their own streams: chunk c+1's inputs go up while chunk c computes, and
    chunk c's output comes down meanwhile (PCIe carries both directions at
    once).  Returns (ms per step, H2D bytes, D2H bytes)."""
    qh = run.q.cpu().pin_memory()
    kh = run.k.cpu().pin_memory()
    vh = run.v.cpu().pin_memory()
    oh = torch.empty(run.out.shape, dtype=run.out.dtype).pin_memory()
    host_views = []
    for c in range(run.n_calls):
        a, b = c * run.chunk, min(run.L, (c + 1) * run.chunk)
        host_views.append(tuple(x[:, a:b] for x in (qh, kh, vh, oh)))
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    times = []
    for i in range(warmup + steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        up.wait_event(e0)
        uploaded = []
        with torch.cuda.stream(up):
            for c in range(run.n_calls):
                q, k, v, _ = run.views[c]
                qh_c, kh_c, vh_c, _ = host_views[c]
                q.copy_(qh_c, non_blocking=True)
                k.copy_(kh_c, non_blocking=True)
                v.copy_(vh_c, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(up)
                uploaded.append(ev)
        for c in range(run.n_calls):
            comp.wait_event(uploaded[c])
            run.run_chunk(c)
            computed = torch.cuda.Event()
            computed.record(comp)
            down.wait_event(computed)
            with torch.cuda.stream(down):
                host_views[c][3].copy_(run.views[c][3], non_blocking=True)
        done = torch.cuda.Event()
        done.record(down)
        comp.wait_event(done)
        e1.record(comp)
        torch.cuda.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()
    return sum(times) / len(times), h2d, d2h


def decode_launches_per_call(dims, swa_mod):
    """Kernels one swa_decode call launches for these dims, as the library
    reports them (swa_decode_launch_info)."""
    return swa_mod.decode_launch_info(dims)[1]


class DecodeRun:
    """One decode step of batch 64 (positions uniform in [4096, 32768))."""

    def __init__(self, wl, out_dtype="bf16", device="cuda"):
        import sliding_window_gqa_chunk_b200 as swa
        self.swa = swa
        s = wl.shape
        self.wl = wl
        self.dims = swa.Dims(wl.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, wl.scale,
                             out_dtype)
        self.kc, self.vc = decode_cache(wl, 0, device=device)
        self.pos0 = decode_positions(wl, device=device)
        self.pos = self.pos0.clone()
        self.inputs = [decode_step_inputs(wl, i, 0, device=device) for i in range(4)]
        self.out = torch.empty((wl.batch, s.n_q_heads, s.head_dim), dtype=self.dims.torch_out_dtype,
                               device=device)
        self.ws = swa.decode_workspace(self.dims, device)
        self.i = 0
        B, W, Hkv, d, Hq = wl.batch, s.window, s.n_kv_heads, s.head_dim, s.n_q_heads
        out_b = 4 if out_dtype == "f32" else 2
        # algorithmic bytes per step: the W cached keys+values of every (seq, kv head),
        # q, the new k/v (read once, written once into the cache), the output
        self.bytes_per_step = B * (2 * W * Hkv * d * 2 + Hq * d * 2 + 2 * Hkv * d * 2 * 2 +
                                   Hq * d * out_b)
        self.launches_per_step = decode_launches_per_call(self.dims, swa)

    def step(self, events=None):
        q, k, v = self.inputs[self.i % len(self.inputs)]
        self.i += 1
        if events is not None:
            events[0][0].record()
        self.swa.decode(self.dims, self.out, q, k, v, self.kc, self.vc, self.pos, self.ws)
        if events is not None:
            events[0][1].record()
        self.pos.add_(1)


class VarlenRun:
    """Batched chunked prefill of 8 prompts (lengths uniform in [1024, 32768]).

    Call c covers tokens [4096 c, 4096 (c + 1)) of every prompt still running;
    the per-call inputs are laid out contiguously before timing."""

    def __init__(self, wl, out_dtype="bf16", device="cuda"):
        import sliding_window_gqa_chunk_b200 as swa
        self.swa = swa
        s = wl.shape
        self.wl = wl
        B, C = wl.batch, wl.chunk
        self.dims = swa.Dims(B, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, wl.scale, out_dtype)
        q, k, v = prefill_inputs(wl, device=device)
        self.kc, self.vc = swa.new_cache(self.dims, device)
        self.ws = swa.prefill_workspace(self.dims, C, device)
        self.n_calls = (max(wl.lengths) + C - 1) // C
        self.calls = []
        flops = 0.0
        for c in range(self.n_calls):
            a = c * C
            counts = [max(0, min(C, n - a)) for n in wl.lengths]
            hi = min(q.shape[1], a + C)
            def take(x):
                buf = torch.zeros((B, C) + tuple(x.shape[2:]), dtype=x.dtype, device=device)
                buf[:, : hi - a] = x[:, a:hi]
                return buf
            qc, kc, vc = take(q), take(k), take(v)
            out = torch.empty((B, C, s.n_q_heads, s.head_dim), dtype=self.dims.torch_out_dtype,
                              device=device)
            sp = torch.tensor([a] * B, dtype=torch.int32, device=device)
            nt = torch.tensor(counts, dtype=torch.int32, device=device)
            self.calls.append((qc, kc, vc, out, sp, nt))
            flops += sum(4.0 * s.head_dim * s.n_q_heads * chunk_pairs_per_head(a, n, s.window)
                         for n in counts if n > 0)
        del q, k, v
        self.flops_per_step = flops
        self.tokens = int(sum(wl.lengths))
        self.launches_per_step = 2 * self.n_calls

    def step(self, events=None):
        for c, (qc, kc, vc, out, sp, nt) in enumerate(self.calls):
            if events is not None:
                events[c][0].record()
            self.swa.prefill_chunk(self.dims, out, qc, kc, vc, self.kc, self.vc, sp, nt,
                                   workspace=self.ws)
            if events is not None:
                events[c][1].record()
            self.swa.cache_append(self.dims, self.kc, self.vc, kc, vc, sp, nt)


class Decode32Run:
    """One decode step through 32 layers (each with its own W = 4096 cache),
    replayed as a CUDA graph of the 32 swa_decode calls."""

    def __init__(self, wl, out_dtype="bf16", device="cuda"):
        import sliding_window_gqa_chunk_b200 as swa
        self.swa = swa
        s = wl.shape
        self.wl = wl
        B = wl.batch
        self.dims = swa.Dims(B, s.n_q_heads, s.n_kv_heads, s.head_dim, s.window, wl.scale, out_dtype)
        g = torch.Generator(device=device)
        g.manual_seed(wl.seed)
        shape = (B, s.n_kv_heads, s.window, s.head_dim)
        self.caches = []
        for _ in range(wl.layers):
            kc = torch.randn(shape, generator=g, device=device, dtype=torch.bfloat16)
            vc = torch.randn(shape, generator=g, device=device, dtype=torch.bfloat16)
            self.caches.append((kc, vc))
        self.q = torch.randn((B, s.n_q_heads, s.head_dim), generator=g, device=device, dtype=torch.bfloat16)
        self.k = torch.randn((B, s.n_kv_heads, s.head_dim), generator=g, device=device, dtype=torch.bfloat16)
        self.v = torch.randn((B, s.n_kv_heads, s.head_dim), generator=g, device=device, dtype=torch.bfloat16)
        self.out = torch.empty((B, s.n_q_heads, s.head_dim), dtype=self.dims.torch_out_dtype, device=device)
        self.pos = decode_positions(wl, device=device)
        self.ws = swa.decode_workspace(self.dims, device)
        out_b = 4 if out_dtype == "f32" else 2
        per_layer = B * (2 * s.window * s.n_kv_heads * s.head_dim * 2 + s.n_q_heads * s.head_dim * 2 +
                         2 * s.n_kv_heads * s.head_dim * 2 * 2 + s.n_q_heads * s.head_dim * out_b)
        self.bytes_per_step = wl.layers * per_layer
        self.graph = None
        self.launches_per_step = wl.layers * decode_launches_per_call(self.dims, swa) + 1

    def _layers(self):
        for kc, vc in self.caches:
            self.swa.decode(self.dims, self.out, self.q, self.k, self.v, kc, vc, self.pos, self.ws)
        self.pos.add_(1)

    def capture(self):
        self._layers()                       # first calls on the device happen outside capture
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._layers()
        torch.cuda.synchronize()

    def step(self, events=None):
        if events is not None:
            events[0][0].record()
        self.graph.replay()
        if events is not None:
            events[0][1].record()

    def release(self):
        self.graph = None
        self.caches = None


def time_steps(fn, steps, warmup, flush, n_events=1):
    """Per-step CUDA-event timing with an L2 flush before every step (outside the
    timed interval).  Returns (mean step ms, mean per-event-pair ms list)."""
    for _ in range(warmup):
        flush()
        fn(None)
    torch.cuda.synchronize()
    step_ms, pair_ms = [], [[] for _ in range(n_events)]
    for _ in range(steps):
        flush()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_events)]
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        fn(ev)
        s1.record()
        torch.cuda.synchronize()
        step_ms.append(s0.elapsed_time(s1))
        for i, (a, b) in enumerate(ev):
            pair_ms[i].append(a.elapsed_time(b))
    return (sum(step_ms) / len(step_ms),
            [sum(x) / len(x) for x in pair_ms])


def bench_ours(args, world, rank, local):
    import sliding_window_gqa_chunk_b200 as swa
    from sliding_window_gqa_chunk_b200.csrc import build as swa_build
    swa_build.build()
    swa.load_library()
    dev = f"cuda:{local}"
    peaks = load_peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    evict_buf = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    phase = args.phase

    def flush():
        # a write larger than L2 evicts everything; reading another buffer
        # larger than L2 then evicts the dirty lines of that write, so their
        # write-back to HBM happens here and not inside the next timed step
        flush_buf.fill_(1)
        evict_buf.max()

    wl = PREFILL_16K
    line = {
        "metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": headline_config(wl, world),
    }
    if phase != "all":
        line["phase"] = phase

    run = None
    kernel_ms = None
    if phase in ("all", "prefill", "dense"):
        run = PrefillRun(wl, "bf16", dev)
    if phase in ("all", "prefill"):
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            ms, per_call = time_steps(lambda ev: run.step(ev), args.steps, args.warmup, flush,
                                      n_events=run.n_calls)
        torch.cuda.synchronize()
        barrier(world)
        ms_max = reduce_max(ms, world)
        swa.device_status()
        flops_step = sum(run.flops_per_call)
        kernel_ms = sum(per_call)                   # prefill kernel time per step
        avg_launch_ms = kernel_ms / run.n_calls
        avg_flops = flops_step / run.n_calls
        achieved = avg_flops / (avg_launch_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        line.update({
            "value": round(world * run.L / (ms_max / 1e3), 1),
            "ms_per_step": round(ms_max, 4),
            "tflops": round(flops_step / (ms_max / 1e3) / 1e12, 1),
            "roofline": {"kernel": "swa_prefill_kernel", "bound": "tensor",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4),
                         "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                         "algorithmic_flops_per_launch": avg_flops,
                         "launch_ms": [round(x, 4) for x in per_call],
                         "traffic": profiled_traffic("swa_prefill_kernel")[0],
                         "traffic_launch": profiled_traffic("swa_prefill_kernel")[1]},
            "gpu_launches": run.launches_per_step * args.steps,
            "clocks": clk.summary(),
        })

    if phase in ("all", "decode"):
        dec = DecodeRun(DECODE_B64, "bf16", dev)
        barrier(world)
        with ClockSampler(local) as dclk:
            dms, dpair = time_steps(lambda ev: dec.step(ev), args.steps, args.warmup, flush,
                                    n_events=1)
        barrier(world)
        dms_max = reduce_max(dms, world)
        dec_kernel_ms = dpair[0]
        dec_gbs = dec.bytes_per_step / (dec_kernel_ms / 1e3) / 1e9
        swa.device_status()
        dec_line = {
            "workload": DECODE_B64.name, "batch": DECODE_B64.batch,
            "tokens_per_s": round(world * DECODE_B64.batch / (dms_max / 1e3), 1),
            "ms_per_step": round(dms_max, 4),
            "roofline": {"kernel": "swa_decode_kernel" + (" (+ combine)" if dec.launches_per_step > 1 else ""),
                         "bound": "hbm",
                         "achieved": round(dec_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(dec_gbs / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peaks['source']} hbm_gbs",
                         "algorithmic_bytes_per_launch": dec.bytes_per_step,
                         "launch_ms": round(dec_kernel_ms, 4),
                         "traffic": profiled_traffic("swa_decode_kernel")[0]},
            "gpu_launches_per_step": dec.launches_per_step,
            "clocks": dclk.summary(),
        }
        line["decode"] = dec_line
        if phase == "decode":
            line.update({"value": dec_line["tokens_per_s"], "ms_per_step": dec_line["ms_per_step"],
                         "roofline": dec_line["roofline"], "clocks": dec_line["clocks"],
                         "gpu_launches": dec.launches_per_step * args.steps})
            line["config"] = {"workload": DECODE_B64.name, "batch": DECODE_B64.batch,
                              "window": 4096, "n_q_heads": 32, "n_kv_heads": 8, "head_dim": 128,
                              "out_dtype": "bf16", "l2": line["config"]["l2"],
                              "parallelism": f"replicas x{world}"}

    if phase in ("all", "dense"):
        # dense causal comparator on the same inputs: one chunk of 16384, W = 16384
        dense_dims = swa.Dims(1, 32, 8, 128, 16384, wl.scale, "bf16")
        dkc, dvc = swa.new_cache(dense_dims, dev)
        dws = swa.prefill_workspace(dense_dims, 16384, dev)
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        full = torch.tensor([16384], dtype=torch.int32, device=dev)

        def dense_step(ev):
            if ev is not None:
                ev[0][0].record()
            swa.prefill_chunk(dense_dims, run.out, run.q, run.k, run.v, dkc, dvc, zero, full,
                              workspace=dws)
            if ev is not None:
                ev[0][1].record()

        _, dense_pair = time_steps(dense_step, max(2, args.steps // 2), 2, flush, n_events=1)
        dense_flops = 4.0 * 128 * 32 * prefill_pairs_per_head(16384, 16384, 16384)
        swa.device_status()
        line["dense"] = {"workload": "dense_causal_16k", "ms": round(dense_pair[0], 4),
                         "tflops": round(dense_flops / (dense_pair[0] / 1e3) / 1e12, 1)}
        if kernel_ms:
            line["dense"]["swa_speedup_vs_dense"] = round(dense_pair[0] / kernel_ms, 3)

    if phase in ("all", "varlen"):
        vr = VarlenRun(varlen_workload(), "bf16", dev)
        barrier(world)
        vms, vpair = time_steps(lambda ev: vr.step(ev), max(3, args.steps // 2), 2, flush,
                                n_events=vr.n_calls)
        vms_max = reduce_max(vms, world)
        swa.device_status()
        vk = sum(vpair)
        line["varlen"] = {
            "workload": vr.wl.name, "lengths": list(vr.wl.lengths),
            "tokens_per_s": round(world * vr.tokens / (vms_max / 1e3), 1),
            "ms_per_step": round(vms_max, 4),
            "tflops": round(vr.flops_per_step / (vms_max / 1e3) / 1e12, 1),
            "roofline": {"kernel": "swa_prefill_kernel", "bound": "tensor",
                         "achieved": round(vr.flops_per_step / (vk / 1e3) / 1e12, 1),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(vr.flops_per_step / (vk / 1e3) / 1e12 / peaks["bf16_tflops"], 4)},
            "gpu_launches_per_step": vr.launches_per_step}
        del vr
        torch.cuda.empty_cache()

    if phase in ("all", "decode32"):
        rows = []
        for B in args.batches:
            dr = Decode32Run(decode_32l_workload(B), "bf16", dev)
            dr.capture()
            barrier(world)
            dms32, dpair32 = time_steps(lambda ev: dr.step(ev), args.steps, args.warmup, flush,
                                        n_events=1)
            dms32 = reduce_max(dms32, world)
            swa.device_status()
            gbs = dr.bytes_per_step / (dpair32[0] / 1e3) / 1e9
            rows.append({"batch": B, "tokens_per_s": round(world * B / (dms32 / 1e3), 1),
                         "ms_per_step": round(dms32, 4),
                         "hbm_gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "gpu_launches_per_step": dr.launches_per_step})
            dr.release()
            del dr
            torch.cuda.empty_cache()
        line["decode_32layer"] = {"workload": "decode_32layer_w4096 (CUDA graph of 32 layer calls)",
                                  "roofline_peak_gbs": peaks["hbm_gbs"], "rows": rows}

    if phase in ("all", "prefill"):
        # end to end through the public API with host buffers
        e2e_ms, h2d, d2h = run_prefill_e2e(run, args.steps, 3, flush)
        e2e_ms = reduce_max(e2e_ms, world)
        line["e2e"] = {"value": round(world * run.L / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(e2e_ms, 4)}
        if rank == 0 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return line


# ----------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------

def oracle_rows(wl, seed: int = 0):
    """Query rows of the whole prompt in a seeded random order: timing the
    oracle on a prefix of this list samples every chunk in proportion to its
    rows, each row with its own min(i + 1, W) keys, so rows / second estimates
    the whole prompt's rate."""
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(wl.lengths[0], generator=g).tolist()


def oracle_inputs(wl):
    """The workload's q/k/v widened once to float64 numpy (outside any timing)."""
    q, k, v = prefill_inputs(wl, device="cpu")
    return tuple(x.double().numpy() for x in (q, k, v))


def oracle_sample(wl, rows, q, k, v):
    """The oracle on the given query rows (all heads, each row against its
    window of keys from the full history; float64 inputs): returns seconds."""
    import numpy as np
    import oracle
    W = wl.shape.window
    t0 = time.perf_counter()
    for i in rows:
        lo = max(0, i - W + 1)
        oracle.attend(q[0, i:i + 1], [i], k[0, lo:i + 1], v[0, lo:i + 1], np.arange(lo, i + 1), W,
                      wl.scale)
    return time.perf_counter() - t0


def sample_note(n_rows, wl):
    return (f"{n_rows} query tokens drawn uniformly at random from the {wl.lengths[0]}-token prompt "
            f"(all 32 heads, each row against its own min(i+1, {wl.shape.window}) keys), float64 C "
            f"oracle, OpenMP over heads")


def cpu_baseline(wl, budget_s=12.0):
    import oracle
    q, k, v = oracle_inputs(wl)
    order = oracle_rows(wl)
    done, spent, batch = 0, 0.0, 32
    while spent < budget_s and done + batch <= len(order):
        spent += oracle_sample(wl, order[done:done + batch], q, k, v)
        done += batch
    return {"value": round(done / spent, 2), "unit": "tokens/s", "cores": oracle.max_threads(),
            "kind": "oracle", "sample": sample_note(done, wl)}


def bench_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    wl = PREFILL_16K
    q, k, v = oracle_inputs(wl)
    rows = args.ref_rows
    order = oracle_rows(wl, seed=1)
    for i in range(args.warmup):
        oracle_sample(wl, order[i * rows:(i + 1) * rows], q, k, v)
    times = []
    for i in range(args.steps):
        a = ((args.warmup + i) * rows) % len(order)
        times.append(oracle_sample(wl, order[a:a + rows], q, k, v))
    per = sum(times) / len(times)
    value = rows / per
    sample = sample_note(rows, wl) + " per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(wl, world),
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                         "cores": oracle.max_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--phase", choices=["all", "prefill", "decode", "dense", "varlen", "decode32"],
                    default="all",
                    help="run one phase only (for profiling); the headline line needs 'all'")
    ap.add_argument("--batches", type=lambda x: [int(b) for b in x.split(",")],
                    default=[1, 4, 8, 16, 64, 128],
                    help="batch sizes of the 32-layer decode phase (comma list)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        # CPU oracle only: no process group; under torchrun rank 0 alone works.
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = bench_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = bench_reference(args, world, rank)
        else:
            line = bench_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
