"""Host-side logic of bench.py that needs no GPU: the algorithmic work counts,
the max-over-ranks reduction (2 gloo ranks on CPU), the rank-0-only reference
arm and the clock-sample parsing."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_pair_counts_match_the_closed_forms():
    # SWA over 16384 tokens with W = 4096: W(W+1)/2 + (L - W) W pairs per head
    assert bench.prefill_pairs_per_head(16384, 4096, 4096) == 4096 * 4097 // 2 + 12288 * 4096
    assert bench.prefill_pairs_per_head(16384, 4096, 4096) == 58_722_304
    # dense causal: L(L+1)/2
    assert bench.prefill_pairs_per_head(16384, 16384, 16384) == 134_225_920
    # per-chunk counts add up to the whole prompt
    total = sum(bench.chunk_pairs_per_head(c * 4096, 4096, 4096) for c in range(4))
    assert total == 58_722_304
    flops = 4 * 128 * 32 * 58_722_304
    assert abs(flops / 1e12 - 0.962) < 1e-3


def test_decode_bytes_per_step():
    from swa_workloads import DECODE_B64
    B, W, Hkv, d, Hq = 64, 4096, 8, 128, 32
    expect = B * (2 * W * Hkv * d * 2 + Hq * d * 2 + 2 * Hkv * d * 2 * 2 + Hq * d * 2)
    assert expect == 1_075_314_688
    assert DECODE_B64.batch == B and DECODE_B64.shape.window == W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        got = bench.reduce_max(1.5 + rank * 2.25, world)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": got}, f)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        with open(tmp_path / f"r{r}.json") as f:
            assert json.load(f)["max"] == 3.75


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup, ref_rows = 1, 0, 4
    assert bench.bench_reference(A, world=2, rank=1) is None
    line = bench.bench_reference(A, world=1, rank=0)
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"] == bench.headline_config(bench.PREFILL_16K, 1)


def test_clock_summary_reports_median_and_reasons():
    cs = bench.ClockSampler(0)
    cs.sm_max = 1965.0
    cs.samples = [(1965.0, 0x0), (1800.0, 0x4), (1700.0, 0x4)]
    s = cs.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    cs.samples.append((1500.0, 0x40))
    assert "hw_thermal_slowdown" in cs.summary()["reasons"]


def test_profiled_traffic_is_dropped_when_the_kernel_changes(monkeypatch):
    rec = dict(bench.PROFILED_TRAFFIC["swa_decode_kernel"])
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "swa_decode_kernel", dict(rec, sha="0" * 16))
    assert bench.profiled_traffic("swa_decode_kernel") == (None, None)


def test_profiled_traffic_matches_the_current_sources():
    for kernel in ("swa_prefill_kernel", "swa_decode_kernel"):
        assert bench.profiled_traffic(kernel)[0] is not None, f"{kernel}: profile record is stale"


def test_source_key_ignores_comments_but_not_code(tmp_path):
    base = "__global__ void k(int* p) {\n  p[0] = 1;  // one\n}\n"
    f = tmp_path / "a.cu"
    f.write_text(base)
    key = bench.source_key(str(f))
    f.write_text("/* header */\n" + base.replace("// one", "// the first element"))
    assert bench.source_key(str(f)) == key
    f.write_text(base.replace("p[0] = 1", "p[0] = 2"))
    assert bench.source_key(str(f)) != key


def test_decode_launch_count_follows_the_split_rule():
    import sliding_window_gqa_chunk_b200 as swa
    mk = lambda B: swa.Dims(B, 32, 8, 128, 4096, 1.0 / 128 ** 0.5, "bf16")
    # batch 1 and 4: one launch (clustered splits); 16: one streaming CTA per
    # (sequence, kv head); 24: 3 splits + combine; 64 and 128: one split per
    # (sequence, kv head), no combine
    assert bench.decode_launches_per_call(mk(1), swa) == 1
    assert bench.decode_launches_per_call(mk(4), swa) == 1
    assert bench.decode_launches_per_call(mk(16), swa) == 1
    assert bench.decode_launches_per_call(mk(24), swa) == 2
    assert bench.decode_launches_per_call(mk(64), swa) == 1
    assert bench.decode_launches_per_call(mk(128), swa) == 1
