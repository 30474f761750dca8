"""Kv-head sharding on one GPU: each shard of the layer (its kv heads, their
query heads and their rolling caches) runs through the library on its own
tensors, in sequence, as the ranks of a multi-GPU job would; the reassembled
output heads must match the float64 oracle on the whole layer.  The shards
share nothing, so this is the whole multi-GPU data path apart from the final
output gather (covered on CPU with gloo ranks)."""
import math

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_chunk_b200 as swa
from sliding_window_gqa_chunk_b200 import sharding
from swa_workloads import random_case
from tests.gpu_helpers import assert_close, dev_i32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("Hq,Hkv,world", [(8, 4, 2), (12, 3, 2), (32, 8, 4)])
def test_kv_head_shards_reassemble_to_the_oracle(Hq, Hkv, world):
    B, L, W, chunk, d, steps = 2, 600, 256, 256, 64, 3
    q, k, v = random_case(900 + Hq + world, B, L + steps, Hq, Hkv, d)
    dims = swa.Dims(B, Hq, Hkv, d, W, 1.0 / math.sqrt(d), "f32")
    shards = sharding.kv_head_shards(dims, world)
    prefill_out, decode_out = [], [[] for _ in range(steps)]
    for s in shards:
        sd = s.dims
        kc, vc = swa.new_cache(sd, DEV)
        ws = swa.prefill_workspace(sd, chunk, DEV)
        qs = sharding.take_q_heads(q, s).to(DEV)
        ks = sharding.take_kv_heads(k, s).to(DEV)
        vs = sharding.take_kv_heads(v, s).to(DEV)
        out = torch.zeros((B, L, s.n_q_heads, d), dtype=torch.float32, device=DEV)
        for st in range(0, L, chunk):
            n = min(chunk, L - st)
            sp, nt = dev_i32([st] * B), dev_i32([n] * B)
            qc, kc_in, vc_in = (x[:, st:st + n].contiguous() for x in (qs, ks, vs))
            oc = torch.zeros((B, n, s.n_q_heads, d), dtype=torch.float32, device=DEV)
            swa.prefill_chunk(sd, oc, qc, kc_in, vc_in, kc, vc, sp, nt, workspace=ws)
            swa.cache_append(sd, kc, vc, kc_in, vc_in, sp, nt)
            out[:, st:st + n] = oc
        prefill_out.append(out.cpu())
        dws = swa.decode_workspace(sd, DEV)
        for i in range(steps):
            p = L + i
            o = torch.zeros((B, s.n_q_heads, d), dtype=torch.float32, device=DEV)
            swa.decode(sd, o, qs[:, p].contiguous(), ks[:, p].contiguous(), vs[:, p].contiguous(),
                       kc, vc, dev_i32([p] * B), dws)
            decode_out[i].append(o.cpu())
        swa.device_status()
    got = sharding.concat_heads(prefill_out).double().numpy()
    ref, cache = oracle.run_chunked_prefill(q[:, :L], k[:, :L], v[:, :L], W, chunk, dims.scale)
    assert_close(got, ref, f"{world} kv-head shards, prefill (Hq={Hq}, Hkv={Hkv})")
    for i in range(steps):
        p = L + i
        expect = oracle.decode(cache, q[:, p], k[:, p], v[:, p], [p] * B, dims.scale)
        got_d = sharding.concat_heads(decode_out[i]).double().numpy()
        assert_close(got_d, expect, f"{world} kv-head shards, decode step {i}")
