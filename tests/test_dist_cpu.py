"""Data-parallel max-logit exchange on CPU (gloo, world size 2).

Each rank computes the oracle max logit over its own batch item; after the
MAX all-reduce every rank holds the max over the whole batch, and the clip
decided from it equals the clip decided by one process that saw every item.
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import oracle
from gated_mla_qk_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from gated_mla_qk_b200.dist import allreduce_maxlogit
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    geom = synth.Geom(H=4, d_model=32, q_lora=16, kv_lora=16, d_c=8, d_s=4, d_v=8)
    inp = synth.attn_core(world, 24, geom, seed=5, hot_heads=2, hot_scale=3.0, dtype="f32")
    mine = {k: None if v is None else v[rank:rank + 1] for k, v in inp.items()}
    _, ml = oracle.attention(mine["Q"], mine["KC"], mine["kS"], mine["V"], mine["g"])
    t = torch.from_numpy(ml.astype(np.float32))
    allreduce_maxlogit(t)
    out[rank] = t.numpy().tolist()
    dist.destroy_process_group()


def test_maxlogit_allreduce_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    geom = synth.Geom(H=4, d_model=32, q_lora=16, kv_lora=16, d_c=8, d_s=4, d_v=8)
    inp = synth.attn_core(world, 24, geom, seed=5, hot_heads=2, hot_scale=3.0, dtype="f32")
    _, ml_all = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"])
    for r in range(world):
        np.testing.assert_array_equal(np.array(out[r], np.float32), ml_all.astype(np.float32))
    tau = float(np.median(ml_all))
    rng = np.random.default_rng(0)
    WQ = rng.standard_normal((geom.q_lora, geom.H * geom.d_qk)).astype(np.float32)
    WKV = rng.standard_normal((geom.kv_lora, geom.H * (geom.d_c + geom.d_v))).astype(np.float32)
    a = oracle.qkclip(WQ, WKV, np.array(out[0], np.float32), tau, geom, "f32")
    b = oracle.qkclip(WQ, WKV, ml_all.astype(np.float32), tau, geom, "f32")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_head_range_partitions_the_heads():
    from gated_mla_qk_b200.dist import head_range
    for H in (1, 4, 96, 97):
        for world in (1, 2, 3, 5, 8):
            ranges = [head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0                      # contiguous, no overlap
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1      # balanced


def test_head_sharded_clip_equals_full_clip_in_the_oracle():
    """The clip of head h reads only maxlogit_h and writes only head h's columns, so
    clipping each rank's contiguous column shard with its slice of the max-logit vector
    and concatenating gives the full clip, bit for bit (the basis of head sharding)."""
    from gated_mla_qk_b200.dist import head_range
    geom = synth.Geom(H=7, d_model=32, q_lora=16, kv_lora=12, d_c=8, d_s=4, d_v=8)
    rng = np.random.default_rng(3)
    WQ = rng.standard_normal((geom.q_lora, geom.H * geom.d_qk)).astype(np.float32)
    WKV = rng.standard_normal((geom.kv_lora, geom.H * (geom.d_c + geom.d_v))).astype(np.float32)
    ml = np.array([3.0, 12.0, 9.0, 10.0, 50.0, -1.0, 10.5], np.float32)
    full = oracle.qkclip(WQ, WKV, ml, 10.0, geom, "bf16")
    w = geom.d_c + geom.d_v
    for world in (2, 3, 7):
        parts = []
        for r in range(world):
            h0, h1 = head_range(geom.H, world, r)
            g = synth.Geom(H=h1 - h0, d_model=geom.d_model, q_lora=geom.q_lora, kv_lora=geom.kv_lora,
                           d_c=geom.d_c, d_s=geom.d_s, d_v=geom.d_v)
            parts.append(oracle.qkclip(WQ[:, h0 * geom.d_qk:h1 * geom.d_qk], WKV[:, h0 * w:h1 * w], ml[h0:h1], 10.0,
                                       g, "bf16"))
        for k, axis in ((0, 1), (1, 1), (2, 0), (3, 0)):
            np.testing.assert_array_equal(np.concatenate([p[k] for p in parts], axis=axis), full[k])
