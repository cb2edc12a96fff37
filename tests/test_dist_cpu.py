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
