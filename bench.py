#!/usr/bin/env python
"""Throughput of the gated MLA hot path on B200.

One step = one pass of the whole hot path on three synthetic workloads:
  * the QK-Clip chain at Kimi K3 size (x[4,4096,7168], bf16): up-projections,
    attention forward + per-head max logit, QK-Clip at tau = 100, and the
    recompute (up-projections + forward) with the clipped weights;
  * the causal gated attention forward with the fused max logit on the
    long-context workload (B=1, T=16384, H=96, d_qk=192, d_v=128, heads 0-7 x4);
  * the absorbed-latent decode of 64 sequences, context lengths U[1024, 8192].
``value`` is the long-context forward's TFLOP/s (causal half including the
diagonal: 2*B*H*T(T+1)/2*320 FLOP per call); every other part is reported
beside it with its own roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs its own independent problem instance
(weak scaling: the path partitions by independent problems); the per-head max
logits are MAX-all-reduced each step, the one exchange data parallelism adds.
``--impl reference`` times the CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal MLA fwd TFLOP/s (+maxlogit) at T=16k; absorbed decode HBM GB/s"
B_FWD, T_FWD = 1, 16384
FWD_FLOP = 2.0 * B_FWD * 96 * T_FWD * (T_FWD + 1) / 2 * (192 + 128)


T_TRAIN = 4096


def workload_config(T_run, decode_tokens, parallelism):
    """The `config` object of the JSON line; both arms print the same workload."""
    return {"workload": "gated MLA attention fwd + maxlogit, B=1 T=16384 H=96 d_qk=192 d_v=128 bf16 "
                        "(heads 0-7 x4); plus the K3 QK-Clip chain x[4,4096,7168] (up-proj, fwd, clip, "
                        "recompute) and absorbed decode 64 seqs L~U[1024,8192] H=96",
            "B": B_FWD, "T": T_run, "H": 96, "decode_tokens": decode_tokens,
            "l2": "inputs larger than L2 (fwd inputs 1.8 GB, decode cache %.0f MB); no flush"
                  % (decode_tokens * 576 * 2 / 1e6),
            "parallelism": parallelism}


def train_leg(args, gm, synth, geom, rank, st, dist):
    """mla_attn_fwd_train + mla_attn_bwd at B=1, T=4096, H=96 (gated, K3 heads)."""
    import torch
    tin = synth.attn_core(1, T_TRAIN, geom, seed=5 + 1000 * rank, hot_heads=8, hot_scale=4.0)
    td = {k: synth.to_torch(v, "bf16", "cuda") for k, v in tin.items()}
    del tin
    H, T = geom.H, T_TRAIN
    f32 = dict(dtype=torch.float32, device="cuda")
    O = torch.empty(1, T, H * 128, **f32)
    lse = torch.empty(1, T, H, **f32)
    ml = torch.empty(H, **f32)
    gen = torch.Generator(device="cuda").manual_seed(6 + rank)
    dO = torch.randn(1, T, H * 128, generator=gen, **f32)
    dQ = torch.empty(1, T, H, 192, **f32)
    dKC = torch.empty(1, T, H, 128, **f32)
    dkS = torch.empty(1, T, 64, **f32)
    dV = torch.empty(1, T, H, 128, **f32)
    dg = torch.empty(1, T, H * 128, **f32)
    ws = torch.empty(gm.mla_attn_bwd_workspace(geom, 1, T), dtype=torch.uint8, device="cuda")

    def run(ev):
        ev[0].record(st)
        gm.mla_attn_fwd_train(geom, td["Q"], td["KC"], td["kS"], td["V"], td["g"], O, ml, lse=lse)
        ev[1].record(st)
        gm.mla_attn_bwd(geom, td["Q"], td["KC"], td["kS"], td["V"], td["g"], O, lse, dO, dQ, dKC, dkS, dV, dg, ws)
        ev[2].record(st)

    warm = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(args.warmup):
        run(warm)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for k in range(args.steps):
        run(evs[k])
    torch.cuda.synchronize()
    t = torch.tensor([sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps,
                      sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps], dtype=torch.float64, device="cuda")
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    f_ms, b_ms = t.tolist()
    pairs = H * T * (T + 1) / 2
    pk_bf16 = peaks()["bf16"]
    f_flop = 2.0 * pairs * (192 + 128)
    b_flop = 2.0 * pairs * (2 * 128 + 2 * 192)          # dV, dA, dQ, dK products (recomputation not counted)
    return {
        "attn_fwd_train_B1_T4096": {"ms": f_ms, "value": f_flop / (f_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                                    "what": "mla_attn_fwd_train (fp32 o, lse)"},
        "attn_bwd_B1_T4096": {"ms": b_ms, "value": b_flop / (b_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                              "what": "mla_attn_bwd: tcgen05 dK/dV and dQ kernels (bf16 operands, fp32 TMEM accumulation)",
                              "roofline": {"bound": "tensor", "peak": pk_bf16, "unit": "TFLOP/s",
                                           "frac": b_flop / (b_ms / 1e3) / 1e12 / pk_bf16}},
    }


def absorbed_leg(args, gm, synth, geom, rank, st, dist):
    """mla_attn_fwd_absorbed (prefill on the latent cache) beside mla_attn_fwd at B=1, T=4096, H=96, gated."""
    import torch
    T, H = T_TRAIN, geom.H
    gen = torch.Generator(device="cuda").manual_seed(7 + rank)
    bf = torch.bfloat16
    rnd = lambda *shape, s=1.0: (torch.randn(*shape, generator=gen, device="cuda") * s).to(bf)
    Q, KC, kS, V = rnd(1, T, H, 192), rnd(1, T, H, 128), rnd(1, T, 64), rnd(1, T, H, 128)
    cache, W, g = rnd(1, T, 576), rnd(512, H * 256, s=512 ** -0.5), rnd(1, T, H * 128)
    O = torch.empty(1, T, H * 128, dtype=bf, device="cuda")
    ml = torch.empty(H, dtype=torch.float32, device="cuda")
    ws = torch.empty(gm.mla_attn_fwd_absorbed_workspace(geom, 1, T), dtype=torch.uint8, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(args.steps):
            fn()
        b.record(st)
        torch.cuda.synchronize()
        t = torch.tensor([a.elapsed_time(b) / args.steps], dtype=torch.float64, device="cuda")
        if dist is not None:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.item()

    ms_abs = timed(lambda: gm.mla_attn_fwd_absorbed(geom, Q, W, cache, g, O, ml, ws))
    ms_mat = timed(lambda: gm.mla_attn_fwd(geom, Q, KC, kS, V, g, O, ml))
    pairs = H * T * (T + 1) / 2
    return {"attn_fwd_absorbed_B1_T4096": {
        "ms": ms_abs, "value": 2.0 * pairs * 320 / (ms_abs / 1e3) / 1e12, "unit": "TFLOP/s",
        "own_work_tflops": 2.0 * pairs * (576 + 512) / (ms_abs / 1e3) / 1e12,
        "materialised_fwd_ms": ms_mat,
        "what": "mla_attn_fwd_absorbed: O and max logit from the latent cache (value counts the materialised "
                "form's 320 MAC per pair, own_work_tflops the absorbed form's 1088)"}}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--T", type=int, default=T_FWD, help="sequence length of the forward (profiling runs)")
    ap.add_argument("--skip-decode", action="store_true", help="time the forward alone (profiling runs)")
    ap.add_argument("--skip-fwd", action="store_true", help="time the decode alone (profiling runs)")
    ap.add_argument("--skip-clip", action="store_true", help="leave out the K3 QK-Clip chain (profiling runs)")
    ap.add_argument("--clip-T", type=int, default=4096, help="sequence length of the K3 QK-Clip chain (profiling runs)")
    ap.add_argument("--no-train", action="store_true", help="skip the training-form leg (fp32-output forward + backward)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


def host_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count()
    threads = n
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            threads = max(i.get("num_threads", n) for i in info)
    except Exception:
        pass
    return threads


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock and throttle-reason samples, kept only inside [t0, t1] (host time)."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.time() + 10.0          # nvidia-smi takes a while to print its first sample
            while not self.lines and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()
        time.sleep(0.06)                           # let the sample that covers the end arrive

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if self.t0 is not None and not (self.t0 <= ts <= self.t1 + 0.06):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(inp, rows_per_step=96):
    """Oracle attention for the heaviest query rows of head 0 (a bounded sample).

    Returns (seconds, flop) where flop counts the causal work of those rows."""
    import numpy as np
    import oracle
    T = inp["Q"].shape[1]
    rows = [(0, t, 0) for t in range(T - rows_per_step, T)]
    flop = sum(2.0 * (t + 1) * 320 for (_, t, _) in rows)
    t0 = time.perf_counter()
    oracle.attention_rows(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], rows)
    return time.perf_counter() - t0, flop


def cpu_baseline(inp, target_s=12.0):
    secs, flops = 0.0, 0.0
    n = 0
    while secs < target_s:
        s, f = oracle_sample(inp)
        secs += s
        flops += f
        n += 1
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"{n} x 96 causal rows (t = 16288..16383) of head 0 at B=1,T=16384, float64 numpy; "
                      f"{secs:.1f} s of CPU work"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from gated_mla_qk_b200 import synth
    inp = synth.attn_core(B_FWD, T_FWD, synth.K3, seed=2, hot_heads=8, hot_scale=4.0)
    decode_tokens = int(synth.decode_lengths(np.random.default_rng(4), 64, 1024, 8192).sum())
    for _ in range(args.warmup):
        oracle_sample(inp, rows_per_step=32)
    tot_s, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        s, f = oracle_sample(inp, rows_per_step=32)
        tot_s += s
        tot_f += f
    v = tot_f / tot_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(T_FWD, decode_tokens, "the oracle on rank 0's host cores"),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                             "sample": "per step: the forward's 32 heaviest causal rows (t=16352..16383) of head 0 "
                                       "at B=1, T=16384, float64 numpy; value = their causal FLOPs / time"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import numpy as np
    import torch
    import gated_mla_qk_b200 as gm
    from gated_mla_qk_b200 import synth
    from gated_mla_qk_b200.dist import allreduce_maxlogit

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    gm.load_library()

    # ---- inputs (seeded; each rank its own independent problem) ----
    geom = synth.K3
    T_run = args.T
    fwd_flop = 2.0 * B_FWD * geom.H * T_run * (T_run + 1) / 2 * (192 + 128)
    inp = synth.attn_core(B_FWD, T_run, geom, seed=2 + 1000 * rank, hot_heads=8, hot_scale=4.0)
    dq = {k: synth.to_torch(v, "bf16", "cuda") for k, v in inp.items()}
    O = torch.empty(B_FWD, T_run, geom.H * geom.d_v, dtype=torch.bfloat16, device="cuda")
    ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    dec = synth.decode_batch(seed=4 + 1000 * rank)
    dd = dict(q=synth.to_torch(dec["q"], "bf16", "cuda"), W_UKV=synth.to_torch(dec["W_UKV"], "bf16", "cuda"),
              cache=synth.to_torch(dec["cache"], "bf16", "cuda"), offs=torch.from_numpy(dec["seq_offsets"]).cuda())
    max_len = int(dec["lens"].max())
    Od = torch.empty(64, geom.H, geom.d_v, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(gm.mla_decode_workspace(geom, gm.GMLA_BF16, 64, max_len), dtype=torch.uint8, device="cuda")
    total_tokens = int(dec["seq_offsets"][-1])
    dec_bytes_cache = total_tokens * 576 * 2
    dec_bytes = dec_bytes_cache + 2 * 512 * 96 * 128 * 2 + 64 * 96 * (192 + 128) * 2
    st = torch.cuda.current_stream()

    # ---- QK-Clip chain at K3 size ----
    chain = None
    if not args.skip_clip:
        L = synth.k3_clip_layer(seed=3 + 1000 * rank, T=args.clip_T)
        Bc, Tc = L["x"].shape[:2]
        bf = torch.bfloat16
        chain = dict(
            x=synth.to_torch(L["x"], "bf16", "cuda"),
            W={k: synth.to_torch(L[k], "bf16", "cuda") for k in ("W_DQ", "w_q", "W_UQ", "W_DKV", "w_kv", "W_UKV")},
            Q=torch.empty(Bc, Tc, 96, 192, dtype=bf, device="cuda"), KC=torch.empty(Bc, Tc, 96, 128, dtype=bf, device="cuda"),
            kS=torch.empty(Bc, Tc, 64, dtype=bf, device="cuda"), V=torch.empty(Bc, Tc, 96, 128, dtype=bf, device="cuda"),
            O=torch.empty(Bc, Tc, 96 * 128, dtype=bf, device="cuda"), ml=torch.empty(96, dtype=torch.float32, device="cuda"),
            clipped=torch.empty(96, dtype=torch.uint8, device="cuda"), tau=L["tau"], B=Bc, T=Tc)
        chain["WQ"] = chain["W"]["W_UQ"].clone()
        chain["WKV"] = chain["W"]["W_UKV"].clone()
        chain["ws"] = torch.empty(gm.mla_up_proj_workspace(geom, gm.GMLA_BF16, Bc, Tc), dtype=torch.uint8, device="cuda")
        del L
    Mc = 4 * args.clip_T
    UP_FLOP = 2.0 * Mc * (7168 * 1536 + 1536 * 18432 + 7168 * 576 + 512 * 24576)
    C3_FLOP = 2.0 * 4 * 96 * args.clip_T * (args.clip_T + 1) / 2 * 320

    def clip_chain(ev):
        c = chain
        c["WQ"].copy_(c["W"]["W_UQ"]); c["WKV"].copy_(c["W"]["W_UKV"])     # pristine weights each step
        W = c["W"]

        def up():
            gm.mla_up_proj(geom, c["x"], W["W_DQ"], W["w_q"], c["WQ"], W["W_DKV"], W["w_kv"], c["WKV"], c["Q"], c["KC"],
                           c["kS"], c["V"], None, c["ws"])

        def att():
            gm.mla_attn_fwd(geom, c["Q"], c["KC"], c["kS"], c["V"], None, c["O"], c["ml"])

        ev[0].record(st); up(); ev[1].record(st); att()
        allreduce_maxlogit(c["ml"])
        ev[2].record(st)
        gm.qkclip_rescale(geom, c["WQ"], c["WKV"], c["ml"], c["tau"], c["clipped"], None)
        ev[3].record(st); up(); ev[4].record(st); att(); ev[5].record(st)

    def fwd():
        if not args.skip_fwd:
            gm.mla_attn_fwd(geom, dq["Q"], dq["KC"], dq["kS"], dq["V"], dq["g"], O, ml)

    def decode():
        if not args.skip_decode:
            gm.mla_decode_absorbed(geom, dd["q"], dd["W_UKV"], dd["cache"], dd["offs"], max_len, None, Od, ws)

    def step(ev):
        if chain is not None:
            clip_chain(ev[4:])
        ev[0].record(st)
        fwd()
        ev[1].record(st)
        allreduce_maxlogit(ml)
        ev[2].record(st)
        decode()
        ev[3].record(st)

    warm_ev = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    for _ in range(args.warmup):
        step(warm_ev)
    torch.cuda.synchronize()
    assert gm.device_status() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = gm.launch_count()
    with ClockSampler(local) as clk:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        start.record(st)
        for k in range(args.steps):
            step(evs[k])
        end.record(st)
        torch.cuda.synchronize()
        clk.mark_end()
    launches = gm.launch_count() - n0
    if dist is not None:
        dist.barrier()
    status = gm.device_status()
    total_ms = start.elapsed_time(end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[2].elapsed_time(e[3]) for e in evs]
    parts = [sum(fwd_ms), sum(dec_ms)]
    if chain is not None:
        parts += [sum(e[4].elapsed_time(e[5]) + e[7].elapsed_time(e[8]) for e in evs),      # up-projections (x2)
                  sum(e[5].elapsed_time(e[6]) + e[8].elapsed_time(e[9]) for e in evs),      # K3 forwards (x2)
                  sum(e[6].elapsed_time(e[7]) for e in evs)]                                 # QK-Clip
    t = torch.tensor([total_ms] + parts, dtype=torch.float64, device="cuda")
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, fwd_sum, dec_sum, *chain_sums = t.tolist()
    n_clipped = int(chain["clipped"].sum().item()) if chain is not None else 0

    # ---- the decode alone: back-to-back calls, not right behind the forward ----
    # In the step the decode follows the forward and shares its power state;
    # this reports it again timed on its own (median of 20 calls; the 375 MB
    # cache is larger than L2).
    dec_alone_ms = None
    if not args.skip_decode:
        for _ in range(3):
            decode()
        torch.cuda.synchronize()
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
        for a, b in ev2:
            a.record(st)
            decode()
            b.record(st)
        torch.cuda.synchronize()
        tt = torch.tensor([sorted(a.elapsed_time(b) for a, b in ev2)[10]], dtype=torch.float64, device="cuda")
        if dist is not None:
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        dec_alone_ms = tt.item()

    # ---- end to end through the public API with host buffers ----
    # Every step uploads its inputs from pinned host memory and reads O and the
    # max logits back.  The uploads run on a stream of their own into one of
    # two device input sets and the downloads on another, from one of two
    # output sets, so step k+1's upload overlaps step k's forward and download
    # (as a serving loop would).
    e2e = None
    if not args.no_e2e:
        pin = {k: dq[k].cpu().pin_memory() for k in ("Q", "KC", "kS", "V", "g")}
        O_h = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        ml_h = torch.empty(ml.shape, dtype=ml.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = O_h.numel() * O_h.element_size() + ml_h.numel() * 4
        del dq
        dev_in = [{k: torch.empty(pin[k].shape, dtype=pin[k].dtype, device="cuda") for k in pin} for _ in range(2)]
        outs = [(O, ml), (torch.empty_like(O), torch.empty_like(ml))]
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        e_steps = max(2, min(args.steps, 5))

        def ev():
            return torch.cuda.Event()

        def run_e2e(n):
            ready = [ev(), ev()]                    # inputs of set i uploaded
            free_in = [None, None]                  # forward done with input set i
            out_done = [None, None]                 # download of output set i finished
            with torch.cuda.stream(s_up):
                for k in pin:
                    dev_in[0][k].copy_(pin[k], non_blocking=True)
                ready[0].record(s_up)
            for step in range(n):
                i = step & 1
                if step + 1 < n:                    # upload the next step's inputs meanwhile
                    j = i ^ 1
                    with torch.cuda.stream(s_up):
                        if free_in[j] is not None:
                            s_up.wait_event(free_in[j])
                        for k in pin:
                            dev_in[j][k].copy_(pin[k], non_blocking=True)
                        ready[j] = ev()
                        ready[j].record(s_up)
                st.wait_event(ready[i])
                if out_done[i] is not None:
                    st.wait_event(out_done[i])      # output set i was read back two steps ago
                d = dev_in[i]
                Oi, mli = outs[i]
                gm.mla_attn_fwd(geom, d["Q"], d["KC"], d["kS"], d["V"], d["g"], Oi, mli)
                done = ev()
                done.record(st)
                free_in[i] = done
                with torch.cuda.stream(s_down):
                    s_down.wait_event(done)
                    O_h.copy_(Oi, non_blocking=True)
                    ml_h.copy_(mli, non_blocking=True)
                    out_done[i] = ev()
                    out_done[i].record(s_down)
            for e in out_done:
                if e is not None:
                    st.wait_event(e)

        run_e2e(2)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        s_up.wait_event(a)
        run_e2e(e_steps)
        b.record(st)
        torch.cuda.synchronize()
        e_ms = torch.tensor([a.elapsed_time(b) / e_steps], dtype=torch.float64, device="cuda")
        if dist is not None:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": world * fwd_flop / (e_ms.item() / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms.item(),
               "what": "mla_attn_fwd with every step's inputs copied from pinned host memory and O + maxlogit "
                       "copied back; uploads and downloads on their own streams, overlapping the neighbouring "
                       "steps' forwards"}
        del dev_in, outs

    # ---- training form, timed on its own after the step: fp32-output forward + backward ----
    train = None
    if not args.no_train:
        train = train_leg(args, gm, synth, geom, rank, st, dist)
        train.update(absorbed_leg(args, gm, synth, geom, rank, st, dist))

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    pk = peaks()
    fwd_avg_ms = fwd_sum / args.steps
    dec_avg_ms = dec_sum / args.steps
    fwd_tflops = fwd_flop / (fwd_avg_ms / 1e3) / 1e12
    dec_gbs = dec_bytes / (dec_avg_ms / 1e3) / 1e9
    prof_traffic = None
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tp):
        prof_traffic = json.load(open(tp)).get("attn_fwd_T16384")
    line = {
        "metric": METRIC,
        "value": world * fwd_tflops,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(T_run, total_tokens,
                                  f"replicas x{world} (independent problems), maxlogit MAX all-reduce"),
        "roofline": {"bound": "tensor", "achieved": fwd_tflops, "peak": pk["bf16"], "unit": "TFLOP/s",
                     "frac": fwd_tflops / pk["bf16"], "traffic": prof_traffic,
                     "kernel": "tc_attn::attn_fwd_kernel", "peak_source": f"{pk['src']} bf16 burst",
                     "frac_of_sustained": fwd_tflops / pk["bf16_sust"] if pk["bf16_sust"] else None},
        "decode": {"value": world * dec_gbs, "unit": "GB/s", "ms": dec_avg_ms,
                   "bytes_per_call": dec_bytes, "cache_only_gbs": dec_bytes_cache / (dec_avg_ms / 1e3) / 1e9,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": pk["hbm"], "unit": "GB/s",
                                "frac": dec_gbs / pk["hbm"]}},
        "fwd_ms": fwd_avg_ms,
        "parts": {},
        "gpu_launches": launches,
        "device_status": status,
        "clocks": clk.summary(),
    }
    if chain is not None:
        up_ms = chain_sums[0] / (2 * args.steps)
        c3_ms = chain_sums[1] / (2 * args.steps)
        clip_ms = chain_sums[2] / args.steps
        clip_bytes = 2 * n_clipped * (1536 * 128 + 1536 * 64 + 512 * 128) * 2
        line["parts"] = {
            "up_proj_B4_T%d" % args.clip_T: {"ms": up_ms, "value": UP_FLOP / (up_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                                 "roofline": {"bound": "tensor", "peak": pk["bf16"],
                                              "frac": UP_FLOP / (up_ms / 1e3) / 1e12 / pk["bf16"]}},
            "attn_fwd_B4_T%d_nogate" % args.clip_T: {"ms": c3_ms, "value": C3_FLOP / (c3_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                                         "roofline": {"bound": "tensor", "peak": pk["bf16"],
                                                      "frac": C3_FLOP / (c3_ms / 1e3) / 1e12 / pk["bf16"]}},
            "qkclip": {"ms": clip_ms, "clipped_heads": n_clipped, "bytes": clip_bytes,
                       "value": clip_bytes / (clip_ms / 1e3) / 1e9, "unit": "GB/s",
                       "roofline": {"bound": "hbm", "peak": pk["hbm"], "frac": clip_bytes / (clip_ms / 1e3) / 1e9 / pk["hbm"]}},
        }
    line["parts"]["attn_fwd_B1_T16384"] = {"ms": fwd_avg_ms, "value": fwd_tflops, "unit": "TFLOP/s"}
    line["parts"]["decode_64seq"] = {"ms": dec_avg_ms, "value": dec_gbs, "unit": "GB/s"}
    if dec_alone_ms is not None:
        alone_gbs = dec_bytes / (dec_alone_ms / 1e3) / 1e9
        line["parts"]["decode_64seq_alone"] = {
            "ms": dec_alone_ms, "value": alone_gbs, "unit": "GB/s",
            "roofline": {"bound": "hbm", "peak": pk["hbm"], "frac": alone_gbs / pk["hbm"]},
            "what": "mla_decode_absorbed timed in back-to-back calls (median of 20), not right behind the forward"}
    if train:
        line["parts"].update(train)
    if e2e:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and T_run == T_FWD:
        line["cpu_baseline"] = cpu_baseline(inp)
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
