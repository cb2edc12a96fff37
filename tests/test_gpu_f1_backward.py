"""Parity of the training forward's log-sum-exp and of mla_attn_bwd with the
oracle (whose backward is pinned by finite differences and torch autograd)."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_F32, Guarded, check_status, dev, guarded_bytes, host, rel_l2

pytestmark = pytest.mark.gpu


def _train_and_backward(inp, geom, dO, gate):
    import torch
    import gated_mla_qk_b200 as gm
    B, T = inp["Q"].shape[:2]
    H = geom.H
    Q, KC, kS, V = (dev(inp[k], "bf16") for k in ("Q", "KC", "kS", "V"))
    g = dev(inp["g"], "bf16") if gate else None
    f32 = dict(dtype=torch.float32, device="cuda")
    O = torch.empty(B, T, H * geom.d_v, **f32)
    lse = torch.empty(B, T, H, **f32)
    ml = torch.empty(H, **f32)
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O, ml, lse=lse)
    dQ = torch.empty(B, T, H, geom.d_qk, **f32)
    dKC = torch.empty(B, T, H, geom.d_c, **f32)
    dkS = torch.empty(B, T, geom.d_s, **f32)
    dV = torch.empty(B, T, H, geom.d_v, **f32)
    dg = torch.empty(B, T, H * geom.d_v, **f32) if gate else None
    gm.mla_attn_bwd(geom, Q, KC, kS, V, g, O, lse, torch.from_numpy(dO).cuda(), dQ, dKC, dkS, dV, dg)
    check_status()
    return host(lse), [host(x) if x is not None else None for x in (dQ, dKC, dkS, dV, dg)]


@pytest.mark.parametrize("B,T,H,gate", [(1, 1, 2, True), (1, 70, 2, True), (2, 129, 3, False), (1, 300, 2, True), (2, 520, 2, True),
                                         (1, 1000, 2, True),
                                         (1, 256, 96, True)])     # every K3 head: k^S's gradient summed over 96 heads
def test_backward_k3_heads(B, T, H, gate):
    """K3 head widths (the tcgen05 training forward feeds o and lse)."""
    geom = synth.Geom(H=H)
    inp = synth.attn_core(B, T, geom, seed=300 + T, hot_heads=1, hot_scale=3.0, gate=gate)
    dO = np.random.default_rng(301 + T).standard_normal((B, T, H * geom.d_v)).astype(np.float32)
    lse, got = _train_and_backward(inp, geom, dO, gate)
    assert np.allclose(lse, oracle.attention_lse(inp["Q"], inp["KC"], inp["kS"]), rtol=1e-5, atol=1e-5)
    want = oracle.attention_backward(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"] if gate else None, dO)
    scale = np.linalg.norm(want[3])                  # dV: never zero
    for name, a, b in zip(("dQ", "dKC", "dkS", "dV", "dg"), got, want):
        if b is None:
            assert a is None
            continue
        a = a.reshape(b.shape)
        if np.linalg.norm(b) == 0:                    # T = 1: one key, so dS = 0 exactly
            # (the tensor-core passes take dO~ in bf16 for dA, D in fp32: bf16-level residue)
            assert np.linalg.norm(a) <= TOL_BF16 * scale, name
            continue
        # o comes from the bf16 tensor-core forward (P rounded to bf16), which D = sum dO * o inherits
        assert rel_l2(a, b) <= TOL_BF16, name


def test_backward_repeated_runs_on_nan_filled_outputs():
    """The tile kernels' hand-offs between the MMA issuer and the four compute
    warps must not depend on timing: with every output and the workspace
    filled with NaN before each call, twenty calls in a row give the same,
    fully written gradients (T = 1000: a partial last key tile and a last
    query tile with 104 valid rows)."""
    import torch
    import gated_mla_qk_b200 as gm
    B, T, H = 1, 1000, 2
    geom = synth.Geom(H=H)
    inp = synth.attn_core(B, T, geom, seed=300 + T, hot_heads=1, hot_scale=3.0, gate=True)
    dO = np.random.default_rng(301 + T).standard_normal((B, T, H * geom.d_v)).astype(np.float32)
    Q, KC, kS, V, g = (dev(inp[k], "bf16") for k in ("Q", "KC", "kS", "V", "g"))
    f32 = dict(dtype=torch.float32, device="cuda")
    O = torch.empty(B, T, H * geom.d_v, **f32)
    lse = torch.empty(B, T, H, **f32)
    ml = torch.empty(H, **f32)
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O, ml, lse=lse)
    dOd = torch.from_numpy(dO).cuda()
    shapes = dict(dQ=(B, T, H, geom.d_qk), dKC=(B, T, H, geom.d_c), dkS=(B, T, geom.d_s), dV=(B, T, H, geom.d_v),
                  dg=(B, T, H * geom.d_v))
    nan = float("nan")
    first = None
    for _ in range(20):
        out = {k: torch.full(s, nan, **f32) for k, s in shapes.items()}
        ws = torch.full((gm.mla_attn_bwd_workspace(geom, B, T),), 0xFF, dtype=torch.uint8, device="cuda")
        gm.mla_attn_bwd(geom, Q, KC, kS, V, g, O, lse, dOd, out["dQ"], out["dKC"], out["dkS"], out["dV"], out["dg"],
                        workspace=ws)
        check_status()
        got = {k: host(v) for k, v in out.items()}
        for k, v in got.items():
            assert np.isfinite(v).all(), k
        if first is None:
            first = got
            want = oracle.attention_backward(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], dO)
            for k, w in zip(("dQ", "dKC", "dkS", "dV", "dg"), want):
                assert rel_l2(got[k].reshape(w.shape), w) <= TOL_BF16, k
        else:
            for k in ("dQ", "dKC", "dV", "dg"):           # no atomics: the same bits every call
                assert np.array_equal(got[k], first[k]), k
            assert rel_l2(got["dkS"], first["dkS"]) <= 1e-6  # cross-head atomic sum: order may vary


def test_backward_other_head_widths_fp32_path():
    """Other head widths: CUDA-core forward and backward, all fp32 arithmetic."""
    geom = synth.TINY
    inp = synth.attn_core(1, 45, geom, seed=311, hot_heads=1, hot_scale=2.0, gate=True)
    dO = np.random.default_rng(312).standard_normal((1, 45, geom.H * geom.d_v)).astype(np.float32)
    lse, got = _train_and_backward(inp, geom, dO, True)
    assert np.allclose(lse, oracle.attention_lse(inp["Q"], inp["KC"], inp["kS"]), rtol=1e-5, atol=1e-5)
    want = oracle.attention_backward(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], dO)
    for name, a, b in zip(("dQ", "dKC", "dkS", "dV", "dg"), got, want):
        assert rel_l2(a.reshape(b.shape), b) <= TOL_F32, name


@pytest.mark.parametrize("geom,B,T,gate", [(synth.Geom(H=96), 1, 129, True), (synth.Geom(H=2), 2, 300, False),
                                           (synth.TINY, 1, 45, True)])
def test_attention_backward_guards(geom, B, T, gate):
    import torch
    import gated_mla_qk_b200 as gm
    dtype = "f32" if geom.d_c != 128 else "bf16"
    inp = synth.attn_core(B, T, geom, seed=600 + T, hot_heads=1, gate=gate, dtype=dtype)
    Q, KC, kS, V = (dev(inp[k], dtype) for k in ("Q", "KC", "kS", "V"))
    g = dev(inp["g"], dtype) if gate else None
    f32 = dict(dtype=torch.float32, device="cuda")
    O = torch.empty(B, T, geom.H * geom.d_v, **f32)
    lse = torch.empty(B, T, geom.H, **f32)
    ml = torch.empty(geom.H, **f32)
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O, ml, lse=lse)
    dO = torch.randn(B, T, geom.H * geom.d_v, generator=torch.Generator().manual_seed(7)).cuda()
    grads = dict(dQ=Guarded((B, T, geom.H, geom.d_qk), torch.float32),
                 dKC=Guarded((B, T, geom.H, geom.d_c), torch.float32),
                 dkS=Guarded((B, T, geom.d_s), torch.float32),
                 dV=Guarded((B, T, geom.H, geom.d_v), torch.float32))
    if gate:
        grads["dg"] = Guarded((B, T, geom.H * geom.d_v), torch.float32)
    ws = guarded_bytes(gm.mla_attn_bwd_workspace(geom, B, T))
    gm.mla_attn_bwd(geom, Q, KC, kS, V, g, O, lse, dO, grads["dQ"].t, grads["dKC"].t, grads["dkS"].t,
                    grads["dV"].t, grads["dg"].t if gate else None, workspace=ws.t)
    check_status()
    for k, v in grads.items():
        v.check(k)
    ws.check("workspace", written=False)
