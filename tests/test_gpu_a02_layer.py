"""Whole-layer parity: the tiny fp32 layer end to end (forward, max logit,
QK-Clip, re-check), bf16 up-projections, and the bf16 clip on K3-sized weights."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_F32, check_status, dev, host, max_rel, rel_l2

pytestmark = pytest.mark.gpu


def _up_proj_gpu(geom, dtype, x, W):
    import torch
    import gated_mla_qk_b200 as gm
    B, T = x.shape[:2]
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {k: dev(W[k], dtype) for k in ("W_DQ", "w_q", "W_UQ", "W_DKV", "w_kv", "W_UKV")}
    xd = dev(x, dtype) if not hasattr(x, "is_cuda") else x
    out = dict(
        Q=torch.empty(B, T, geom.H, geom.d_qk, dtype=td, device="cuda"),
        KC=torch.empty(B, T, geom.H, geom.d_c, dtype=td, device="cuda"),
        kS=torch.empty(B, T, geom.d_s, dtype=td, device="cuda"),
        V=torch.empty(B, T, geom.H, geom.d_v, dtype=td, device="cuda"),
        cache=torch.empty(B, T, geom.kv_lora + geom.d_s, dtype=td, device="cuda"),
    )
    gm.mla_up_proj(geom, xd, d["W_DQ"], d["w_q"], d["W_UQ"], d["W_DKV"], d["w_kv"], d["W_UKV"],
                   out["Q"], out["KC"], out["kS"], out["V"], out["cache"])
    return out


def _layer_gpu(L, W_UQ, W_UKV):
    """Tiny fp32 layer on the GPU: up-proj, gate GEMM, attention, output GEMM."""
    import torch
    import gated_mla_qk_b200 as gm
    geom = L["geom"]
    W = dict(L, W_UQ=W_UQ, W_UKV=W_UKV)
    up = _up_proj_gpu(geom, "f32", L["x"], W)
    x = dev(L["x"], "f32")
    B, T = x.shape[:2]
    g = torch.empty(B, T, geom.H * geom.d_v, device="cuda")
    gm.mla_gemm(x.view(B * T, -1), dev(L["W_g"], "f32"), g.view(B * T, -1))
    o = torch.empty_like(g)
    ml = torch.empty(geom.H, device="cuda")
    gm.mla_attn_fwd(geom, up["Q"], up["KC"], up["kS"], up["V"], g, o, ml)
    delta = torch.empty(B, T, geom.d_model, device="cuda")
    gm.mla_gemm(o.view(B * T, -1), dev(L["W_O"], "f32"), delta.view(B * T, -1))
    check_status()
    return dict(up, g=g, o=o, maxlogit=ml, delta=delta)


def test_tiny_fp32_layer_clip_and_recheck():
    import torch
    import gated_mla_qk_b200 as gm
    L = synth.tiny_layer(0)
    geom, tau = L["geom"], L["tau"]
    ref = oracle.layer_forward(L["x"], L, geom, "f32")
    got = _layer_gpu(L, L["W_UQ"], L["W_UKV"])
    for k in ("Q", "KC", "kS", "V", "cache", "g", "o", "delta"):
        want = ref[k].reshape(host(got[k]).shape)
        assert rel_l2(host(got[k]), want) <= TOL_F32, k
    ml_gpu = host(got["maxlogit"])
    assert max_rel(ml_gpu, ref["maxlogit"]) <= 1e-5

    # (1) Same maxlogit vector on both sides -> bit-identical rescaled weights.
    ml32 = ref["maxlogit"].astype(np.float32)
    WQ_ref, WKV_ref, clip_ref, gam_ref = oracle.qkclip(L["W_UQ"], L["W_UKV"], ml32, tau, geom, "f32")
    WQ, WKV = dev(L["W_UQ"], "f32"), dev(L["W_UKV"], "f32")
    clipped = torch.empty(geom.H, dtype=torch.uint8, device="cuda")
    gamma = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.qkclip_rescale(geom, WQ, WKV, torch.from_numpy(ml32).cuda(), tau, clipped, gamma)
    check_status()
    np.testing.assert_array_equal(host(WQ).view(np.uint32), WQ_ref.view(np.uint32))
    np.testing.assert_array_equal(host(WKV).view(np.uint32), WKV_ref.view(np.uint32))
    np.testing.assert_array_equal(host(clipped), clip_ref)
    np.testing.assert_array_equal(host(gamma).view(np.uint32), gam_ref.view(np.uint32))

    # (2) GPU chain: its own max logit decides the clip; the clipped set must equal the oracle's.
    WQ2, WKV2 = dev(L["W_UQ"], "f32"), dev(L["W_UKV"], "f32")
    gm.qkclip_rescale(geom, WQ2, WKV2, got["maxlogit"], tau, clipped, gamma)
    check_status()
    np.testing.assert_array_equal(host(clipped), clip_ref)
    after = _layer_gpu(L, host(WQ2), host(WKV2))
    ml_after = host(after["maxlogit"])
    for h in range(geom.H):
        if clip_ref[h]:
            assert abs(ml_after[h] - tau) / tau <= TOL_F32
        else:
            assert ml_after[h] == ml_gpu[h]


@pytest.mark.parametrize("T", [100, 150])   # M = 200: two one-CTA launches for x's products; M = 300: one pair launch, ragged rows
def test_up_proj_bf16_k3_geometry(T):
    geom = synth.K3
    rng = np.random.default_rng(21)
    W = {k: synth.round_storage(v, "bf16") for k, v in synth.layer_weights(geom, rng, with_gate_out=False).items()}
    x = synth.round_storage(rng.standard_normal((2, T, geom.d_model)).astype(np.float32), "bf16")
    got = _up_proj_gpu(geom, "bf16", x, W)
    check_status()
    ref = oracle.up_proj(x, W["W_DQ"], W["w_q"], W["W_UQ"], W["W_DKV"], W["w_kv"], W["W_UKV"], geom, "bf16")
    for k in ("Q", "KC", "kS", "V", "cache"):
        assert rel_l2(host(got[k]), ref[k]) <= TOL_BF16, k


def test_clip_bf16_k3_weights_bit_exact():
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.K3
    rng = np.random.default_rng(22)
    W = synth.layer_weights(geom, rng, with_gate_out=False)
    WQ0 = synth.round_storage(W["W_UQ"], "bf16")
    WKV0 = synth.round_storage(W["W_UKV"], "bf16")
    ml = rng.uniform(20, 180, geom.H).astype(np.float32)
    ml[5] = np.float32(100.0)        # equal to tau: not clipped
    ml[6] = -3.0
    tau = 100.0
    WQ_ref, WKV_ref, clip_ref, gam_ref = oracle.qkclip(WQ0, WKV0, ml, tau, geom, "bf16")
    WQ, WKV = dev(WQ0, "bf16"), dev(WKV0, "bf16")
    clipped = torch.empty(geom.H, dtype=torch.uint8, device="cuda")
    gamma = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.qkclip_rescale(geom, WQ, WKV, torch.from_numpy(ml).cuda(), tau, clipped, gamma)
    check_status()
    np.testing.assert_array_equal(host(clipped), clip_ref)
    assert clip_ref[5] == 0 and clip_ref[6] == 0 and clip_ref.sum() > 30
    np.testing.assert_array_equal(host(gamma).view(np.uint32), gam_ref.view(np.uint32))
    np.testing.assert_array_equal(host(WQ).view(np.uint32), WQ_ref.view(np.uint32))
    np.testing.assert_array_equal(host(WKV).view(np.uint32), WKV_ref.view(np.uint32))
