"""The QK-Clip chain at Kimi K3 size (bf16): x[4,4096,7168] -> up-projections
-> attention max logit over the batch -> clip at tau = 100 -> recompute.

Checked against the oracle on sampled tokens (up-projections), on 16 sampled
heads (the 12 scaled heads and 4 others: max logit over all 16,384 query
positions, clipped set), and through the clip's own invariants after the
recompute: clipped heads land on tau within the bf16 bound, unclipped heads'
max logits are bit-identical to the first pass."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_MAXLOGIT, check_status, dev, host, max_rel, rel_l2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sub_geom(geom, H):
    return synth.Geom(H=H, d_model=geom.d_model, q_lora=geom.q_lora, kv_lora=geom.kv_lora, d_c=geom.d_c,
                      d_s=geom.d_s, d_v=geom.d_v, rms_eps=geom.rms_eps)


def _head_cols(W_UQ, W_UKV, geom, heads):
    q = np.concatenate([W_UQ[:, h * geom.d_qk:(h + 1) * geom.d_qk] for h in heads], axis=1)
    w = geom.d_c + geom.d_v
    kv = np.concatenate([W_UKV[:, h * w:(h + 1) * w] for h in heads], axis=1)
    return q, kv


def test_k3_clip_chain():
    import torch
    import gated_mla_qk_b200 as gm
    L = synth.k3_clip_layer()
    geom, tau = L["geom"], L["tau"]
    B, T = L["x"].shape[:2]
    x = dev(L["x"], "bf16")
    Wd = {k: dev(L[k], "bf16") for k in ("W_DQ", "w_q", "W_UQ", "W_DKV", "w_kv", "W_UKV")}
    bf = torch.bfloat16

    def run(W_UQ, W_UKV):
        Q = torch.empty(B, T, geom.H, geom.d_qk, dtype=bf, device="cuda")
        KC = torch.empty(B, T, geom.H, geom.d_c, dtype=bf, device="cuda")
        kS = torch.empty(B, T, geom.d_s, dtype=bf, device="cuda")
        V = torch.empty(B, T, geom.H, geom.d_v, dtype=bf, device="cuda")
        gm.mla_up_proj(geom, x, Wd["W_DQ"], Wd["w_q"], W_UQ, Wd["W_DKV"], Wd["w_kv"], W_UKV, Q, KC, kS, V)
        O = torch.empty(B, T, geom.H * geom.d_v, dtype=bf, device="cuda")
        ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
        gm.mla_attn_fwd(geom, Q, KC, kS, V, None, O, ml)
        check_status()
        return Q, KC, kS, V, ml

    Q, KC, kS, V, ml = run(Wd["W_UQ"], Wd["W_UKV"])
    ml1 = host(ml)

    # (1) up-projections on 48 sampled tokens, against the oracle on those rows
    rng = np.random.default_rng(0)
    toks = [(int(b), int(t)) for b, t in zip(rng.integers(0, B, 48), rng.integers(0, T, 48))]
    xs = np.stack([L["x"][b, t] for b, t in toks])[None]
    ref = oracle.up_proj(xs, L["W_DQ"], L["w_q"], L["W_UQ"], L["W_DKV"], L["w_kv"], L["W_UKV"], geom, "bf16")
    for name, t_ in (("Q", Q), ("KC", KC), ("kS", kS), ("V", V)):
        got = np.stack([host(t_[b, t]) for b, t in toks])
        assert rel_l2(got, ref[name][0]) <= TOL_BF16, name

    # (2) max logit of 16 heads over the whole batch (oracle restricted to those heads' columns)
    heads = sorted(set(L["hot_heads"]) | {0, 31, 62, 95})[:16]
    WQs, WKVs = _head_cols(L["W_UQ"], L["W_UKV"], geom, heads)
    g16 = _sub_geom(geom, len(heads))
    up16 = oracle.up_proj(L["x"], L["W_DQ"], L["w_q"], WQs, L["W_DKV"], L["w_kv"], WKVs, g16, "bf16")
    ref_ml = oracle.head_maxlogit(up16["Q"], up16["KC"], up16["kS"], range(len(heads)))
    want = np.array([ref_ml[i] for i in range(len(heads))])
    got = ml1[heads]
    assert max_rel(got, want) <= TOL_MAXLOGIT
    margins = np.abs(want - tau) / tau
    print("max logit (oracle) of sampled heads:", dict(zip(heads, np.round(want, 3))))
    print("relative margin to tau:", dict(zip(heads, np.round(margins, 4))))

    # (3) clip on the GPU with its own max logits; clipped set on the sampled heads equals the oracle's
    WQ, WKV = Wd["W_UQ"].clone(), Wd["W_UKV"].clone()
    clipped = torch.empty(geom.H, dtype=torch.uint8, device="cuda")
    gamma = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.qkclip_rescale(geom, WQ, WKV, ml, tau, clipped, gamma)
    check_status()
    clip_gpu = host(clipped)
    np.testing.assert_array_equal(clip_gpu[heads], (want.astype(np.float32) > np.float32(tau)).astype(np.uint8))
    assert clip_gpu.sum() >= 1
    # every head outside the scaled set stays under tau
    assert set(np.nonzero(clip_gpu)[0]) <= set(L["hot_heads"])

    # (4) recompute with the clipped weights
    _, _, _, _, ml2 = run(WQ, WKV)
    ml2 = host(ml2)
    for h in range(geom.H):
        if clip_gpu[h]:
            assert abs(ml2[h] - tau) / tau <= TOL_BF16, (h, ml1[h], ml2[h])
        else:
            assert ml2[h] == ml1[h], h
