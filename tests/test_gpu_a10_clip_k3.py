"""The QK-Clip chain at Kimi K3 size (bf16): x[4,4096,7168] -> up-projections
-> attention max logit over the batch -> clip at tau = 100 -> recompute.

Checked against the oracle in full:
  * every element of Q, K^C, k^S and V against the oracle's up-projection of
    the same x (a many-tile GEMM: M = 16384 rows, each persistent CTA walks
    dozens of output tiles);
  * the max logit of all 96 heads, both from the Q / K^C / k^S the attention
    kernel received and from the oracle's own up-projection;
  * the clipped set over all 96 heads, bit-exact against both oracle sets,
    with every head's margin to tau reported;
  * the clipped weights bit-exact against the oracle's clip of the same max
    logits; after the recompute, clipped heads land on tau within the bf16
    bound and unclipped heads' max logits are bit-identical to the first pass.
"""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_MAXLOGIT, check_status, dev, host, max_rel, per_head, rel_l2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _all_heads_maxlogit(Q, KC, kS, H):
    ref = per_head(lambda h: oracle.head_maxlogit(Q, KC, kS, [h])[h], range(H))
    return np.array([ref[h] for h in range(H)])


def test_k3_clip_chain():
    import torch
    import gated_mla_qk_b200 as gm
    L = synth.k3_clip_layer()
    geom, tau = L["geom"], L["tau"]
    B, T = L["x"].shape[:2]
    H = geom.H
    x = dev(L["x"], "bf16")
    Wd = {k: dev(L[k], "bf16") for k in ("W_DQ", "w_q", "W_UQ", "W_DKV", "w_kv", "W_UKV")}
    bf = torch.bfloat16

    def run(W_UQ, W_UKV):
        Q = torch.empty(B, T, H, geom.d_qk, dtype=bf, device="cuda")
        KC = torch.empty(B, T, H, geom.d_c, dtype=bf, device="cuda")
        kS = torch.empty(B, T, geom.d_s, dtype=bf, device="cuda")
        V = torch.empty(B, T, H, geom.d_v, dtype=bf, device="cuda")
        gm.mla_up_proj(geom, x, Wd["W_DQ"], Wd["w_q"], W_UQ, Wd["W_DKV"], Wd["w_kv"], W_UKV, Q, KC, kS, V)
        O = torch.empty(B, T, H * geom.d_v, dtype=bf, device="cuda")
        ml = torch.empty(H, dtype=torch.float32, device="cuda")
        gm.mla_attn_fwd(geom, Q, KC, kS, V, None, O, ml)
        check_status()
        return Q, KC, kS, V, ml

    Q, KC, kS, V, ml = run(Wd["W_UQ"], Wd["W_UKV"])
    ml1 = host(ml)
    got = {name: host(t) for name, t in (("Q", Q), ("KC", KC), ("kS", kS), ("V", V))}
    del Q, KC, kS, V

    # (1) the up-projections, every element, against the oracle on the same x
    ref = oracle.up_proj(L["x"], L["W_DQ"], L["w_q"], L["W_UQ"], L["W_DKV"], L["w_kv"], L["W_UKV"], geom, "bf16")
    for name in ("Q", "KC", "kS", "V"):
        assert rel_l2(got[name], ref[name]) <= TOL_BF16, name

    # (2) the max logit of every head: (a) from what the attention kernel received,
    # (b) from the oracle's own up-projection
    ml_a = _all_heads_maxlogit(got["Q"], got["KC"], got["kS"], H)
    assert max_rel(ml1, ml_a) <= TOL_MAXLOGIT
    del got
    ml_b = _all_heads_maxlogit(ref["Q"], ref["KC"], ref["kS"], H)
    del ref
    assert max_rel(ml1, ml_b) <= TOL_MAXLOGIT
    margins = np.abs(ml_b - tau) / tau
    print("max logit (oracle) per head:", dict(enumerate(np.round(ml_b, 3))))
    print("relative margin to tau: min %.4f at head %d" % (margins.min(), int(margins.argmin())))
    # a head within the max logit's own error of tau would make the clipped set ill-posed
    assert margins.min() > 1e-4, "a head sits within 1e-4 of tau"

    # (3) clip on the GPU with its own max logits: the clipped set over all heads,
    # and the clipped weights, bit-exact
    WQ, WKV = Wd["W_UQ"].clone(), Wd["W_UKV"].clone()
    clipped = torch.empty(H, dtype=torch.uint8, device="cuda")
    gamma = torch.empty(H, dtype=torch.float32, device="cuda")
    gm.qkclip_rescale(geom, WQ, WKV, ml, tau, clipped, gamma)
    check_status()
    clip_gpu = host(clipped)
    for want in (ml_a, ml_b):
        np.testing.assert_array_equal(clip_gpu, (want.astype(np.float32) > np.float32(tau)).astype(np.uint8))
    assert 1 <= clip_gpu.sum() <= len(L["hot_heads"])
    WQ_ref, WKV_ref, clip_ref, gamma_ref = oracle.qkclip(L["W_UQ"], L["W_UKV"], ml1, tau, geom, "bf16")
    np.testing.assert_array_equal(clip_gpu, clip_ref)
    np.testing.assert_array_equal(host(WQ).view(np.uint32), WQ_ref.view(np.uint32))
    np.testing.assert_array_equal(host(WKV).view(np.uint32), WKV_ref.view(np.uint32))
    g = host(gamma)
    np.testing.assert_array_equal(g[clip_gpu == 1], np.asarray(gamma_ref)[clip_gpu == 1])

    # (4) recompute with the clipped weights
    _, _, _, _, ml2 = run(WQ, WKV)
    ml2 = host(ml2)
    for h in range(H):
        if clip_gpu[h]:
            assert abs(ml2[h] - tau) / tau <= TOL_BF16, (h, ml1[h], ml2[h])
        else:
            assert ml2[h] == ml1[h], h
