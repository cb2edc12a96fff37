"""Pins for the oracle's bf16 rounding, RMSNorm, up-projections, QK-Clip and the tiny layer."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from gated_mla_qk_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --- bf16 rounding -----------------------------------------------------------
def test_bf16_round_matches_torch_cast_f32():
    rng = np.random.default_rng(0)
    a = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 10 ** rng.uniform(-6, 6, 100000).astype(np.float32),
        # exact ties between two bf16 values, both parities of the kept field
        (np.arange(1, 2000, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32),
    ])
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(oracle.bf16_round(a).view(np.uint32), want.view(np.uint32))


def test_bf16_round_f64_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(20000) * 10 ** rng.uniform(-5, 5, 20000)
    r = oracle.bf16_round(a).astype(np.float64)
    bits = oracle.bf16_round(a).view(np.uint32)
    up = (bits + np.uint32(0x10000)).view(np.float32).astype(np.float64)
    dn = (bits - np.uint32(0x10000)).view(np.float32).astype(np.float64)
    err = np.abs(a - r)
    assert np.all(err <= np.abs(a - up)) and np.all(err <= np.abs(a - dn))
    # a value exactly halfway between two bf16 neighbours goes to the even one
    lo = np.float64(np.uint32(0x3F810000).view(np.float32))     # odd kept field
    hi = np.float64(np.uint32(0x3F820000).view(np.float32))
    assert oracle.bf16_round(np.array([(lo + hi) / 2])).view(np.uint32)[0] == 0x3F820000


# --- RMSNorm -----------------------------------------------------------------
def test_rms_norm_matches_torch():
    rng = np.random.default_rng(2)
    c = rng.standard_normal((5, 7, 64)) * 3
    w = rng.standard_normal(64)
    want = torch.nn.functional.rms_norm(torch.from_numpy(c), (64,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rms_norm(c, w, 1e-6), want, rtol=1e-13, atol=1e-13)


def test_rms_norm_unit_mean_square():
    rng = np.random.default_rng(3)
    c = rng.standard_normal((4, 512)) * 7
    out = oracle.rms_norm(c, np.ones(512), 1e-6)
    ms = np.mean(c * c, axis=-1)
    np.testing.assert_allclose(np.mean(out * out, axis=-1), ms / (ms + 1e-6), rtol=1e-13)


# --- up-projection layout ----------------------------------------------------
def test_up_proj_head_split_with_identity_weights():
    """Identity projections expose where each head's q^C, q^S, K^C, V and k^S come from."""
    geom = synth.Geom(H=3, d_model=20, q_lora=3 * 6, kv_lora=3 * 9, d_c=4, d_s=2, d_v=5, rms_eps=0.0)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 3, geom.d_model))
    W_DQ = np.zeros((geom.d_model, geom.q_lora)); W_DQ[:geom.q_lora, :] = np.eye(geom.q_lora)
    W_UQ = np.eye(geom.q_lora)
    W_UKV = np.eye(geom.kv_lora)
    # d_model < kv_lora + d_s: build W_DKV so column j reads x[j mod d_model]
    W_DKV = np.zeros((geom.d_model, geom.kv_lora + geom.d_s))
    for j in range(geom.kv_lora + geom.d_s):
        W_DKV[j % geom.d_model, j] = 1.0
    up = oracle.up_proj(x, W_DQ, np.ones(geom.q_lora), W_UQ, W_DKV, np.ones(geom.kv_lora), W_UKV, geom, "f64")
    cq = x[..., :geom.q_lora]
    cq_hat = cq / np.sqrt(np.mean(cq * cq, -1, keepdims=True))
    ckv_ks = x[..., [j % geom.d_model for j in range(geom.kv_lora + geom.d_s)]]
    ckv = ckv_ks[..., :geom.kv_lora]
    ckv_hat = ckv / np.sqrt(np.mean(ckv * ckv, -1, keepdims=True))
    for h in range(geom.H):
        np.testing.assert_allclose(up["Q"][:, :, h, :], cq_hat[..., h * 6:(h + 1) * 6], rtol=1e-14)
        np.testing.assert_allclose(up["KC"][:, :, h, :], ckv_hat[..., h * 9:h * 9 + 4], rtol=1e-14)
        np.testing.assert_allclose(up["V"][:, :, h, :], ckv_hat[..., h * 9 + 4:(h + 1) * 9], rtol=1e-14)
    # k^S is the un-normalised tail of the joint down-projection
    np.testing.assert_array_equal(up["kS"], ckv_ks[..., geom.kv_lora:])
    np.testing.assert_allclose(up["cache"], np.concatenate([ckv_hat, ckv_ks[..., geom.kv_lora:]], -1), rtol=1e-14)


def test_k3_parameter_accounting_matches_page():
    facts = json.load(open(os.path.join(GOLDEN, "k3_page_facts.json")))
    g = synth.K3
    for k, v in facts["geometry"].items():
        assert getattr(g, k) == v
    W = {k: v.shape for k, v in {
        "W_DQ": np.empty((g.d_model, g.q_lora), np.int8), "w_q": np.empty(g.q_lora, np.int8),
        "W_UQ": np.empty((g.q_lora, g.H * g.d_qk), np.int8),
        "W_DKV": np.empty((g.d_model, g.kv_lora + g.d_s), np.int8), "w_kv": np.empty(g.kv_lora, np.int8),
        "W_UKV": np.empty((g.kv_lora, g.H * (g.d_c + g.d_v)), np.int8),
        "W_g": np.empty((g.d_model, g.H * g.d_v), np.int8), "W_O": np.empty((g.H * g.d_v, g.d_model), np.int8),
    }.items()}
    n = {k: int(np.prod(s)) for k, s in W.items()}
    assert n["W_DQ"] + n["w_q"] + n["W_UQ"] == facts["params_query_heads"]
    assert n["W_DKV"] + n["w_kv"] + n["W_UKV"] == facts["params_key_value_heads"]
    assert n["W_g"] == facts["params_output_gate"]
    assert n["W_O"] == facts["params_output_proj"]
    assert sum(n.values()) == facts["params_per_instance"]
    assert sum(n.values()) * facts["mla_layers"] == facts["params_24_layers"]
    # cache table: 2 * H * d_v values per token uncompressed vs kv_lora + d_s with the latent
    assert 2 * g.H * g.d_v == facts["cache_values_per_token_uncompressed"]
    assert (g.kv_lora, g.d_s) == (facts["cache_values_per_token_mla_latent"], facts["cache_values_per_token_mla_shared_key"])
    assert round(facts["cache_values_per_token_uncompressed"] / (g.kv_lora + g.d_s)) == facts["cache_ratio_approx"]
    # 1M tokens x 576 x 24 layers x 2 B: the page's "29" matches decimal GB (27.0 GiB)
    nbytes = 1048576 * (g.kv_lora + g.d_s) * 24 * 2
    assert round(nbytes / 1e9) == facts["cache_1M_tokens_bf16_approx_gib_printed"]


def test_up_proj_bf16_outputs_are_bf16_values():
    geom = synth.Geom(H=2, d_model=32, q_lora=16, kv_lora=16, d_c=8, d_s=4, d_v=8)
    rng = np.random.default_rng(5)
    W = synth.layer_weights(geom, rng, with_gate_out=False)
    x = rng.standard_normal((1, 5, 32)).astype(np.float32)
    up = oracle.up_proj(x, W["W_DQ"], W["w_q"], W["W_UQ"], W["W_DKV"], W["w_kv"], W["W_UKV"], geom, "bf16")
    for k in ("Q", "KC", "kS", "V"):
        a = up[k].astype(np.float32)
        np.testing.assert_array_equal(oracle.bf16_round(a), a)


# --- QK-Clip -----------------------------------------------------------------
def _tiny_layer_pieces():
    L = synth.tiny_layer(0)
    return L, L["geom"]


def _maxlogit_from_weights(L, geom, WQ, WKV):
    up = oracle.up_proj(L["x"], L["W_DQ"], L["w_q"], WQ, L["W_DKV"], L["w_kv"], WKV, geom, "f64")
    _, ml = oracle.attention(up["Q"], up["KC"], up["kS"], up["V"], None)
    return ml, up


def test_clip_brings_clipped_heads_to_tau_and_leaves_others():
    L, geom = _tiny_layer_pieces()
    tau = L["tau"]
    ml, up = _maxlogit_from_weights(L, geom, L["W_UQ"], L["W_UKV"])
    WQ, WKV, clipped, gamma = oracle.qkclip(L["W_UQ"], L["W_UKV"], ml.astype(np.float32), tau, geom, "f32")
    assert clipped.tolist() == [int(m > tau) for m in ml.astype(np.float32)]
    assert clipped.sum() >= 1, "the tiny layer is built so that at least one head clips"
    ml2, up2 = _maxlogit_from_weights(L, geom, WQ, WKV)
    for h in range(geom.H):
        if clipped[h]:
            assert ml2[h] == pytest.approx(tau, rel=1e-6)
            # every logit of the head scaled by gamma: S' = gamma * S
            S = np.einsum("btd,bsd->bts", up["Q"][:, :, h], np.concatenate([up["KC"][:, :, h], up["kS"]], -1))
            S2 = np.einsum("btd,bsd->bts", up2["Q"][:, :, h], np.concatenate([up2["KC"][:, :, h], up2["kS"]], -1))
            np.testing.assert_allclose(S2, float(gamma[h]) * S, rtol=1e-5, atol=1e-5 * np.abs(S).max())
        else:
            assert ml2[h] == ml[h]
            q0, k0 = h * geom.d_qk, h * (geom.d_c + geom.d_v)
            np.testing.assert_array_equal(WQ[:, q0:q0 + geom.d_qk], L["W_UQ"][:, q0:q0 + geom.d_qk])
            np.testing.assert_array_equal(WKV[:, k0:k0 + geom.d_c], L["W_UKV"][:, k0:k0 + geom.d_c])
    # V columns are never touched
    for h in range(geom.H):
        k0 = h * (geom.d_c + geom.d_v) + geom.d_c
        np.testing.assert_array_equal(WKV[:, k0:k0 + geom.d_v], L["W_UKV"][:, k0:k0 + geom.d_v])


def test_clip_threshold_is_strict_and_ignores_negative():
    geom = synth.Geom(H=4, d_model=8, q_lora=4, kv_lora=4, d_c=2, d_s=1, d_v=2)
    rng = np.random.default_rng(6)
    WQ = rng.standard_normal((4, 4 * 3)).astype(np.float32)
    WKV = rng.standard_normal((4, 4 * 4)).astype(np.float32)
    ml = np.array([10.0, 10.000001, -50.0, -np.inf], np.float32)
    WQ2, WKV2, clipped, gamma = oracle.qkclip(WQ, WKV, ml, 10.0, geom, "f32")
    assert clipped.tolist() == [0, 1, 0, 0]
    assert gamma[0] == 1 and gamma[2] == 1 and gamma[3] == 1
    assert gamma[1] == np.float32(10.0) / np.float32(10.000001)


def test_clip_bf16_bits_match_torch_float32_then_cast():
    geom = synth.Geom(H=3, d_model=8, q_lora=16, kv_lora=16, d_c=4, d_s=2, d_v=4)
    rng = np.random.default_rng(7)
    WQ = synth.round_storage(rng.standard_normal((16, 3 * 6)), "bf16")
    WKV = synth.round_storage(rng.standard_normal((16, 3 * 8)), "bf16")
    ml = np.array([3.0, 41.7, 123.4], np.float32)
    WQ2, WKV2, clipped, gamma = oracle.qkclip(WQ, WKV, ml, 20.0, geom, "bf16")
    tq, tkv = torch.from_numpy(WQ.copy()), torch.from_numpy(WKV.copy())
    for h in (1, 2):
        gam = torch.tensor(20.0, dtype=torch.float32) / torch.tensor(float(ml[h]), dtype=torch.float32)
        root = torch.sqrt(gam)
        assert float(gam) == float(gamma[h])
        tq[:, h * 6:h * 6 + 4] = (tq[:, h * 6:h * 6 + 4] * root).to(torch.bfloat16).float()
        tq[:, h * 6 + 4:h * 6 + 6] = (tq[:, h * 6 + 4:h * 6 + 6] * gam).to(torch.bfloat16).float()
        tkv[:, h * 8:h * 8 + 4] = (tkv[:, h * 8:h * 8 + 4] * root).to(torch.bfloat16).float()
    np.testing.assert_array_equal(WQ2.view(np.uint32), tq.numpy().view(np.uint32))
    np.testing.assert_array_equal(WKV2.view(np.uint32), tkv.numpy().view(np.uint32))
    assert clipped.tolist() == [0, 1, 1]


def test_tiny_layer_forward_and_clip_recheck():
    """The tiny fp32 layer end to end: forward, max logit, clip, re-check to 1e-5."""
    L, geom = _tiny_layer_pieces()
    res = oracle.layer_forward(L["x"], L, geom, "f32")
    assert res["delta"].shape == (1, 64, geom.d_model)
    ml = res["maxlogit"]
    # the head scales [1, 2, 4, 8] order the max logits
    assert ml[0] < ml[1] < ml[2] < ml[3]
    WQ, WKV, clipped, gamma = oracle.qkclip(L["W_UQ"], L["W_UKV"], ml.astype(np.float32), L["tau"], geom, "f32")
    W2 = dict(L, W_UQ=WQ, W_UKV=WKV)
    res2 = oracle.layer_forward(L["x"], W2, geom, "f32")
    for h in range(geom.H):
        if clipped[h]:
            assert abs(res2["maxlogit"][h] - L["tau"]) / L["tau"] < 1e-5
        else:
            assert res2["maxlogit"][h] == ml[h]
