"""Pins for the oracle's absorbed-latent decode.

The absorbed form is an exact algebraic rewrite of attention over
materialised per-head keys and values, so the two oracle functions must agree
to rounding; the materialised form is in turn checked against torch SDPA, the
one-token case against its closed form, and the whole decode against the
causal attention oracle at the last position of a prefix.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_mla_qk_b200 import synth

G = synth.Geom(H=3, d_model=24, q_lora=16, kv_lora=12, d_c=5, d_s=3, d_v=4)


def _case(lens=(1, 7, 20), seed=0, gate=False):
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    cache = rng.standard_normal((int(offs[-1]), G.kv_lora + G.d_s))
    q = rng.standard_normal((len(lens), G.H, G.d_qk))
    W_UKV = rng.standard_normal((G.kv_lora, G.H * (G.d_c + G.d_v))) / math.sqrt(G.kv_lora)
    g = rng.standard_normal((len(lens), G.H * G.d_v)) if gate else None
    return q, W_UKV, cache, offs, g


@pytest.mark.parametrize("gate", [False, True])
def test_absorbed_equals_materialised(gate):
    q, W, cache, offs, g = _case(gate=gate)
    a = oracle.decode_absorbed(q, W, cache, offs, G, g)
    m = oracle.decode_materialised(q, W, cache, offs, G, g)
    assert np.linalg.norm(a - m) / np.linalg.norm(m) < 1e-12


def test_materialised_matches_sdpa():
    q, W, cache, offs, _ = _case(lens=(9,), seed=1)
    m = oracle.decode_materialised(q, W, cache, offs, G)
    C = torch.from_numpy(cache)
    for h in range(G.H):
        c0 = h * (G.d_c + G.d_v)
        Wt = torch.from_numpy(W)
        K = torch.cat([C[:, :G.kv_lora] @ Wt[:, c0:c0 + G.d_c], C[:, G.kv_lora:]], -1)
        Vh = C[:, :G.kv_lora] @ Wt[:, c0 + G.d_c:c0 + G.d_c + G.d_v]
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, h])[None, None, None], K[None, None], Vh[None, None],
            scale=1.0 / math.sqrt(G.d_qk))
        np.testing.assert_allclose(m[0, h], o[0, 0, 0].numpy(), rtol=1e-12, atol=1e-14)


def test_single_token_context_is_its_value():
    q, W, cache, offs, _ = _case(lens=(1,), seed=2)
    a = oracle.decode_absorbed(q, W, cache, offs, G)
    for h in range(G.H):
        c0 = h * (G.d_c + G.d_v)
        want = cache[0, :G.kv_lora] @ W[:, c0 + G.d_c:c0 + G.d_c + G.d_v]
        np.testing.assert_allclose(a[0, h], want, rtol=1e-13, atol=1e-15)


def test_decode_equals_causal_attention_at_last_position():
    """Latent cache from the up-projection oracle + absorbed decode == row T-1 of causal attention."""
    geom = synth.Geom(H=2, d_model=20, q_lora=12, kv_lora=10, d_c=4, d_s=3, d_v=5)
    rng = np.random.default_rng(3)
    W = synth.layer_weights(geom, rng, with_gate_out=False)
    x = rng.standard_normal((1, 13, geom.d_model))
    up = oracle.up_proj(x, W["W_DQ"], W["w_q"], W["W_UQ"], W["W_DKV"], W["w_kv"], W["W_UKV"], geom, "f64")
    O, _ = oracle.attention(up["Q"], up["KC"], up["kS"], up["V"], None)
    T = x.shape[1]
    dec = oracle.decode_absorbed(up["Q"][:, T - 1], W["W_UKV"], up["cache"][0], np.array([0, T]), geom)
    np.testing.assert_allclose(dec[0], O[0, T - 1], rtol=1e-11, atol=1e-13)


def test_planted_mistake_wrong_scale_is_caught():
    q, W, cache, offs, _ = _case(seed=4)
    a = oracle.decode_absorbed(q, W, cache, offs, G)
    # the same numbers read with a 576-wide "head" scale would differ from the 192-wide one
    scale_ratio = math.sqrt((G.kv_lora + G.d_s) / G.d_qk)
    b = oracle.decode_absorbed(q / scale_ratio, W, cache, offs, G)
    assert not np.allclose(a, b, rtol=1e-6)


@pytest.mark.parametrize("fn", [oracle.decode_absorbed, oracle.decode_materialised])
def test_empty_cache_gives_zero_and_leaves_the_others(fn):
    """A sequence with no cached token decodes to 0 (the empty sum; the pages
    never decode an empty cache), and dropping it changes no other sequence."""
    lens = (0, 7, 0, 20, 0)
    q, W, cache, offs, g = _case(lens=lens, seed=3, gate=True)
    got = fn(q, W, cache, offs, G, g)
    keep = [i for i, L in enumerate(lens) if L > 0]
    for i, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(got[i], np.zeros_like(got[i]))
    offs2 = np.concatenate([[0], np.cumsum([lens[i] for i in keep])]).astype(np.int64)
    want = fn(q[keep], W, cache, offs2, G, g[keep])
    assert np.array_equal(got[keep], want)
