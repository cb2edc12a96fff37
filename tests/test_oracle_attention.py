"""Pins for the oracle's causal gated attention and per-head max logit.

Each test ties ``oracle.attention`` to something other than itself: torch's
scaled_dot_product_attention (an independent library routine), closed forms
(t = 0, T = 1, identical keys), invariants (rows of A sum to one, future keys
do not matter, the max logit ignores V and g) and brute force on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_mla_qk_b200 import synth


def _tiny(B=2, T=9, H=3, d_c=8, d_s=4, d_v=5, seed=0, gate=True):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, T, H, d_c + d_s))
    KC = rng.standard_normal((B, T, H, d_c))
    kS = rng.standard_normal((B, T, d_s))
    V = rng.standard_normal((B, T, H, d_v))
    g = rng.standard_normal((B, T, H * d_v)) if gate else None
    return Q, KC, kS, V, g


def _sdpa(Q, KC, kS, V, g):
    """Library routine: torch SDPA in float64 with K_h = [K^C_h | k^S] broadcast to all heads."""
    B, T, H, d_qk = Q.shape
    q = torch.from_numpy(Q).permute(0, 2, 1, 3)
    k = torch.cat([torch.from_numpy(KC), torch.from_numpy(kS)[:, :, None, :].expand(B, T, H, kS.shape[-1])], -1)
    k = k.permute(0, 2, 1, 3)
    v = torch.from_numpy(V).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=1.0 / math.sqrt(d_qk))
    o = o.permute(0, 2, 1, 3).numpy()
    if g is not None:
        o = o * (1.0 / (1.0 + np.exp(-g.reshape(o.shape))))
    return o


def _brute_maxlogit(Q, KC, kS):
    B, T, H, d_qk = Q.shape
    out = []
    for h in range(H):
        best = -math.inf
        for b in range(B):
            for t in range(T):
                for s in range(t + 1):
                    dot = 0.0
                    for k in range(KC.shape[-1]):
                        dot += Q[b, t, h, k] * KC[b, s, h, k]
                    for k in range(kS.shape[-1]):
                        dot += Q[b, t, h, KC.shape[-1] + k] * kS[b, s, k]
                    best = max(best, dot / math.sqrt(d_qk))
        out.append(best)
    return np.array(out)


def test_matches_torch_sdpa():
    Q, KC, kS, V, g = _tiny()
    O, _ = oracle.attention(Q, KC, kS, V, g)
    np.testing.assert_allclose(O, _sdpa(Q, KC, kS, V, g), rtol=1e-12, atol=1e-12)


def test_matches_torch_sdpa_across_row_chunks():
    Q, KC, kS, V, g = _tiny(B=1, T=37, seed=3)
    O, _ = oracle.attention(Q, KC, kS, V, g, row_chunk=8)
    np.testing.assert_allclose(O, _sdpa(Q, KC, kS, V, g), rtol=1e-12, atol=1e-12)


def test_rows_of_A_sum_to_one():
    Q, KC, kS, V, _ = _tiny(seed=1)
    O, _ = oracle.attention(Q, KC, kS, np.ones_like(V), None)
    assert np.max(np.abs(O - 1.0)) < 1e-12


def test_first_position_is_gated_first_value():
    Q, KC, kS, V, g = _tiny(seed=2)
    O, _ = oracle.attention(Q, KC, kS, V, g)
    B, T, H, d_v = V.shape
    sig = 1.0 / (1.0 + np.exp(-g.reshape(B, T, H, d_v)))
    np.testing.assert_allclose(O[:, 0], sig[:, 0] * V[:, 0], rtol=0, atol=1e-15)


def test_single_position_sequence():
    Q, KC, kS, V, g = _tiny(T=1, seed=4)
    O, ml = oracle.attention(Q, KC, kS, V, None)
    np.testing.assert_allclose(O[:, 0], V[:, 0], rtol=0, atol=1e-15)
    want = [max(float(np.dot(Q[b, 0, h], np.concatenate([KC[b, 0, h], kS[b, 0]]))) for b in range(Q.shape[0]))
            / math.sqrt(Q.shape[-1]) for h in range(Q.shape[2])]
    np.testing.assert_allclose(ml, want, rtol=1e-14)


def test_identical_keys_average_values():
    Q, KC, kS, V, _ = _tiny(seed=5)
    KC[:] = KC[:, :1]
    kS[:] = kS[:, :1]
    O, _ = oracle.attention(Q, KC, kS, V, None)
    T = V.shape[1]
    prefix_mean = np.cumsum(V, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    np.testing.assert_allclose(O, prefix_mean, rtol=1e-12, atol=1e-12)


def test_future_keys_do_not_matter():
    Q, KC, kS, V, g = _tiny(T=12, seed=6)
    t = 5
    O, _ = oracle.attention(Q, KC, kS, V, g)
    rng = np.random.default_rng(7)
    KC2, kS2, V2 = KC.copy(), kS.copy(), V.copy()
    KC2[:, t + 1:] = rng.standard_normal(KC2[:, t + 1:].shape) * 50
    kS2[:, t + 1:] = rng.standard_normal(kS2[:, t + 1:].shape) * 50
    V2[:, t + 1:] = rng.standard_normal(V2[:, t + 1:].shape) * 50
    O2, _ = oracle.attention(Q, KC2, kS2, V2, g)
    np.testing.assert_array_equal(O[:, :t + 1], O2[:, :t + 1])


def test_maxlogit_brute_force_and_invariance():
    Q, KC, kS, V, g = _tiny(B=2, T=6, seed=8)
    _, ml = oracle.attention(Q, KC, kS, V, g)
    np.testing.assert_allclose(ml, _brute_maxlogit(Q, KC, kS), rtol=1e-13)
    _, ml2 = oracle.attention(Q, KC, kS, V * 7 + 3, None)
    np.testing.assert_array_equal(ml, ml2)
    hm = oracle.head_maxlogit(Q, KC, kS, range(Q.shape[2]), row_chunk=4)
    np.testing.assert_allclose([hm[h] for h in range(Q.shape[2])], ml, rtol=1e-13)


def test_maxlogit_ignores_masked_pairs():
    # A huge logit planted only at s > t must not be counted.
    Q, KC, kS, V, _ = _tiny(B=1, T=4, H=1, seed=9)
    KC[0, 3, 0, :] = 1e3 * Q[0, 0, 0, :KC.shape[-1]]
    _, ml = oracle.attention(Q, KC, kS, V, None)
    np.testing.assert_allclose(ml, _brute_maxlogit(Q, KC, kS), rtol=1e-13)
    assert ml[0] < 100


def test_attention_rows_agree_with_full():
    Q, KC, kS, V, g = _tiny(B=2, T=11, seed=10)
    O, _ = oracle.attention(Q, KC, kS, V, g)
    rows = [(0, 0, 0), (1, 10, 2), (0, 7, 1)]
    Or, rmax = oracle.attention_rows(Q, KC, kS, V, g, rows)
    for i, (b, t, h) in enumerate(rows):
        np.testing.assert_allclose(Or[i], O[b, t, h], rtol=1e-13, atol=1e-15)


def test_k3_geometry_scale_is_one_over_sqrt_192():
    # With q = k = e_0 * a the only logit at t=0 is a^2 / sqrt(192).
    g = synth.K3
    Q = np.zeros((1, 1, 1, g.d_qk)); KC = np.zeros((1, 1, 1, g.d_c)); kS = np.zeros((1, 1, g.d_s))
    Q[0, 0, 0, 0] = 3.0; KC[0, 0, 0, 0] = 4.0
    Q[0, 0, 0, g.d_c] = 2.0; kS[0, 0, 0] = 5.0   # the shared-key part contributes too
    _, ml = oracle.attention(Q, KC, kS, np.zeros((1, 1, 1, g.d_v)), None)
    assert ml[0] == pytest.approx((12.0 + 10.0) / math.sqrt(192.0), rel=1e-15)


# --- planted mistakes: each broken variant must fail a pin above -------------
def _broken_no_shared_key(Q, KC, kS, V, g):
    return oracle.attention(Q, KC, np.zeros_like(kS), V, g)


def _broken_wrong_scale(Q, KC, kS, V, g):
    return oracle.attention(Q * math.sqrt(Q.shape[-1] / KC.shape[-1]), KC, kS, V, g)


def _broken_anticausal(Q, KC, kS, V, g):
    O, ml = oracle.attention(Q[:, ::-1], KC[:, ::-1], kS[:, ::-1], V[:, ::-1], None if g is None else g[:, ::-1])
    return O[:, ::-1], ml


@pytest.mark.parametrize("broken", [_broken_no_shared_key, _broken_wrong_scale, _broken_anticausal])
def test_planted_mistakes_are_caught(broken):
    Q, KC, kS, V, g = _tiny(seed=11)
    O, _ = broken(Q, KC, kS, V, g)
    assert not np.allclose(O, _sdpa(Q, KC, kS, V, g), rtol=1e-6, atol=1e-6)
