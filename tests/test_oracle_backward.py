"""Pins of the oracle's training functions: the backward is checked against
central finite differences of the forward oracle (independent of the
backward's own algebra) and against torch autograd in float64 (a library
routine); the row log-sum-exp against scipy's logsumexp."""
import numpy as np
import pytest

import oracle


def _case(B, T, H, d_c, d_s, d_v, seed, gate=True):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, T, H, d_c + d_s))
    KC = rng.standard_normal((B, T, H, d_c))
    kS = rng.standard_normal((B, T, d_s))
    V = rng.standard_normal((B, T, H, d_v))
    g = rng.standard_normal((B, T, H * d_v)) if gate else None
    W = rng.standard_normal((B, T, H * d_v))          # L = sum(W * o), so dL/do = W
    return Q, KC, kS, V, g, W


def _loss(Q, KC, kS, V, g, W):
    O, _ = oracle.attention(Q, KC, kS, V, g)
    B, T = Q.shape[:2]
    return float((O.reshape(B, T, -1) * W).sum())


@pytest.mark.parametrize("gate", [True, False])
def test_backward_matches_finite_differences(gate):
    Q, KC, kS, V, g, W = _case(2, 5, 2, 4, 2, 3, seed=11, gate=gate)
    grads = oracle.attention_backward(Q, KC, kS, V, g, W)
    args = [Q, KC, kS, V, g]
    eps = 1e-6
    for which, (x, dx) in enumerate(zip(args, grads)):
        if x is None:
            assert dx is None
            continue
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            ap, am = list(args), list(args)
            ap[which], am[which] = xp, xm
            num[i] = (_loss(*ap, W) - _loss(*am, W)) / (2 * eps)
        assert np.allclose(dx, num, rtol=1e-5, atol=1e-7), which


def test_backward_matches_torch_autograd():
    torch = pytest.importorskip("torch")
    Q, KC, kS, V, g, W = _case(1, 9, 3, 6, 4, 5, seed=12)
    t = {k: torch.tensor(v, requires_grad=True) for k, v in zip("Q KC kS V g".split(), (Q, KC, kS, V, g))}
    B, T, H, d_qk = Q.shape
    d_v = V.shape[-1]
    outs = []
    for h in range(H):
        K = torch.cat([t["KC"][:, :, h], t["kS"]], dim=-1)
        o = torch.nn.functional.scaled_dot_product_attention(
            t["Q"][:, :, h].unsqueeze(1), K.unsqueeze(1), t["V"][:, :, h].unsqueeze(1), is_causal=True)[:, 0]
        outs.append(o)
    O = torch.stack(outs, dim=2).reshape(B, T, H * d_v) * torch.sigmoid(t["g"])
    (O * torch.tensor(W)).sum().backward()
    got = oracle.attention_backward(Q, KC, kS, V, g, W)
    for name, d in zip("Q KC kS V g".split(), got):
        assert np.allclose(d, t[name].grad.numpy(), rtol=1e-10, atol=1e-12), name


def test_shared_key_gradient_is_the_sum_over_heads():
    """Duplicating a head's parameters doubles k^S's gradient share and leaves
    each head's own gradients unchanged."""
    Q, KC, kS, V, g, W = _case(1, 6, 1, 4, 2, 3, seed=13)
    one = oracle.attention_backward(Q, KC, kS, V, g, W)
    two = oracle.attention_backward(np.concatenate([Q, Q], 2), np.concatenate([KC, KC], 2), kS,
                                    np.concatenate([V, V], 2), np.concatenate([g, g], 2),
                                    np.concatenate([W, W], 2))
    assert np.allclose(two[2], 2 * one[2])
    assert np.allclose(two[0][:, :, 1], one[0][:, :, 0]) and np.allclose(two[3][:, :, 0], one[3][:, :, 0])


def test_lse_matches_scipy_and_brackets_the_row_max():
    scipy_special = pytest.importorskip("scipy.special")
    Q, KC, kS, V, g, W = _case(2, 7, 2, 4, 2, 3, seed=14)
    lse = oracle.attention_lse(Q, KC, kS)
    B, T, H, d_qk = Q.shape
    for b in range(B):
        for h in range(H):
            K = np.concatenate([KC[b, :, h], kS[b]], -1)
            S = Q[b, :, h] @ K.T / np.sqrt(d_qk)
            for t in range(T):
                row = S[t, :t + 1]
                assert np.isclose(lse[b, t, h], scipy_special.logsumexp(row), rtol=1e-13)
                assert row.max() - 1e-12 <= lse[b, t, h] <= row.max() + np.log(t + 1) + 1e-12
