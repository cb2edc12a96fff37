"""Planted mistakes in the oracle must be caught by its pins.

Each mutant is one oracle function with one plausible mistake planted in its
own source: a wrong sign, a dropped factor or term, a swapped exponent, a
wrong slice, axis or threshold.  The source is edited as text and executed in
a copy of the oracle module's namespace.  Every pin below checks an
implementation against something other than the oracle's own formula: a
library routine (torch SDPA), brute force, central finite differences of the
forward, the materialised decode form, a closed form or an invariant of the
clip.  The real oracle passes every pin, and each mutant fails at least one.
CPU only.
"""
import inspect
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.mla as M
from gated_mla_qk_b200 import synth


def mutant(name, old, new, helper=None):
    """`name` from the oracle with `old` replaced by `new` in its source (or in
    the source of `helper`, a function `name` calls).  `old` and `new` may be
    tuples of edits made together."""
    ns = dict(vars(M))
    target = helper or name
    src = inspect.getsource(getattr(M, target))
    for o, n in (zip(old, new) if isinstance(old, tuple) else [(old, new)]):
        assert src.count(o) == 1, (target, o)
        src = src.replace(o, n)
    exec(compile(src, f"<mutant of {target}>", "exec"), ns)
    if helper:                                     # re-bind `name` to the namespace that holds the mutated helper
        exec(compile(inspect.getsource(getattr(M, name)), f"<{name}>", "exec"), ns)
    return ns[name]


def failing_pins(pins, impl):
    failed = []
    for pin in pins:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _attn_case():
    rng = np.random.default_rng(21)
    B, T, H, d_c, d_s, d_v = 2, 7, 2, 4, 3, 5
    return (rng.standard_normal((B, T, H, d_c + d_s)), rng.standard_normal((B, T, H, d_c)),
            rng.standard_normal((B, T, d_s)), rng.standard_normal((B, T, H, d_v)),
            rng.standard_normal((B, T, H * d_v)))


def pin_attention_vs_sdpa(impl):
    Q, KC, kS, V, g = _attn_case()
    O, _ = impl(Q, KC, kS, V, g)
    B, T, H, _ = Q.shape
    for h in range(H):
        K = torch.cat([torch.from_numpy(KC[:, :, h]), torch.from_numpy(kS)], -1)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[:, :, h])[:, None], K[:, None], torch.from_numpy(V[:, :, h])[:, None], is_causal=True)[:, 0]
        d_v = V.shape[-1]
        want = o.numpy() * (1 / (1 + np.exp(-g[:, :, h * d_v:(h + 1) * d_v])))
        assert np.allclose(O[:, :, h], want, rtol=1e-10, atol=1e-12)


def pin_maxlogit_brute_force(impl):
    Q, KC, kS, V, g = _attn_case()
    _, ml = impl(Q, KC, kS, V, g)
    B, T, H, d_qk = Q.shape
    for h in range(H):
        best = -math.inf
        for b in range(B):
            for t in range(T):
                for s in range(t + 1):
                    k = list(KC[b, s, h]) + list(kS[b, s])
                    best = max(best, sum(a * c for a, c in zip(Q[b, t, h], k)) / math.sqrt(d_qk))
        assert ml[h] == pytest.approx(best, rel=1e-12)


ATTN_PINS = [pin_attention_vs_sdpa, pin_maxlogit_brute_force]
ATTN_MUTANTS = {
    "anti-causal mask": ("attention", "<= np.arange(t0, t1)[:, None]", ">= np.arange(t0, t1)[:, None]"),
    "scale 1/sqrt(d_v)": ("attention", "scale = 1.0 / math.sqrt(d_qk)", "scale = 1.0 / math.sqrt(d_v)"),
    "gate without sigmoid": ("attention", "O = O * _sigmoid(_f64(g)", "O = O * (_f64(g)"),
    "unscaled max logit": ("attention", "m_h = max(m_h, float(S.max()))", "m_h = max(m_h, float(S.max()) / scale)"),
    "row max over the wrong axis": ("attention", "m = S.max(axis=1, keepdims=True)", "m = S.max(axis=0, keepdims=True)"),
    "shared key dropped": ("attention", "kS[b]], axis=-1)", "0 * kS[b]], axis=-1)", "_head_keys"),
    "shared key from batch item 0": ("attention", "kS[b]], axis=-1)", "kS[0]], axis=-1)", "_head_keys"),
}


def test_attention_pins_pass_on_the_oracle():
    assert failing_pins(ATTN_PINS, oracle.attention) == []


@pytest.mark.parametrize("what", sorted(ATTN_MUTANTS))
def test_attention_mutant_is_caught(what):
    impl = mutant(*ATTN_MUTANTS[what])
    assert failing_pins(ATTN_PINS, impl), what


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
_BWD = {}


def _bwd_case():
    if not _BWD:
        rng = np.random.default_rng(22)
        B, T, H, d_c, d_s, d_v = 2, 4, 2, 3, 2, 3
        args = [rng.standard_normal((B, T, H, d_c + d_s)), rng.standard_normal((B, T, H, d_c)),
                rng.standard_normal((B, T, d_s)), rng.standard_normal((B, T, H, d_v)),
                rng.standard_normal((B, T, H * d_v))]
        W = rng.standard_normal((B, T, H * d_v))

        def loss(a):
            O, _ = oracle.attention(*a)
            return float((O.reshape(B, T, -1) * W).sum())

        eps = 1e-6
        num = []
        for which, x in enumerate(args):
            d = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                i = it.multi_index
                ap, am = list(args), list(args)
                ap[which], am[which] = x.copy(), x.copy()
                ap[which][i] += eps
                am[which][i] -= eps
                d[i] = (loss(ap) - loss(am)) / (2 * eps)
            num.append(d)
        _BWD.update(args=args, W=W, num=num)
    return _BWD


def pin_backward_finite_differences(impl):
    c = _bwd_case()
    got = impl(*c["args"], c["W"])
    for name, a, n in zip(("dQ", "dKC", "dkS", "dV", "dg"), got, c["num"]):
        assert np.allclose(a.reshape(n.shape), n, rtol=1e-5, atol=1e-7), name


BWD_PINS = [pin_backward_finite_differences]
BWD_MUTANTS = {
    "softmax Jacobian sign": ("attention_backward", "(dA - (dA * A).sum(axis=1, keepdims=True))",
                              "(dA + (dA * A).sum(axis=1, keepdims=True))"),
    "gate dropped from dO~": ("attention_backward", "dOt = dO[b, :, h, :] * sg", "dOt = dO[b, :, h, :]"),
    "sigmoid derivative": ("attention_backward", "* Ot * sg * (1.0 - sg)", "* Ot * sg"),
    "shared key gradient of the last head only": ("attention_backward", "dkS[b] += dK[:, d_c:]", "dkS[b] = dK[:, d_c:]"),
    "dK without the scale": ("attention_backward", "dK = (dS.T @ Qh) * scale", "dK = (dS.T @ Qh)"),
    "dV from A instead of A^T": ("attention_backward", "dV[b, :, h, :] = A.T @ dOt", "dV[b, :, h, :] = A @ dOt"),
}


def test_backward_pins_pass_on_the_oracle():
    assert failing_pins(BWD_PINS, oracle.attention_backward) == []


@pytest.mark.parametrize("what", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(what):
    impl = mutant(*BWD_MUTANTS[what])
    assert failing_pins(BWD_PINS, impl), what


# ---------------------------------------------------------------------------
# absorbed decode
# ---------------------------------------------------------------------------
G = synth.Geom(H=3, d_model=24, q_lora=16, kv_lora=12, d_c=5, d_s=3, d_v=4)


def _dec_case(lens, seed):
    rng = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return (rng.standard_normal((len(lens), G.H, G.d_qk)),
            rng.standard_normal((G.kv_lora, G.H * (G.d_c + G.d_v))) / math.sqrt(G.kv_lora),
            rng.standard_normal((int(offs[-1]), G.kv_lora + G.d_s)), offs,
            rng.standard_normal((len(lens), G.H * G.d_v)))


def pin_decode_vs_materialised(impl):
    q, W, cache, offs, g = _dec_case((1, 6, 17), seed=23)
    a = impl(q, W, cache, offs, G, g)
    m = oracle.decode_materialised(q, W, cache, offs, G, g)
    assert np.linalg.norm(a - m) / np.linalg.norm(m) < 1e-12


def pin_decode_one_token(impl):
    q, W, cache, offs, _ = _dec_case((1,), seed=24)
    a = impl(q, W, cache, offs, G)
    for h in range(G.H):
        c0 = h * (G.d_c + G.d_v)
        assert np.allclose(a[0, h], cache[0, :G.kv_lora] @ W[:, c0 + G.d_c:c0 + G.d_c + G.d_v], rtol=1e-13, atol=1e-15)


DEC_PINS = [pin_decode_vs_materialised, pin_decode_one_token]
DEC_MUTANTS = {
    "576-wide scale": ("decode_absorbed", "scale = 1.0 / math.sqrt(geom.d_qk)",
                       "scale = 1.0 / math.sqrt(geom.kv_lora + geom.d_s)"),
    "shared-key query part dropped": ("decode_absorbed", "q[i, :, geom.d_c:]], axis=-1)", "0 * q[i, :, geom.d_c:]], axis=-1)"),
    "softmax normalised over heads": ("decode_absorbed", "p /= p.sum(axis=0, keepdims=True)", "p /= p.sum(axis=1, keepdims=True)"),
    "K^C columns used as W_UV": ("decode_absorbed", "W_UV = W[:, :, geom.d_c:]", "W_UV = W[:, :, :geom.d_v]"),
    "gate without sigmoid": ("decode_absorbed", "O = O * _sigmoid(_f64(g)", "O = O * (_f64(g)"),
    "W_UK transposed per head": ("decode_absorbed", 'np.einsum("lhc,hc->hl", W_UK', 'np.einsum("lhc,hc->hl", W_UK[::-1]'),
}


def test_decode_pins_pass_on_the_oracle():
    assert failing_pins(DEC_PINS, oracle.decode_absorbed) == []


@pytest.mark.parametrize("what", sorted(DEC_MUTANTS))
def test_decode_mutant_is_caught(what):
    impl = mutant(*DEC_MUTANTS[what])
    assert failing_pins(DEC_PINS, impl), what


# ---------------------------------------------------------------------------
# QK-Clip
# ---------------------------------------------------------------------------
def pin_clip_rechecks_to_tau(impl):
    """On the tiny layer: clipped heads' recomputed max logit is tau, every
    logit of a clipped head scales by gamma, other heads and all V columns keep their bits."""
    L = synth.tiny_layer(0)
    geom, tau = L["geom"], L["tau"]

    def logits(WQ, WKV):
        up = oracle.up_proj(L["x"], L["W_DQ"], L["w_q"], WQ, L["W_DKV"], L["w_kv"], WKV, geom, "f64")
        _, ml = oracle.attention(up["Q"], up["KC"], up["kS"], up["V"], None)
        return ml, up

    ml, up = logits(L["W_UQ"], L["W_UKV"])
    WQ, WKV, clipped, gamma = impl(L["W_UQ"], L["W_UKV"], ml.astype(np.float32), tau, geom, "f32")
    assert clipped.tolist() == [int(m > tau) for m in ml.astype(np.float32)]
    ml2, up2 = logits(WQ, WKV)
    for h in range(geom.H):
        q0, k0 = h * geom.d_qk, h * (geom.d_c + geom.d_v)
        if clipped[h]:
            assert ml2[h] == pytest.approx(tau, rel=1e-6)
            S = np.einsum("btd,bsd->bts", up["Q"][:, :, h], np.concatenate([up["KC"][:, :, h], up["kS"]], -1))
            S2 = np.einsum("btd,bsd->bts", up2["Q"][:, :, h], np.concatenate([up2["KC"][:, :, h], up2["kS"]], -1))
            assert np.allclose(S2, float(gamma[h]) * S, rtol=1e-5, atol=1e-5 * np.abs(S).max())
        else:
            assert np.array_equal(WQ[:, q0:q0 + geom.d_qk], L["W_UQ"][:, q0:q0 + geom.d_qk])
            assert np.array_equal(WKV[:, k0:k0 + geom.d_c], L["W_UKV"][:, k0:k0 + geom.d_c])
        assert np.array_equal(WKV[:, k0 + geom.d_c:k0 + geom.d_c + geom.d_v],
                              L["W_UKV"][:, k0 + geom.d_c:k0 + geom.d_c + geom.d_v])


def pin_clip_threshold_is_strict(impl):
    geom = synth.Geom(H=4, d_model=8, q_lora=4, kv_lora=4, d_c=2, d_s=1, d_v=2)
    rng = np.random.default_rng(25)
    WQ = rng.standard_normal((4, 4 * 3)).astype(np.float32)
    WKV = rng.standard_normal((4, 4 * 4)).astype(np.float32)
    ml = np.array([10.0, 10.000001, -50.0, -np.inf], np.float32)
    _, _, clipped, gamma = impl(WQ, WKV, ml, 10.0, geom, "f32")
    assert clipped.tolist() == [0, 1, 0, 0]
    assert gamma[1] == np.float32(10.0) / np.float32(10.000001)


CLIP_PINS = [pin_clip_rechecks_to_tau, pin_clip_threshold_is_strict]
CLIP_MUTANTS = {
    "threshold not strict": ("qkclip", "if not (ml[h] > tau32)", "if not (ml[h] >= tau32)"),
    "q^C scaled by gamma": ("qkclip", "WQ[:, q0:q0 + geom.d_c] = scaled(WQ[:, q0:q0 + geom.d_c], root)",
                            "WQ[:, q0:q0 + geom.d_c] = scaled(WQ[:, q0:q0 + geom.d_c], gam)"),
    "q^S scaled by sqrt(gamma)": ("qkclip", "scaled(WQ[:, q0 + geom.d_c:q0 + geom.d_qk], gam)",
                                  "scaled(WQ[:, q0 + geom.d_c:q0 + geom.d_qk], root)"),
    "K^C left unscaled": ("qkclip", "WKV[:, k0:k0 + geom.d_c] = scaled(WKV[:, k0:k0 + geom.d_c], root)",
                          "WKV[:, k0:k0 + geom.d_c] = WKV[:, k0:k0 + geom.d_c]"),
    "V block scaled instead of K^C": ("qkclip", "k0 = h * (geom.d_c + geom.d_v)", "k0 = h * (geom.d_c + geom.d_v) + geom.d_c"),
    "W_UQ head stride d_c": ("qkclip", "q0 = h * geom.d_qk", "q0 = h * geom.d_c"),
    "gamma inverted": ("qkclip", "gam = np.float32(tau32 / ml[h])", "gam = np.float32(ml[h] / tau32)"),
}


def test_clip_pins_pass_on_the_oracle():
    assert failing_pins(CLIP_PINS, oracle.qkclip) == []


@pytest.mark.parametrize("what", sorted(CLIP_MUTANTS))
def test_clip_mutant_is_caught(what):
    impl = mutant(*CLIP_MUTANTS[what])
    assert failing_pins(CLIP_PINS, impl), what


# ---------------------------------------------------------------------------
# up-projections and RMSNorm
# ---------------------------------------------------------------------------
def pin_rms_norm_vs_torch(impl):
    rng = np.random.default_rng(26)
    c = rng.standard_normal((5, 7, 64)) * 3
    w = rng.standard_normal(64)
    want = torch.nn.functional.rms_norm(torch.from_numpy(c), (64,), torch.from_numpy(w), eps=1e-6).numpy()
    assert np.allclose(impl(c, w, 1e-6), want, rtol=1e-13, atol=1e-13)


def pin_up_proj_identity_layout(impl):
    """Identity projections: every head's q^C, q^S, K^C, V, the un-normalised k^S and the cache row."""
    geom = synth.Geom(H=3, d_model=20, q_lora=3 * 6, kv_lora=3 * 9, d_c=4, d_s=2, d_v=5, rms_eps=0.0)
    rng = np.random.default_rng(27)
    x = rng.standard_normal((2, 3, geom.d_model))
    W_DQ = np.zeros((geom.d_model, geom.q_lora))
    W_DQ[:geom.q_lora, :] = np.eye(geom.q_lora)
    W_DKV = np.zeros((geom.d_model, geom.kv_lora + geom.d_s))
    for j in range(geom.kv_lora + geom.d_s):
        W_DKV[j % geom.d_model, j] = 1.0
    up = impl(x, W_DQ, np.ones(geom.q_lora), np.eye(geom.q_lora), W_DKV, np.ones(geom.kv_lora),
              np.eye(geom.kv_lora), geom, "f64")
    cq = x[..., :geom.q_lora]
    cq_hat = cq / np.sqrt(np.mean(cq * cq, -1, keepdims=True))
    ckv_ks = x[..., [j % geom.d_model for j in range(geom.kv_lora + geom.d_s)]]
    ckv = ckv_ks[..., :geom.kv_lora]
    ckv_hat = ckv / np.sqrt(np.mean(ckv * ckv, -1, keepdims=True))
    for h in range(geom.H):
        assert np.allclose(up["Q"][:, :, h, :], cq_hat[..., h * 6:(h + 1) * 6], rtol=1e-14)
        assert np.allclose(up["KC"][:, :, h, :], ckv_hat[..., h * 9:h * 9 + 4], rtol=1e-14)
        assert np.allclose(up["V"][:, :, h, :], ckv_hat[..., h * 9 + 4:(h + 1) * 9], rtol=1e-14)
    assert np.array_equal(up["kS"], ckv_ks[..., geom.kv_lora:])
    assert np.allclose(up["cache"], np.concatenate([ckv_hat, ckv_ks[..., geom.kv_lora:]], -1), rtol=1e-14)


NORM_MUTANTS = {
    "mean of |c| instead of c^2": ("rms_norm", "np.mean(c * c, axis=-1, keepdims=True)",
                                   "np.mean(np.abs(c), axis=-1, keepdims=True)"),
    "weight not applied": ("rms_norm", "return c / np.sqrt(ms + eps) * _f64(w)", "return c / np.sqrt(ms + eps)"),
    "sum instead of mean": ("rms_norm", "np.mean(c * c, axis=-1, keepdims=True)", "np.sum(c * c, axis=-1, keepdims=True)"),
}
UP_MUTANTS = {
    "query from the un-normalised latent": ("up_proj", "q = _store(c_Q_hat @ _f64(W_UQ)", "q = _store(c_Q @ _f64(W_UQ)"),
    "k^S normalised with the latent": ("up_proj", "k_S = ckv_ks[..., geom.kv_lora:]",
                                       "k_S = rms_norm(ckv_ks, 1.0, geom.rms_eps)[..., geom.kv_lora:]"),
    "K^C and V swapped per head": ("up_proj", "KC=kv[..., :geom.d_c].copy()", "KC=kv[..., geom.d_v:].copy()"),
    "cache keeps the un-normalised latent": ("up_proj", "cache=np.concatenate([c_KV_hat, k_S], axis=-1)",
                                             "cache=np.concatenate([c_KV, k_S], axis=-1)"),
}


def test_norm_and_up_proj_pins_pass_on_the_oracle():
    assert failing_pins([pin_rms_norm_vs_torch], oracle.rms_norm) == []
    assert failing_pins([pin_up_proj_identity_layout], oracle.up_proj) == []


@pytest.mark.parametrize("what", sorted(NORM_MUTANTS))
def test_rms_norm_mutant_is_caught(what):
    assert failing_pins([pin_rms_norm_vs_torch], mutant(*NORM_MUTANTS[what])), what


@pytest.mark.parametrize("what", sorted(UP_MUTANTS))
def test_up_proj_mutant_is_caught(what):
    assert failing_pins([pin_up_proj_identity_layout], mutant(*UP_MUTANTS[what])), what


# ---------------------------------------------------------------------------
# row sampler, max-logit-only pass, log-sum-exp, materialised decode
# ---------------------------------------------------------------------------
def _sdpa_rows(Q, KC, kS, V, g, rows):
    out = []
    d_v = V.shape[-1]
    for (b, t, h) in rows:
        K = torch.cat([torch.from_numpy(KC[b, :t + 1, h]), torch.from_numpy(kS[b, :t + 1])], -1)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[b, t, h])[None, None, None], K[None, None], torch.from_numpy(V[b, :t + 1, h])[None, None])
        out.append(o[0, 0, 0].numpy() / (1 + np.exp(-g[b, t, h * d_v:(h + 1) * d_v])))
    return np.stack(out)


def pin_rows_vs_sdpa(impl):
    Q, KC, kS, V, g = _attn_case()
    rows = [(0, 0, 0), (1, 6, 1), (0, 3, 1), (1, 5, 0)]
    got, _ = impl(Q, KC, kS, V, g, rows)
    assert np.allclose(got, _sdpa_rows(Q, KC, kS, V, g, rows), rtol=1e-10, atol=1e-12)


def pin_head_maxlogit_brute_force(impl):
    Q, KC, kS, V, g = _attn_case()
    got = impl(Q, KC, kS, heads=[0, 1])
    pin_maxlogit_brute_force(lambda *a: (None, np.array([got[0], got[1]])))


def pin_lse_vs_scipy(impl):
    sp = pytest.importorskip("scipy.special")
    Q, KC, kS, V, g = _attn_case()
    lse = impl(Q, KC, kS)
    B, T, H, d_qk = Q.shape
    for b in range(B):
        for h in range(H):
            S = Q[b, :, h] @ np.concatenate([KC[b, :, h], kS[b]], -1).T / math.sqrt(d_qk)
            for t in range(T):
                assert lse[b, t, h] == pytest.approx(sp.logsumexp(S[t, :t + 1]), rel=1e-12)


def pin_materialised_vs_sdpa(impl):
    q, W, cache, offs, _ = _dec_case((9,), seed=28)
    m = impl(q, W, cache, offs, G)
    C, Wt = torch.from_numpy(cache), torch.from_numpy(W)
    for h in range(G.H):
        c0 = h * (G.d_c + G.d_v)
        K = torch.cat([C[:, :G.kv_lora] @ Wt[:, c0:c0 + G.d_c], C[:, G.kv_lora:]], -1)
        Vh = C[:, :G.kv_lora] @ Wt[:, c0 + G.d_c:c0 + G.d_c + G.d_v]
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, h])[None, None, None], K[None, None], Vh[None, None], scale=1.0 / math.sqrt(G.d_qk))
        assert np.allclose(m[0, h], o[0, 0, 0].numpy(), rtol=1e-12, atol=1e-14)


MISC = {
    "row sample reads one key past the row": (pin_rows_vs_sdpa, (
        "attention_rows", ("_f64(KC[b, :t + 1, h, :])", "_f64(kS[b, :t + 1])", "_f64(V[b, :t + 1, h, :])"),
        ("_f64(KC[b, :t + 2, h, :])", "_f64(kS[b, :t + 2])", "_f64(V[b, :t + 2, h, :])"))),
    "row sample queries from the previous position": (pin_rows_vs_sdpa, ("attention_rows", "q = _f64(Q[b, t, h, :])",
                                                                         "q = _f64(Q[b, max(t - 1, 0), h, :])")),
    "row sample gate of head 0": (pin_rows_vs_sdpa, ("attention_rows", "g[b, t, h * d_v:(h + 1) * d_v]", "g[b, t, :d_v]")),
    "max-logit pass anti-causal": (pin_head_maxlogit_brute_force, ("head_maxlogit", "<= np.arange(t0, t1)[:, None]",
                                                                   ">= np.arange(t0, t1)[:, None]")),
    "max-logit pass unscaled": (pin_head_maxlogit_brute_force, ("head_maxlogit", "scale = 1.0 / math.sqrt(d_qk)", "scale = 1.0")),
    "lse without the max": (pin_lse_vs_scipy, ("attention_lse", "(m + np.log(", "(0 * m + np.log(")),
    "lse anti-causal": (pin_lse_vs_scipy, ("attention_lse", "causal = np.arange(T)[None, :] <= np.arange(T)[:, None]",
                                           "causal = np.arange(T)[None, :] >= np.arange(T)[:, None]")),
    "materialised 576-wide scale": (pin_materialised_vs_sdpa, ("decode_materialised", "scale = 1.0 / math.sqrt(geom.d_qk)",
                                                               "scale = 1.0 / math.sqrt(geom.kv_lora + geom.d_s)")),
    "materialised values from the K^C block": (pin_materialised_vs_sdpa, ("decode_materialised", "Vh = C[:, :geom.kv_lora] @ W_UV",
                                                                          "Vh = C[:, :geom.kv_lora] @ W_UK[:, :geom.d_v]")),
    "materialised keys without k^S": (pin_materialised_vs_sdpa, ("decode_materialised", "C[:, :geom.kv_lora] @ W_UK, C[:, geom.kv_lora:]",
                                                                 "C[:, :geom.kv_lora] @ W_UK, 0 * C[:, geom.kv_lora:]")),
}


def test_misc_pins_pass_on_the_oracle():
    assert failing_pins([pin_rows_vs_sdpa], oracle.attention_rows) == []
    assert failing_pins([pin_head_maxlogit_brute_force], oracle.head_maxlogit) == []
    assert failing_pins([pin_lse_vs_scipy], oracle.attention_lse) == []
    assert failing_pins([pin_materialised_vs_sdpa], oracle.decode_materialised) == []


@pytest.mark.parametrize("what", sorted(MISC))
def test_misc_mutant_is_caught(what):
    pin, spec = MISC[what]
    assert failing_pins([pin], mutant(*spec)), what


# ---------------------------------------------------------------------------
# whole layer: the output gate g = x W_g and the output projection Delta = o W_O
# ([OMA] "All 20 steps", output gate and output projection)
# ---------------------------------------------------------------------------
def _layer_case():
    L = synth.tiny_layer(0)
    return L, L["geom"]


def _ungated_sdpa(L, geom):
    """O~ (no gate) of the tiny layer from torch SDPA in float64 on the oracle's
    up-projection outputs (the up-projection has its own pins above)."""
    up = oracle.up_proj(L["x"], L["W_DQ"], L["w_q"], L["W_UQ"], L["W_DKV"], L["w_kv"], L["W_UKV"], geom, "f64")
    B, T = L["x"].shape[:2]
    out = np.empty((B, T, geom.H, geom.d_v))
    for h in range(geom.H):
        K = torch.cat([torch.from_numpy(up["KC"][:, :, h]), torch.from_numpy(up["kS"])], -1)
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(up["Q"][:, :, h])[:, None], K[:, None], torch.from_numpy(up["V"][:, :, h])[:, None],
            is_causal=True)[:, 0]
        out[:, :, h] = o.numpy()
    return out.reshape(B, T, -1)


def pin_layer_zero_gate_halves_the_output(impl):
    """W_g = 0 gives g = 0 and sigmoid(0) = 1/2 on every output column."""
    L, geom = _layer_case()
    L = dict(L, W_g=np.zeros_like(L["W_g"]))
    res = impl(L["x"], L, geom, "f64")
    assert np.allclose(res["o"], 0.5 * _ungated_sdpa(L, geom), rtol=1e-10, atol=1e-13)


def pin_layer_gate_columns_line_up(impl):
    """W_g[:, j] = c_j e_k: output column j is scaled by sigmoid(x_k c_j), c_j distinct per column."""
    L, geom = _layer_case()
    k = 5
    c = np.linspace(-3.0, 3.0, geom.H * geom.d_v)
    W_g = np.zeros_like(L["W_g"], dtype=np.float64)
    W_g[k, :] = c
    L = dict(L, W_g=W_g)
    res = impl(L["x"], L, geom, "f64")
    gate = torch.sigmoid(torch.from_numpy(L["x"][..., k:k + 1].astype(np.float64) * c)).numpy()
    assert np.allclose(res["o"], gate * _ungated_sdpa(L, geom), rtol=1e-10, atol=1e-13)


def pin_layer_output_projection_identity(impl):
    """W_O = [I | 0] copies o into the first H d_v columns of Delta and leaves the rest 0;
    a column permutation of it permutes Delta the same way."""
    L, geom = _layer_case()
    n = geom.H * geom.d_v
    W_O = np.zeros((n, geom.d_model))
    W_O[:, :n] = np.eye(n)
    perm = np.random.default_rng(29).permutation(geom.d_model)
    for W in (W_O, W_O[:, perm]):
        res = impl(L["x"], dict(L, W_O=W), geom, "f64")
        want = np.zeros(res["o"].shape[:2] + (geom.d_model,))
        want[..., :n] = res["o"]
        if W is not W_O:
            want = want[..., perm]
        assert np.array_equal(res["delta"], want)
        assert np.allclose(res["o"], _layer_case_gated_reference(L, geom), rtol=1e-10, atol=1e-13)


def _layer_case_gated_reference(L, geom):
    gate = torch.sigmoid(torch.from_numpy(L["x"].astype(np.float64) @ L["W_g"].astype(np.float64))).numpy()
    return gate * _ungated_sdpa(L, geom)


LAYER_PINS = [pin_layer_zero_gate_halves_the_output, pin_layer_gate_columns_line_up, pin_layer_output_projection_identity]
LAYER_MUTANTS = {
    "gate dropped": ("layer_forward", 'up["V"], g)', 'up["V"], None)'),
    "gate negated": ("layer_forward", 'up["V"], g)', 'up["V"], -g)'),
    "gate read from W_O": ("layer_forward", 'g = _store(_f64(x) @ _f64(W["W_g"]), dtype)',
                           'g = _store(_f64(x) @ _f64(W["W_O"]).T, dtype)'),
    "gate columns reversed": ("layer_forward", 'g = _store(_f64(x) @ _f64(W["W_g"]), dtype)',
                              'g = _store(_f64(x) @ _f64(W["W_g"])[:, ::-1], dtype)'),
    "output projection from W_g": ("layer_forward", 'delta = o @ _f64(W["W_O"])', 'delta = o @ _f64(W["W_g"]).T'),
    "output projection dropped": ("layer_forward", 'delta = o @ _f64(W["W_O"])', 'delta = _f64(x)'),
    "o flattened feature-major": ("layer_forward", "o = _store(O.reshape(B, T, -1), dtype)",
                                  "o = _store(O.transpose(0, 1, 3, 2).reshape(B, T, -1), dtype)"),
}


def test_layer_pins_pass_on_the_oracle():
    assert failing_pins(LAYER_PINS, oracle.layer_forward) == []


@pytest.mark.parametrize("what", sorted(LAYER_MUTANTS))
def test_layer_mutant_is_caught(what):
    assert failing_pins(LAYER_PINS, mutant(*LAYER_MUTANTS[what])), what
