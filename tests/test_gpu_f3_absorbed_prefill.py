"""Parity of mla_attn_fwd_absorbed (the forward computed on the latent cache:
"Kimi Qkclip" section 3's inference form applied to a prefill) with the
oracle's attention over keys and values materialised from the same cache, and
with mla_attn_fwd on the up-projection's outputs."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, check_status, dev, host, rel_l2

pytestmark = pytest.mark.gpu


def _inputs(B, T, seed, gate):
    """Q, the latent cache and W_UKV (bf16), and the keys / values they imply in float64."""
    geom = synth.K3
    rng = np.random.default_rng(seed)
    Q = synth.round_storage(rng.standard_normal((B, T, geom.H, geom.d_qk)).astype(np.float32), "bf16")
    Q[:, :, :4] *= 3.0                                     # a few heads with larger logits
    Q = synth.round_storage(Q, "bf16")
    cache = synth.round_storage(rng.standard_normal((B, T, geom.kv_lora + geom.d_s)).astype(np.float32), "bf16")
    W = synth.round_storage((rng.standard_normal((geom.kv_lora, geom.H * (geom.d_c + geom.d_v))) /
                             np.sqrt(geom.kv_lora)).astype(np.float32), "bf16")
    g = synth.round_storage(rng.standard_normal((B, T, geom.H * geom.d_v)).astype(np.float32), "bf16") if gate else None
    Wr = W.astype(np.float64).reshape(geom.kv_lora, geom.H, geom.d_c + geom.d_v)
    lat = cache[..., :geom.kv_lora].astype(np.float64)
    KC = np.einsum("btl,lhc->bthc", lat, Wr[:, :, :geom.d_c])
    V = np.einsum("btl,lhc->bthc", lat, Wr[:, :, geom.d_c:])
    kS = cache[..., geom.kv_lora:].astype(np.float64)
    return geom, Q, cache, W, g, KC, kS, V


def _q_abs_bound(Q, W, cache, geom):
    """Per head, how far the bf16 rounding of the absorbed query can move a logit.

    q~ = [q^C W_UK^T | q^S] enters the tensor core rounded to bf16 (relative
    error at most 2^-8 per element), so a logit q~ . c / sqrt(d_qk) moves by
    at most 2^-8 sum_k |q~_k c_k| / sqrt(d_qk) <= 2^-8 |q~|_2 |c|_2 / sqrt(d_qk)
    (Cauchy-Schwarz), and so does the max logit."""
    Wr = np.asarray(W, np.float64).reshape(geom.kv_lora, geom.H, geom.d_c + geom.d_v)
    Q = np.asarray(Q, np.float64)
    q_abs = np.concatenate([np.einsum("bthc,lhc->bthl", Q[..., :geom.d_c], Wr[:, :, :geom.d_c]), Q[..., geom.d_c:]],
                           axis=-1)
    c = np.asarray(cache, np.float64).reshape(-1, geom.kv_lora + geom.d_s)
    return 2.0 ** -8 * np.linalg.norm(q_abs, axis=-1).max(axis=(0, 1)) * np.linalg.norm(c, axis=-1).max() / \
        np.sqrt(geom.d_qk)


def _run_absorbed(geom, Q, cache, W, g):
    import torch
    import gated_mla_qk_b200 as gm
    B, T = Q.shape[:2]
    O = torch.full((B, T, geom.H * geom.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd_absorbed(geom, dev(Q, "bf16"), dev(W, "bf16"), dev(cache, "bf16"), dev(g, "bf16"), O, ml)
    check_status()
    return host(O).reshape(B, T, geom.H, geom.d_v), host(ml)


@pytest.mark.parametrize("B,T,gate", [(1, 1, True), (1, 96, False), (2, 129, True), (1, 300, True), (1, 1000, False)])
def test_absorbed_prefill_vs_materialised_oracle(B, T, gate):
    geom, Q, cache, W, g, KC, kS, V = _inputs(B, T, seed=900 + T, gate=gate)
    O, ml = _run_absorbed(geom, Q, cache, W, g)
    O_ref, ml_ref = oracle.attention(Q, KC, kS, V, g)
    assert np.isfinite(O).all()
    assert rel_l2(O, O_ref) <= TOL_BF16
    for h in range(geom.H):                            # no head may hide in the whole-tensor norm
        assert rel_l2(O[:, :, h], O_ref[:, :, h]) <= TOL_BF16, h
    assert np.all(np.abs(ml - ml_ref) <= _q_abs_bound(Q, W, cache, geom))


def test_absorbed_prefill_agrees_with_the_materialised_forward():
    """Same layer, both forms on the GPU: mla_up_proj -> mla_attn_fwd against
    mla_up_proj's latent cache -> mla_attn_fwd_absorbed."""
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.K3
    B, T = 1, 700
    rng = np.random.default_rng(910)
    W = synth.layer_weights(geom, rng, with_gate_out=False)
    x = synth.round_storage(rng.standard_normal((B, T, geom.d_model)).astype(np.float32), "bf16")
    bf = torch.bfloat16
    Wd = {k: dev(synth.round_storage(v, "bf16"), "bf16") for k, v in W.items()}
    Qd = torch.empty(B, T, geom.H, geom.d_qk, dtype=bf, device="cuda")
    KC = torch.empty(B, T, geom.H, geom.d_c, dtype=bf, device="cuda")
    kS = torch.empty(B, T, geom.d_s, dtype=bf, device="cuda")
    V = torch.empty(B, T, geom.H, geom.d_v, dtype=bf, device="cuda")
    cache = torch.empty(B, T, geom.kv_lora + geom.d_s, dtype=bf, device="cuda")
    gm.mla_up_proj(geom, dev(x, "bf16"), Wd["W_DQ"], Wd["w_q"], Wd["W_UQ"], Wd["W_DKV"], Wd["w_kv"], Wd["W_UKV"],
                   Qd, KC, kS, V, cache)
    g = dev(synth.round_storage(rng.standard_normal((B, T, geom.H * geom.d_v)).astype(np.float32), "bf16"), "bf16")
    O1 = torch.empty(B, T, geom.H * geom.d_v, dtype=bf, device="cuda")
    ml1 = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd(geom, Qd, KC, kS, V, g, O1, ml1)
    O2 = torch.empty(B, T, geom.H * geom.d_v, dtype=bf, device="cuda")
    ml2 = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd_absorbed(geom, Qd, Wd["W_UKV"], cache, g, O2, ml2)
    check_status()
    # K^C and V are rounded to bf16 in one form, q~ in the other: both within the bf16 bar of each other
    assert rel_l2(host(O2), host(O1)) <= 2 * TOL_BF16
    # one form rounds K^C to bf16, the other q~: each max logit within twice the bound of one such rounding
    assert np.all(np.abs(host(ml2) - host(ml1)) <= 2 * _q_abs_bound(host(Qd), host(Wd["W_UKV"]), host(cache), geom))


@pytest.mark.parametrize("B,T,gate", [(1, 129, True), (2, 45, False)])
def test_absorbed_prefill_writes_exactly_its_outputs(B, T, gate):
    import torch
    import gated_mla_qk_b200 as gm
    from gpu_util import Guarded, guarded_bytes
    geom, Q, cache, W, g, *_ = _inputs(B, T, seed=920 + T, gate=gate)
    O = Guarded((B, T, geom.H * geom.d_v), torch.bfloat16)
    ml = Guarded((geom.H,), torch.float32)
    ws = guarded_bytes(gm.mla_attn_fwd_absorbed_workspace(geom, B, T))
    gm.mla_attn_fwd_absorbed(geom, dev(Q, "bf16"), dev(W, "bf16"), dev(cache, "bf16"), dev(g, "bf16"), O.t, ml.t,
                             workspace=ws.t)
    check_status()
    O.check("O")
    ml.check("maxlogit")
    ws.check("workspace", written=False)
