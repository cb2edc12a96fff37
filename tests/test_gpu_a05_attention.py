"""Parity of mla_attn_fwd (bf16, K3 head geometry -> tcgen05 kernel) with the oracle.

Small cases cover ragged and single-tile sequences against the full oracle.
The attention-core workload B=2, T=2048, H=96 is checked whole, head by head,
with every head's max logit; the long-context workload B=1, T=16384, H=96 is
checked on every head's max logit, on the whole output of 16 heads (heads
0-7 and 8 seeded others) and on sampled rows of every head."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_MAXLOGIT, check_status, dev, host, max_rel, per_head, rel_l2

pytestmark = pytest.mark.gpu


def _run(inp, geom, gate=True):
    import torch
    import gated_mla_qk_b200 as gm
    Q, KC, kS, V = (dev(inp[k], "bf16") for k in ("Q", "KC", "kS", "V"))
    g = dev(inp["g"], "bf16") if gate else None
    B, T = Q.shape[:2]
    O = torch.empty(B, T, geom.H * geom.d_v, dtype=torch.bfloat16, device="cuda")
    ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd(geom, Q, KC, kS, V, g, O, ml)
    check_status()
    return host(O).reshape(B, T, geom.H, geom.d_v), host(ml)


def _geom(H):
    return synth.Geom(H=H)


@pytest.mark.parametrize("B,T,H,hot,gate", [
    (1, 1, 2, 0, True),        # single position: o_0 = sigmoid(g_0) V_0
    (1, 128, 2, 1, True),      # exactly one tile
    (2, 129, 3, 1, True),      # one full tile + a 1-row ragged tile
    (1, 300, 2, 1, False),     # ragged, no gate
    (2, 640, 4, 2, True),      # several tiles, several kv tiles per query tile
    (1, 1000, 3, 3, True),
    (1, 300, 96, 8, True),     # every K3 head: the head-major grid and the max-logit atomics over 96 heads
])
def test_small_against_full_oracle(B, T, H, hot, gate):
    geom = _geom(H)
    inp = synth.attn_core(B, T, geom, seed=100 + T, hot_heads=hot, hot_scale=3.0, gate=gate)
    O, ml = _run(inp, geom, gate)
    O_ref, ml_ref = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"] if gate else None)
    assert rel_l2(O, O_ref) <= TOL_BF16
    assert max_rel(ml, ml_ref) <= TOL_MAXLOGIT


def test_first_row_is_gated_first_value():
    geom = _geom(2)
    inp = synth.attn_core(1, 256, geom, seed=7, hot_heads=0)
    O, _ = _run(inp, geom)
    V0 = inp["V"][:, 0]
    g0 = inp["g"][:, 0].reshape(1, geom.H, geom.d_v)
    want = V0 / (1 + np.exp(-g0))
    assert rel_l2(O[:, 0], want) <= 1e-2


def test_heavy_logits_dominate_softmax():
    """Hot heads (x4) give near one-hot softmax rows; lazy rescaling must stay exact."""
    geom = _geom(2)
    inp = synth.attn_core(1, 512, geom, seed=9, hot_heads=2, hot_scale=4.0)
    O, ml = _run(inp, geom)
    O_ref, ml_ref = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"])
    assert ml_ref.min() > 30
    assert rel_l2(O, O_ref) <= TOL_BF16
    assert max_rel(ml, ml_ref) <= TOL_MAXLOGIT


def test_repeated_calls_identical():
    geom = _geom(3)
    inp = synth.attn_core(1, 384, geom, seed=11, hot_heads=1)
    O1, ml1 = _run(inp, geom)
    O2, ml2 = _run(inp, geom)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(ml1, ml2)


@pytest.mark.slow
def test_core_T2048_every_head():
    """B=2, T=2048, H=96, heads 0-7 x3: the whole output, head by head, and the
    max logit of all 96 heads against the oracle."""
    inp = synth.attn_core_config("core_T2048")
    O, ml = _run(inp, synth.K3)
    def one(h):                                    # keep only head h of the oracle's [B,T,H,d_v] result
        O_ref, ml_ref = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], heads=[h])
        return O_ref[:, :, h].copy(), ml_ref[h]
    res = per_head(one, range(synth.K3.H))
    for h, (O_h, ml_h) in res.items():
        assert rel_l2(O[:, :, h], O_h) <= TOL_BF16, h
        assert max_rel(ml[[h]], [ml_h]) <= TOL_MAXLOGIT, h
    want = np.array([res[h][1] for h in range(synth.K3.H)])
    assert want[:8].min() > 2 * want[8:].max()     # the hot heads stand out


@pytest.mark.slow
def test_long_T16384_heads_rows_and_every_max_logit():
    """B=1, T=16384, H=96, heads 0-7 x4: the max logit of all 96 heads; the
    whole output of heads 0-7 and of 8 seeded random heads at full T; and
    sampled rows of every head."""
    inp = synth.attn_core_config("long_T16384")
    O, ml = _run(inp, synth.K3)
    H = synth.K3.H
    ref = per_head(lambda h: oracle.head_maxlogit(inp["Q"], inp["KC"], inp["kS"], [h])[h], range(H))
    want = np.array([ref[h] for h in range(H)])
    assert max_rel(ml, want) <= TOL_MAXLOGIT
    assert want[:8].min() > 2 * want[8:].max()
    rng = np.random.default_rng(2)
    heads = list(range(8)) + sorted(int(h) for h in rng.choice(np.arange(8, H), 8, replace=False))
    full = per_head(lambda h: oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], heads=[h])[0][:, :, h].copy(),
                    heads, workers=4)
    for h in heads:
        assert rel_l2(O[:, :, h], full[h]) <= TOL_BF16, h
    rows = [(0, t, h) for h in range(H) for t in (0, 127, 128, 8191, 16383)]
    rows += [(0, int(t), int(h)) for t, h in zip(rng.integers(0, 16384, 96), rng.integers(0, H, 96))]
    want_rows, _ = oracle.attention_rows(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"], rows)
    got = np.stack([O[b, t, h] for (b, t, h) in rows])
    assert rel_l2(got, want_rows) <= TOL_BF16
