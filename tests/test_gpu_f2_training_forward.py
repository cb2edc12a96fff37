"""Parity of mla_attn_fwd_train, the training form of the forward ("Gated MLA
et NoPE", "Un détail de précision numérique": the attention output stays in
float32 while training), with the oracle and with the bf16 form."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_F32, TOL_MAXLOGIT, check_status, dev, host, max_rel, rel_l2

pytestmark = pytest.mark.gpu


def _run_bf16(inp, geom, gate):
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


@pytest.mark.parametrize("B,T,H,gate", [(1, 300, 2, True), (2, 129, 3, False)])
def test_training_form_keeps_fp32_output(B, T, H, gate):
    """mla_attn_fwd_train: the same forward with o kept in float32 ("Gated MLA
    et NoPE", "Un détail de précision numérique").  Its output is the bf16
    form's before rounding: bf16(o_fp32) is bit-identical to mla_attn_fwd's o."""
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.Geom(H=H)
    inp = synth.attn_core(B, T, geom, seed=200 + T, hot_heads=1, hot_scale=3.0, gate=gate)
    Q, KC, kS, V = (dev(inp[k], "bf16") for k in ("Q", "KC", "kS", "V"))
    g = dev(inp["g"], "bf16") if gate else None
    O32 = torch.empty(B, T, H * geom.d_v, dtype=torch.float32, device="cuda")
    ml32 = torch.empty(H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O32, ml32)
    check_status()
    O16, ml16 = _run_bf16(inp, geom, gate)
    O_ref, ml_ref = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"] if gate else None)
    got = host(O32).reshape(B, T, H, geom.d_v)
    assert rel_l2(got, O_ref) <= TOL_BF16
    assert rel_l2(got, O_ref) <= rel_l2(O16, O_ref) * 1.05        # no worse than the rounded form
    assert np.array_equal(oracle.bf16_round(got), O16)
    assert np.array_equal(host(ml32), ml16)


def test_training_form_cuda_core_shapes():
    """Other head widths (bf16 in, fp32 out) run the CUDA-core kernel."""
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.TINY
    inp = synth.attn_core(1, 70, geom, seed=9, hot_heads=0, gate=True)
    Q, KC, kS, V, g = (dev(inp[k], "bf16") for k in ("Q", "KC", "kS", "V", "g"))
    O32 = torch.empty(1, 70, geom.H * geom.d_v, dtype=torch.float32, device="cuda")
    ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O32, ml)
    check_status()
    O_ref, ml_ref = oracle.attention(inp["Q"], inp["KC"], inp["kS"], inp["V"], inp["g"])
    assert rel_l2(host(O32).reshape(O_ref.shape), O_ref) <= TOL_F32    # fp32 arithmetic on bf16 inputs
    assert max_rel(host(ml), ml_ref) <= TOL_MAXLOGIT
