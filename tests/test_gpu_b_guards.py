"""Every entry point writes exactly its outputs: each output (and each caller
workspace) sits inside one device buffer between guard regions, the whole
buffer is filled with 0xFF bytes first (a NaN in bf16 and fp32), and after the
call on ragged sizes (T not a multiple of any tile, odd decode lengths, ragged
GEMM shapes) the guards must still hold 0xFF and the outputs no NaN.
"""
import numpy as np
import pytest

from gated_mla_qk_b200 import synth
from gpu_util import Guarded, check_status, dev, guarded_bytes as _bytes

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,geom,B,T", [("bf16", synth.K3, 1, 129), ("bf16", synth.Geom(H=8), 2, 300),
                                            ("f32", synth.TINY, 1, 45)])
def test_up_proj_guards(dtype, geom, B, T):
    import torch
    import gated_mla_qk_b200 as gm
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    rng = np.random.default_rng(B * 1000 + T)
    W = {k: dev(synth.round_storage(v, dtype), dtype)
         for k, v in synth.layer_weights(geom, rng, with_gate_out=False).items()}
    x = dev(synth.round_storage(rng.standard_normal((B, T, geom.d_model)).astype(np.float32), dtype), dtype)
    out = dict(Q=Guarded((B, T, geom.H, geom.d_qk), td), KC=Guarded((B, T, geom.H, geom.d_c), td),
               kS=Guarded((B, T, geom.d_s), td), V=Guarded((B, T, geom.H, geom.d_v), td),
               cache=Guarded((B, T, geom.kv_lora + geom.d_s), td))
    ws = _bytes(gm.mla_up_proj_workspace(geom, gm.GMLA_F32 if dtype == "f32" else gm.GMLA_BF16, B, T))
    gm.mla_up_proj(geom, x, W["W_DQ"], W["w_q"], W["W_UQ"], W["W_DKV"], W["w_kv"], W["W_UKV"],
                   *(out[k].t for k in ("Q", "KC", "kS", "V", "cache")), workspace=ws.t)
    check_status()
    for k, v in out.items():
        v.check(k)
    ws.check("workspace", written=False)


@pytest.mark.parametrize("dtype,geom,B,T,gate", [("bf16", synth.K3, 1, 129, True), ("bf16", synth.Geom(H=3), 2, 300, False),
                                                 ("bf16", synth.Geom(H=2), 1, 1, True), ("f32", synth.TINY, 2, 45, True)])
def test_attention_forward_guards(dtype, geom, B, T, gate):
    import torch
    import gated_mla_qk_b200 as gm
    inp = synth.attn_core(B, T, geom, seed=500 + T, hot_heads=1, gate=gate, dtype=dtype)
    Q, KC, kS, V = (dev(inp[k], dtype) for k in ("Q", "KC", "kS", "V"))
    g = dev(inp["g"], dtype) if gate else None
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    O = Guarded((B, T, geom.H * geom.d_v), td)
    ml = Guarded((geom.H,), torch.float32)
    gm.mla_attn_fwd(geom, Q, KC, kS, V, g, O.t, ml.t)
    check_status()
    O.check("O")
    ml.check("maxlogit")
    # the training form: fp32 output and the row log-sum-exp
    O32 = Guarded((B, T, geom.H * geom.d_v), torch.float32)
    lse = Guarded((B, T, geom.H), torch.float32)
    ml2 = Guarded((geom.H,), torch.float32)
    gm.mla_attn_fwd_train(geom, Q, KC, kS, V, g, O32.t, ml2.t, lse=lse.t)
    check_status()
    O32.check("O (train)")
    lse.check("lse")
    ml2.check("maxlogit (train)")


@pytest.mark.parametrize("dtype,geom", [("bf16", synth.K3), ("f32", synth.TINY), ("bf16", synth.Geom(H=5))])
def test_qkclip_guards(dtype, geom):
    import torch
    import gated_mla_qk_b200 as gm
    rng = np.random.default_rng(geom.H)
    W = synth.layer_weights(geom, rng, with_gate_out=False)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    WQ = Guarded((geom.q_lora, geom.H * geom.d_qk), td, init=dev(synth.round_storage(W["W_UQ"], dtype), dtype))
    WKV = Guarded((geom.kv_lora, geom.H * (geom.d_c + geom.d_v)), td,
                  init=dev(synth.round_storage(W["W_UKV"], dtype), dtype))
    ml = torch.from_numpy(rng.uniform(50, 150, geom.H).astype(np.float32)).cuda()
    clipped = Guarded((geom.H,), torch.uint8)
    gamma = Guarded((geom.H,), torch.float32)
    gm.qkclip_rescale(geom, WQ.t, WKV.t, ml, 100.0, clipped.t, gamma.t)
    check_status()
    WQ.check("W_UQ")
    WKV.check("W_UKV")
    clipped.check("clipped")
    assert set(clipped.t.cpu().tolist()) <= {0, 1}
    gamma.check("gamma")


@pytest.mark.parametrize("lens,gate", [((1, 127, 1000, 129), True), ((5,), False), ((2048, 3, 4097), False),
                                       ((0, 127, 0, 1000, 0), True)])
def test_decode_guards(lens, gate):
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.K3
    d = synth.decode_batch(n_seq=len(lens), lo=1, hi=2, seed=70, gate=gate)
    rng = np.random.default_rng(71)
    lens = np.array(lens)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cache = synth.round_storage(rng.standard_normal((int(offs[-1]), 576)).astype(np.float32), "bf16")
    args = (dev(d["q"], "bf16"), dev(d["W_UKV"], "bf16"), dev(cache, "bf16"), torch.from_numpy(offs).cuda(),
            int(lens.max()), dev(d["g"], "bf16") if gate else None)
    O = Guarded((len(lens), geom.H, geom.d_v), torch.bfloat16)
    ws = _bytes(gm.mla_decode_workspace(geom, gm.GMLA_BF16, len(lens), int(lens.max())))
    gm.mla_decode_absorbed(geom, *args, O.t, workspace=ws.t)
    check_status()
    O.check("O")
    ws.check("workspace", written=False)
    O2 = Guarded((len(lens), geom.H, geom.d_v), torch.bfloat16)
    gm.mla_decode_absorbed_noalloc(geom, *args, O2.t)
    check_status()
    O2.check("O (fixed scratch)")


@pytest.mark.parametrize("M,N,K,dtype", [(300, 264, 520, "bf16"), (512, 72, 128, "bf16"), (1, 1536, 1536, "bf16"), (129, 8, 8, "bf16"),
                                         (70, 45, 33, "f32")])
def test_gemm_guards(M, N, K, dtype):
    import torch
    import gated_mla_qk_b200 as gm
    rng = np.random.default_rng(M * N + K)
    A = dev(synth.round_storage(rng.standard_normal((M, K)).astype(np.float32), dtype), dtype)
    Bm = dev(synth.round_storage(rng.standard_normal((K, N)).astype(np.float32), dtype), dtype)
    C = Guarded((M, N), torch.bfloat16 if dtype == "bf16" else torch.float32)
    gm.mla_gemm(A, Bm, C.t)
    check_status()
    C.check("C")
