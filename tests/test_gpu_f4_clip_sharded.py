"""QK-Clip under head (tensor) parallelism on K3-sized bf16 weights: each
rank's contiguous column shard clipped with its slice of the global max-logit
vector equals the full clip, bit for bit, and equals the oracle.  The ranks
run one after another on one GPU (the clip has no cross-rank exchange)."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import check_status, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 5])
def test_head_sharded_clip_matches_full_clip(world):
    import torch
    from gated_mla_qk_b200.dist import head_range, qkclip_rescale_heads
    geom = synth.K3
    W = synth.layer_weights(geom, np.random.default_rng(40 + world), with_gate_out=False)
    WQ0, WKV0 = synth.round_storage(W["W_UQ"], "bf16"), synth.round_storage(W["W_UKV"], "bf16")
    ml = np.random.default_rng(50 + world).uniform(20.0, 200.0, geom.H).astype(np.float32)
    ml[::7] = 100.0                                     # equality never clips
    tau = 100.0
    WQ_ref, WKV_ref, clip_ref, gamma_ref = oracle.qkclip(WQ0, WKV0, ml, tau, geom, "bf16")
    ml_d = torch.from_numpy(ml).cuda()
    w = geom.d_c + geom.d_v
    outs_q, outs_kv, clipped, gammas = [], [], [], []
    for r in range(world):
        h0, h1 = head_range(geom.H, world, r)
        q = synth.to_torch(np.ascontiguousarray(WQ0[:, h0 * geom.d_qk:h1 * geom.d_qk]), "bf16", "cuda")
        kv = synth.to_torch(np.ascontiguousarray(WKV0[:, h0 * w:h1 * w]), "bf16", "cuda")
        c = torch.empty(h1 - h0, dtype=torch.uint8, device="cuda")
        g = torch.empty(h1 - h0, dtype=torch.float32, device="cuda")
        qkclip_rescale_heads(geom, q, kv, ml_d, tau, h0, c, g)
        outs_q.append(host(q)); outs_kv.append(host(kv)); clipped.append(host(c)); gammas.append(host(g))
    check_status()
    WQ = np.concatenate(outs_q, axis=1)
    WKV = np.concatenate(outs_kv, axis=1)
    np.testing.assert_array_equal(np.concatenate(clipped), clip_ref)
    np.testing.assert_array_equal(np.concatenate(gammas).view(np.uint32), gamma_ref.view(np.uint32))
    np.testing.assert_array_equal(WQ.view(np.uint32), WQ_ref.view(np.uint32))
    np.testing.assert_array_equal(WKV.view(np.uint32), WKV_ref.view(np.uint32))
