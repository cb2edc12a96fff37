"""The non-allocating decode entry point (mla_decode_absorbed_noalloc).

It exists for callers that cannot allocate device memory on their request
path (a serving loop that must not call cudaMalloc/cudaFree, a plugin whose
host owns all device memory).  The test calls it through the C ABI, twice in a
row with different inputs, and checks each result against the workspace-taking
entry point and against the oracle on the same inputs; at the size limit it
checks that 9 sequences of 8192 tokens (16,201,728 bytes of scratch) run and
match the oracle, and that 10 (18,001,920 bytes) are refused on the host.  This file sorts last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, rel_l2

pytestmark = pytest.mark.gpu


def _case(seed, lens):
    rng = np.random.default_rng(seed)
    d = synth.decode_batch(n_seq=len(lens), lo=1, hi=2, seed=seed, gate=True)
    lens = np.array(lens)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    d.update(lens=lens, seq_offsets=offs,
             cache=synth.round_storage(rng.standard_normal((int(offs[-1]), 576)).astype(np.float32), "bf16"))
    return d


def _noalloc_via_abi(lib, d, O):
    import torch
    import gated_mla_qk_b200 as gm
    geom = gm.CGeom.of(d["geom"])
    q = synth.to_torch(d["q"], "bf16", "cuda")
    W = synth.to_torch(d["W_UKV"], "bf16", "cuda")
    cache = synth.to_torch(d["cache"], "bf16", "cuda")
    g = synth.to_torch(d["g"], "bf16", "cuda")
    offs = torch.from_numpy(d["seq_offsets"]).cuda()
    st = lib.mla_decode_absorbed_noalloc(ctypes.byref(geom), gm.GMLA_BF16, len(d["lens"]), q.data_ptr(),
                                         W.data_ptr(), cache.data_ptr(), offs.data_ptr(), int(d["lens"].max()),
                                         g.data_ptr(), O.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, st
    assert gm.device_status() == 0
    return O.float().cpu().numpy()


def _with_workspace(d):
    import torch
    import gated_mla_qk_b200 as gm
    O = torch.empty(len(d["lens"]), 96, 128, dtype=torch.bfloat16, device="cuda")
    gm.mla_decode_absorbed(synth.K3, synth.to_torch(d["q"], "bf16", "cuda"), synth.to_torch(d["W_UKV"], "bf16", "cuda"),
                           synth.to_torch(d["cache"], "bf16", "cuda"), torch.from_numpy(d["seq_offsets"]).cuda(),
                           int(d["lens"].max()), synth.to_torch(d["g"], "bf16", "cuda"), O)
    assert gm.device_status() == 0
    return O.float().cpu().numpy()


def _oracle(d):
    return oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], synth.K3, d["g"])


def test_noalloc_decode_matches_workspace_decode_twice():
    import torch
    import gated_mla_qk_b200 as gm
    lib = gm.load_library()
    O = torch.empty(6, 96, 128, dtype=torch.bfloat16, device="cuda")
    for seed, lens in ((41, (1, 300, 1024, 2047, 3000, 17)), (42, (2500, 5, 129, 128, 999, 2048))):
        d = _case(seed, lens)
        got = _noalloc_via_abi(lib, d, O)
        assert rel_l2(got, _with_workspace(d)) <= TOL_BF16
        assert rel_l2(got, _oracle(d)) <= TOL_BF16


def _scratch_need(n, max_len, H=96, kv_lora=512, d_s=64):
    """The CUDA-core decode's scratch bytes, as include/gmla.h states them."""
    al = lambda x: (x + 255) // 256 * 256
    S = -(-max_len // 1024)
    return al(4 * n * H * (kv_lora + d_s)) + al(4 * n * H * S * 2) + 4 * n * H * S * kv_lora


def test_noalloc_decode_at_the_size_limit():
    """9 sequences of 8192 tokens need 16,201,728 bytes of the 16 MiB scratch:
    they run and match the oracle; 10 need 18,001,920 and are refused before
    anything is enqueued."""
    import torch
    import gated_mla_qk_b200 as gm
    lib = gm.load_library()
    geom = gm.CGeom.of(synth.K3)
    assert _scratch_need(9, 8192) == 16201728 <= (16 << 20) < _scratch_need(10, 8192) == 18001920
    p = torch.empty(16, dtype=torch.bfloat16, device="cuda").data_ptr()
    n0 = gm.launch_count()
    st = lib.mla_decode_absorbed_noalloc(ctypes.byref(geom), gm.GMLA_BF16, 10, p, p, p, p, 8192, None, p, None)
    assert st == -6          # GMLA_EWORKSPACE, nothing enqueued
    assert gm.launch_count() == n0
    d = _case(43, (8192,) * 9)
    O = torch.empty(9, 96, 128, dtype=torch.bfloat16, device="cuda")
    got = _noalloc_via_abi(lib, d, O)
    assert rel_l2(got, _oracle(d)) <= TOL_BF16
