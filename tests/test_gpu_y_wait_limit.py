"""Failure detection without a fault: every device-side wait of the kernels is
bounded in wall time, and a wait that runs out must come back to the host as
GMLA_ETIMEOUT with the context still usable.

The self-test kernel (gmla_selftest_wait) holds tensor memory and waits,
through the same bounded wait as the pipeline kernels, on an mbarrier that
nothing ever arrives at.  The tests check that
  * the wait gives up once the limit has passed (a short limit set with
    gmla_set_wait_limit_ns, and the 2 s default), and gmla_device_status
    reports GMLA_ETIMEOUT once and then clears it;
  * kernels launched while the error is pending return at once: an attention
    forward behind the self-test leaves its output untouched;
  * nothing is left behind: after the error is read, the same forward, a
    full-grid GEMM and the decode (tensor-memory kernels; the persistent ones
    put one CTA on every SM, which could not allocate tensor memory a CTA
    had failed to free) give results bit-identical to runs made before.
This file sorts after the other GPU parity tests, so a failure here cannot
hide them.
"""
import numpy as np
import pytest

from gated_mla_qk_b200 import synth
from gpu_util import dev, host

pytestmark = pytest.mark.gpu

GMLA_ETIMEOUT = -5


def _selftest(gm, limit_ns):
    import torch
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    gm.set_wait_limit_ns(limit_ns)
    try:
        gm.selftest_wait(elapsed)
        torch.cuda.synchronize()
    finally:
        gm.set_wait_limit_ns(0)
    ns, gave_up = (int(v) for v in elapsed.cpu())
    return ns, gave_up


@pytest.mark.parametrize("limit_ns", [1_000_000, 0])      # 1 ms, and the 2 s default
def test_wait_on_a_barrier_nothing_arrives_at_gives_up(limit_ns):
    import gated_mla_qk_b200 as gm
    assert gm.device_status() == 0
    ns, gave_up = _selftest(gm, limit_ns)
    limit = limit_ns or 2_000_000_000
    print(f"wait limit {limit} ns: gave up after {ns} ns")
    assert gave_up == 1
    assert limit <= ns < limit + 5_000_000_000
    assert gm.device_status() == GMLA_ETIMEOUT
    assert gm.device_status() == 0                 # read once, then cleared


def test_kernels_behind_a_timeout_return_at_once_and_the_library_recovers():
    import torch
    import gated_mla_qk_b200 as gm
    geom = synth.K3
    inp = synth.attn_core(1, 8192, geom, seed=90, hot_heads=8, hot_scale=3.0)
    d = {k: dev(v, "bf16") for k, v in inp.items()}
    bf = dict(dtype=torch.bfloat16, device="cuda")
    O = torch.empty(1, 8192, geom.H * geom.d_v, **bf)
    ml = torch.empty(geom.H, dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(91)
    A = synth.to_torch(synth.round_storage(rng.standard_normal((4096, 1536)).astype(np.float32), "bf16"), "bf16", "cuda")
    B = synth.to_torch(synth.round_storage(rng.standard_normal((1536, 6144)).astype(np.float32) / 40, "bf16"), "bf16", "cuda")
    C = torch.empty(4096, 6144, **bf)
    db = synth.decode_batch(n_seq=16, lo=500, hi=3000, seed=92)
    Od = torch.empty(16, geom.H, geom.d_v, **bf)

    def forward():
        gm.mla_attn_fwd(geom, d["Q"], d["KC"], d["kS"], d["V"], d["g"], O, ml)

    def others():
        gm.mla_gemm(A, B, C)
        gm.mla_decode_absorbed(geom, dev(db["q"], "bf16"), dev(db["W_UKV"], "bf16"), dev(db["cache"], "bf16"),
                               torch.from_numpy(db["seq_offsets"]).cuda(), int(db["lens"].max()), None, Od)

    assert gm.device_status() == 0
    forward()
    others()
    assert gm.device_status() == 0
    O_ref, ml_ref, C_ref, Od_ref = host(O), host(ml), host(C), host(Od)

    # the self-test times out and leaves the error pending; the forward behind it returns at once
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    gm.set_wait_limit_ns(1_000_000)
    try:
        gm.selftest_wait(elapsed)
    finally:
        gm.set_wait_limit_ns(0)
    O.fill_(float("nan"))
    forward()
    assert gm.device_status() == GMLA_ETIMEOUT
    assert int(elapsed[1]) == 1
    assert bool(torch.isnan(O).all())              # no CTA of the forward wrote anything

    for _ in range(2):
        for t in (O, C, Od):
            t.fill_(float("nan"))
        forward()
        others()
        assert gm.device_status() == 0
        np.testing.assert_array_equal(host(O), O_ref)
        np.testing.assert_array_equal(host(ml), ml_ref)
        np.testing.assert_array_equal(host(C), C_ref)
        np.testing.assert_array_equal(host(Od), Od_ref)
