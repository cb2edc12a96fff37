"""Parity of the bf16 tensor-core GEMM behind the projections (mla_gemm and
mla_up_proj) with a float64 matrix product of the same bf16 inputs."""
import numpy as np
import pytest

from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, check_status, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 64),        # one tile, one k-block
    (200, 576, 7168),      # ragged M, N = 2 tiles + 64 (the joint KV down-projection width)
    (1, 1536, 1536),       # a single row
    (300, 264, 520),       # ragged everything (N, K multiples of 8)
    (257, 520, 64),        # one row past a 256-row pair tile; the last 64-column store box holds 8 columns
    (512, 72, 128),        # N below one 256-column tile: a full box, an 8-column box, two boxes past N
    (1024, 2048, 512),
    (4096, 6144, 1536),    # 768 output tiles: every persistent CTA walks five or six, both TMEM accumulators cycle
])
def test_gemm_bf16_vs_float64(M, N, K):
    import torch
    import gated_mla_qk_b200 as gm
    rng = np.random.default_rng(M + N + K)
    A = synth.round_storage(rng.standard_normal((M, K)).astype(np.float32), "bf16")
    B = synth.round_storage((rng.standard_normal((K, N)) / np.sqrt(K)).astype(np.float32), "bf16")
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    gm.mla_gemm(synth.to_torch(A, "bf16", "cuda"), synth.to_torch(B, "bf16", "cuda"), C)
    check_status()
    want = A.astype(np.float64) @ B.astype(np.float64)
    assert rel_l2(host(C), want) <= TOL_BF16
    # bf16 output rounding dominates: every element within a few ulps of the exact product
    err = np.abs(host(C) - want)
    assert np.all(err <= 2.0 ** -7 * np.abs(want) + 1e-2 * np.sqrt(K / 512))


def test_gemm_fp32_path():
    import torch
    import gated_mla_qk_b200 as gm
    rng = np.random.default_rng(5)
    A = rng.standard_normal((70, 33)).astype(np.float32)
    B = rng.standard_normal((33, 45)).astype(np.float32)
    C = torch.empty(70, 45, device="cuda")
    gm.mla_gemm(torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda(), C)
    check_status()
    assert rel_l2(host(C), A.astype(np.float64) @ B) <= 1e-5
