"""Parity of mla_decode_absorbed with the oracle (absorbed form; the oracle's
absorbed form is itself pinned to the materialised-key form)."""
import numpy as np
import pytest

import oracle
from gated_mla_qk_b200 import synth
from gpu_util import TOL_BF16, TOL_F32, check_status, dev, host, rel_l2

pytestmark = pytest.mark.gpu


def _run(d, dtype):
    import torch
    import gated_mla_qk_b200 as gm
    geom = d["geom"]
    n = len(d["lens"])
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    O = torch.empty(n, geom.H, geom.d_v, dtype=td, device="cuda")
    offs = torch.from_numpy(d["seq_offsets"]).cuda()
    gm.mla_decode_absorbed(geom, dev(d["q"], dtype), dev(d["W_UKV"], dtype), dev(d["cache"], dtype), offs,
                           max(1, int(d["lens"].max())), dev(d["g"], dtype), O)
    check_status()
    return host(O)


@pytest.mark.parametrize("lens,gate", [((1, 2, 3), False), ((1, 127, 128, 129, 1000), True), ((4096, 33), False)])
def test_small_bf16(lens, gate):
    d = synth.decode_batch(n_seq=len(lens), lo=1, hi=2, seed=31, gate=gate)
    # replace the drawn lengths with the listed ones (and redraw the cache to match)
    rng = np.random.default_rng(32)
    lens = np.array(lens)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    d.update(lens=lens, seq_offsets=offs,
             cache=synth.round_storage(rng.standard_normal((int(offs[-1]), 576)).astype(np.float32), "bf16"))
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    assert rel_l2(got, want) <= TOL_BF16


def test_small_fp32_tiny_geometry():
    geom = synth.TINY
    rng = np.random.default_rng(33)
    lens = np.array([1, 5, 64, 300])
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    d = dict(geom=geom, lens=lens, seq_offsets=offs,
             cache=rng.standard_normal((int(offs[-1]), geom.kv_lora + geom.d_s)).astype(np.float32),
             q=rng.standard_normal((4, geom.H, geom.d_qk)).astype(np.float32),
             W_UKV=(rng.standard_normal((geom.kv_lora, geom.H * (geom.d_c + geom.d_v))) / 8).astype(np.float32),
             g=rng.standard_normal((4, geom.H * geom.d_v)).astype(np.float32))
    got = _run(d, "f32")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], geom, d["g"])
    assert rel_l2(got, want) <= TOL_F32


@pytest.mark.slow
def test_decode_64_sequences_1k_to_8k():
    """64 sequences, lengths U[1024, 8192], 96 heads, bf16 (the decode workload)."""
    d = synth.decode_batch()
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    assert rel_l2(got, want) <= TOL_BF16


def _with_lengths(lens, seed, ramp=0.0, gate=False):
    """decode_batch's q / W_UKV with the listed lengths and a fresh cache; with
    ramp > 0 the cache rows of each sequence grow in magnitude along the
    sequence, so the running max of every head moves often."""
    d = synth.decode_batch(n_seq=len(lens), lo=1, hi=2, seed=seed, gate=gate)
    rng = np.random.default_rng(seed + 1)
    lens = np.array(lens)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cache = rng.standard_normal((int(offs[-1]), 576)).astype(np.float32)
    if ramp:
        for i in range(len(lens)):
            a, b = offs[i], offs[i + 1]
            cache[a:b] *= (1.0 + ramp * np.arange(b - a) / max(1, b - a - 1))[:, None]
    d.update(lens=lens, seq_offsets=offs, cache=synth.round_storage(cache, "bf16"))
    return d


def test_running_max_moves_often():
    """Logits that grow along each sequence (by far more than the 2^8 rescale
    threshold) exercise the rescale of the accumulated latent sums."""
    d = _with_lengths((3000, 700, 64, 65), seed=41, ramp=6.0)
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    assert rel_l2(got, want) <= TOL_BF16


def test_many_short_sequences():
    """160 sequences of 1-200 tokens: work ranges start and end inside
    sequences and most ranges hold several sequences."""
    lens = np.random.default_rng(43).integers(1, 201, size=160)
    d = _with_lengths(tuple(int(x) for x in lens), seed=44, gate=True)
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    assert rel_l2(got, want) <= TOL_BF16


@pytest.mark.parametrize("lens,gate", [((0, 5, 0, 0, 1000, 0, 129, 0), True), ((0,), False), ((0, 0, 0), True),
                                       ((4096, 0), False)])
def test_empty_caches_bf16(lens, gate):
    """Sequences with an empty cache (a free serving slot) decode to rows of
    zeros and leave every other sequence's output as the oracle has it."""
    d = _with_lengths(lens, seed=45, gate=gate)
    if d["cache"].shape[0] == 0:                  # no cached token at all: one row, never read
        d["cache"] = np.zeros((1, 576), np.float32)
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    empty = np.array(lens) == 0
    assert np.array_equal(got[empty], np.zeros_like(got[empty]))
    if (~empty).any():
        assert rel_l2(got[~empty], want[~empty]) <= TOL_BF16


def test_many_short_sequences_with_empty_slots():
    """160 sequences of 0-200 tokens, a third of them empty: ranges step over
    the empty ones wherever they fall (first, last, in runs)."""
    rng = np.random.default_rng(46)
    lens = rng.integers(1, 201, size=160) * (rng.random(160) > 0.33)
    lens[:3] = 0
    lens[-2:] = 0
    d = _with_lengths(tuple(int(x) for x in lens), seed=47, gate=True)
    got = _run(d, "bf16")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], d["geom"], d["g"])
    empty = lens == 0
    assert np.array_equal(got[empty], np.zeros_like(got[empty]))
    assert rel_l2(got[~empty], want[~empty]) <= TOL_BF16


def test_empty_caches_fp32_tiny_geometry():
    geom = synth.TINY
    rng = np.random.default_rng(48)
    lens = np.array([0, 5, 0, 300, 0])
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    n = len(lens)
    d = dict(geom=geom, lens=lens, seq_offsets=offs,
             cache=rng.standard_normal((int(offs[-1]), geom.kv_lora + geom.d_s)).astype(np.float32),
             q=rng.standard_normal((n, geom.H, geom.d_qk)).astype(np.float32),
             W_UKV=(rng.standard_normal((geom.kv_lora, geom.H * (geom.d_c + geom.d_v))) / 8).astype(np.float32),
             g=rng.standard_normal((n, geom.H * geom.d_v)).astype(np.float32))
    got = _run(d, "f32")
    want = oracle.decode_absorbed(d["q"], d["W_UKV"], d["cache"], d["seq_offsets"], geom, d["g"])
    assert np.array_equal(got[lens == 0], np.zeros_like(got[lens == 0]))
    assert rel_l2(got, want) <= TOL_F32
