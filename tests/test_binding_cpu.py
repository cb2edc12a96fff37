"""The Python binding's marshalling, on CPU: every entry point is called with
correctly laid-out tensors against a stand-in for the shared library that
records its arguments, and with one tensor at a time one element wider along
its last dimension (or a leading tensor of the wrong rank), which must be
refused before the library is called: a wrong size would let a kernel run past
the tensor, which the C ABI cannot see."""
import ctypes

import pytest
import torch

import gated_mla_qk_b200 as gm
from gated_mla_qk_b200 import synth

G = synth.TINY                     # H=4, d_model=256, q_lora=128, kv_lora=64, d_c=32, d_s=16, d_v=32
B, T, NSEQ, TOK = 2, 5, 3, 11
bf, f32 = torch.bfloat16, torch.float32


class FakeLib:
    """Records each call; workspace queries return 256 bytes, everything else GMLA_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append((name, args))
            return 256 if name.endswith("_workspace") else 0
        return f


@pytest.fixture
def lib(monkeypatch):
    fake = FakeLib()
    monkeypatch.setattr(gm, "_lib", fake)
    monkeypatch.setattr(gm, "_require_cuda", lambda t, name: None)
    monkeypatch.setattr(gm, "_stream", lambda stream=None: None)
    return fake


def _t(shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def _calls():
    """(entry point, kwargs builder) pairs with exact tensors for geometry G."""
    g = G
    W = dict(W_DQ=_t((g.d_model, g.q_lora)), w_q=_t(g.q_lora), W_UQ=_t((g.q_lora, g.H * g.d_qk)),
             W_DKV=_t((g.d_model, g.kv_lora + g.d_s)), w_kv=_t(g.kv_lora), W_UKV=_t((g.kv_lora, g.H * (g.d_c + g.d_v))))
    attn = dict(Q=_t((B, T, g.H, g.d_qk)), KC=_t((B, T, g.H, g.d_c)), kS=_t((B, T, g.d_s)), V=_t((B, T, g.H, g.d_v)),
                g=_t((B, T, g.H * g.d_v)))
    return {
        "mla_up_proj": (gm.mla_up_proj, dict(
            geom=g, x=_t((B, T, g.d_model)), **W, Q=_t((B, T, g.H, g.d_qk)), KC=_t((B, T, g.H, g.d_c)),
            kS=_t((B, T, g.d_s)), V=_t((B, T, g.H, g.d_v)), cache=_t((B, T, g.kv_lora + g.d_s)),
            workspace=_t(256, torch.uint8))),
        "mla_attn_fwd": (gm.mla_attn_fwd, dict(geom=g, **attn, O=_t((B, T, g.H * g.d_v)), maxlogit=_t(g.H, f32))),
        "mla_attn_fwd_train": (gm.mla_attn_fwd_train, dict(
            geom=g, **attn, O=_t((B, T, g.H * g.d_v), f32), maxlogit=_t(g.H, f32), lse=_t((B, T, g.H), f32))),
        "mla_attn_bwd": (gm.mla_attn_bwd, dict(
            geom=g, **attn, O=_t((B, T, g.H * g.d_v), f32), lse=_t((B, T, g.H), f32), dO=_t((B, T, g.H * g.d_v), f32),
            dQ=_t((B, T, g.H, g.d_qk), f32), dKC=_t((B, T, g.H, g.d_c), f32), dkS=_t((B, T, g.d_s), f32),
            dV=_t((B, T, g.H, g.d_v), f32), dg=_t((B, T, g.H * g.d_v), f32), workspace=_t(256, torch.uint8))),
        "qkclip_rescale": (gm.qkclip_rescale, dict(
            geom=g, W_UQ=W["W_UQ"], W_UKV=W["W_UKV"], maxlogit=_t(g.H, f32), tau=1.0,
            clipped=_t(g.H, torch.uint8), gamma=_t(g.H, f32))),
        "mla_decode_absorbed": (gm.mla_decode_absorbed, dict(
            geom=g, q=_t((NSEQ, g.H, g.d_qk)), W_UKV=W["W_UKV"], cache=_t((TOK, g.kv_lora + g.d_s)),
            seq_offsets=torch.tensor([0, 2, 9, 11], dtype=torch.int32), max_len=7, g=_t((NSEQ, g.H * g.d_v)),
            O=_t((NSEQ, g.H, g.d_v)), workspace=_t(256, torch.uint8))),
        "mla_decode_absorbed_noalloc": (gm.mla_decode_absorbed_noalloc, dict(
            geom=g, q=_t((NSEQ, g.H, g.d_qk)), W_UKV=W["W_UKV"], cache=_t((TOK, g.kv_lora + g.d_s)),
            seq_offsets=torch.tensor([0, 2, 9, 11], dtype=torch.int32), max_len=7, g=_t((NSEQ, g.H * g.d_v)),
            O=_t((NSEQ, g.H, g.d_v)))),
        "mla_attn_fwd_absorbed": (gm.mla_attn_fwd_absorbed, dict(
            geom=g, Q=attn["Q"], W_UKV=W["W_UKV"], cache=_t((B, T, g.kv_lora + g.d_s)), g=attn["g"],
            O=_t((B, T, g.H * g.d_v)), maxlogit=_t(g.H, f32), workspace=_t(256, torch.uint8))),
        "mla_gemm": (gm.mla_gemm, dict(A=_t((7, 24)), B=_t((24, 16)), C=_t((7, 16)))),
    }


@pytest.mark.parametrize("name", sorted(_calls()))
def test_exact_shapes_reach_the_library(lib, name):
    fn, kw = _calls()[name]
    fn(**kw)
    called = [c for c, _ in lib.calls if not c.endswith("_workspace")]
    assert called == [name]
    args = [a for c, a in lib.calls if c == name][0]
    ptrs = {t.data_ptr() for t in kw.values() if isinstance(t, torch.Tensor)}
    assert ptrs <= set(a for a in args if isinstance(a, int))   # every tensor went through as its pointer


def test_sizes_passed_to_the_library(lib):
    calls = _calls()
    fn, kw = calls["mla_attn_fwd"]
    fn(**kw)
    fn, kw = calls["mla_decode_absorbed"]
    fn(**kw)
    fn, kw = calls["mla_gemm"]
    fn(**kw)
    by = {c: a for c, a in lib.calls}
    assert by["mla_attn_fwd"][1:4] == (gm.GMLA_BF16, B, T)
    assert by["mla_decode_absorbed"][1:3] == (gm.GMLA_BF16, NSEQ) and by["mla_decode_absorbed"][7] == 7
    assert by["mla_gemm"][:4] == (gm.GMLA_BF16, 7, 16, 24)
    assert isinstance(by["mla_attn_fwd"][0], type(ctypes.byref(gm.CGeom.of(G))))


def _cases():
    out = []
    for name, (_, kw) in _calls().items():
        for arg, t in kw.items():
            if isinstance(t, torch.Tensor) and arg != "workspace":
                out.append((name, arg))
    return out


def _kernel_calls(lib):
    return [c for c, _ in lib.calls if not c.endswith("_workspace")]


@pytest.mark.parametrize("name,arg", _cases())
def test_a_wider_last_dimension_is_refused(lib, name, arg):
    """Each tensor in turn gets one more element along its last dimension."""
    fn, kw = _calls()[name]
    t = kw[arg]
    kw[arg] = torch.zeros(*t.shape[:-1], t.shape[-1] + 1, dtype=t.dtype)
    with pytest.raises(ValueError):
        fn(**kw)
    assert _kernel_calls(lib) == []


@pytest.mark.parametrize("name,arg", [("mla_up_proj", "x"), ("mla_attn_fwd", "Q"), ("mla_attn_bwd", "Q"),
                                      ("mla_decode_absorbed", "q"), ("mla_gemm", "A")])
def test_a_leading_tensor_of_the_wrong_rank_is_refused(lib, name, arg):
    fn, kw = _calls()[name]
    kw[arg] = kw[arg].reshape(-1)
    with pytest.raises(ValueError):
        fn(**kw)
    assert _kernel_calls(lib) == []


def test_cache_must_hold_whole_rows_and_gemm_inner_sizes_must_agree(lib):
    fn, kw = _calls()["mla_decode_absorbed"]
    kw["cache"] = torch.zeros(TOK * (G.kv_lora + G.d_s) + 3, dtype=bf)
    with pytest.raises(ValueError):
        fn(**kw)
    fn, kw = _calls()["mla_gemm"]
    kw["B"] = torch.zeros((25, 16), dtype=bf)
    with pytest.raises(ValueError):
        fn(**kw)
    assert _kernel_calls(lib) == []


def test_dtype_mismatch_is_refused(lib):
    fn, kw = _calls()["mla_attn_fwd"]
    kw["V"] = kw["V"].float()
    with pytest.raises(TypeError):
        fn(**kw)
    assert lib.calls == []
