"""The C ABI library: it builds, loads without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gmla.h")


@pytest.fixture(scope="module")
def lib():
    from gated_mla_qk_b200 import build
    build.build()
    import gated_mla_qk_b200 as g
    return g.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b([a-z][a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.startswith(("if", "defined"))))


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("mla_up_proj", "mla_attn_fwd", "qkclip_rescale", "mla_decode_absorbed"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    import gated_mla_qk_b200 as g
    names = _declared_functions()
    assert set(g.EXPORTS) <= set(names) | {"gmla_launch_count"}
    raw = ctypes.CDLL(g.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in gmla.h but not exported"


def test_version_and_strerror(lib):
    assert lib.gmla_version() >= 100
    assert lib.gmla_strerror(0) == b"ok"
    assert lib.gmla_strerror(-5) == b"device-side wait timed out"
    assert lib.gmla_strerror(12345) == b"unknown status"


def _geom(g=None):
    import gated_mla_qk_b200 as m
    return m.CGeom.of(g or m.K3)


def test_host_validation_without_gpu(lib):
    import gated_mla_qk_b200 as m
    launches_before = m.launch_count()            # other tests in this process may have launched kernels
    G = ctypes.byref(_geom())
    ok = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails earlier
    bad = ctypes.c_void_p(0x10008)     # not 16-byte aligned
    # null geometry, non-positive sizes, null or misaligned pointers
    assert lib.mla_attn_fwd(None, 0, 1, 1, ok, ok, ok, ok, None, ok, ok, None) == -1
    assert lib.mla_attn_fwd(G, 0, 0, 1, ok, ok, ok, ok, None, ok, ok, None) == -1
    assert lib.mla_attn_fwd(G, 0, 1, 1, None, ok, ok, ok, None, ok, ok, None) == -1
    assert lib.mla_attn_fwd(G, 0, 1, 1, bad, ok, ok, ok, None, ok, ok, None) == -2
    assert lib.mla_attn_fwd(G, 7, 1, 1, ok, ok, ok, ok, None, ok, ok, None) == -1
    assert lib.mla_attn_fwd(G, 0, 1, 1, ok, ok, ok, ok, bad, ok, ok, None) == -2
    # the fp32-output training form validates the same way (lse is optional)
    assert lib.mla_attn_fwd_train(None, 0, 1, 1, ok, ok, ok, ok, None, ok, None, ok, None) == -1
    assert lib.mla_attn_fwd_train(G, 0, 1, 0, ok, ok, ok, ok, None, ok, None, ok, None) == -1
    assert lib.mla_attn_fwd_train(G, 0, 1, 1, ok, ok, ok, ok, None, None, None, ok, None) == -1
    assert lib.mla_attn_fwd_train(G, 0, 1, 1, ok, ok, ok, ok, None, bad, None, ok, None) == -2
    assert lib.mla_attn_fwd_train(G, 0, 1, 1, ok, ok, ok, ok, None, ok, bad, ok, None) == -2
    assert lib.mla_attn_fwd_train(G, 0, 1, 1, ok, ok, ok, ok, None, ok, None, None, None) == -1
    # backward: every gradient buffer, O, lse, dO and a large enough workspace are required
    bneed = lib.mla_attn_bwd_workspace(G, 1, 1)
    assert bneed > 0 and lib.mla_attn_bwd_workspace(None, 1, 1) == 0
    full = lambda **kw: [kw.get(n, ok) for n in ("Q", "KC", "kS", "V", "g", "O", "lse", "dO", "dQ", "dKC", "dkS", "dV", "dg")]
    assert lib.mla_attn_bwd(G, 0, 0, 1, *full(), ok, bneed, None) == -1
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(lse=None), ok, bneed, None) == -1
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(dkS=None), ok, bneed, None) == -1
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(dg=None), ok, bneed, None) == -1        # gated needs dg
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(dQ=bad), ok, bneed, None) == -2
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(), ok, bneed - 1, None) == -6
    assert lib.mla_attn_bwd(G, 0, 1, 1, *full(), None, bneed, None) == -6
    # clip: tau must be positive and finite
    assert lib.qkclip_rescale(G, 0, ok, ok, ok, ctypes.c_float(0.0), None, None, None) == -1
    assert lib.qkclip_rescale(G, 0, ok, ok, ok, ctypes.c_float(float("inf")), None, None, None) == -1
    assert lib.qkclip_rescale(G, 0, ok, ok, None, ctypes.c_float(1.0), None, None, None) == -1
    # workspace too small / missing
    need = lib.mla_decode_workspace(G, 0, 4, 100)
    assert need > 0
    assert lib.mla_decode_absorbed(G, 0, 4, ok, ok, ok, ok, 100, None, ok, None, 0, None) == -6
    assert lib.mla_decode_absorbed(G, 0, 4, ok, ok, ok, ok, 100, None, ok, ok, need - 1, None) == -6
    assert lib.mla_decode_absorbed(G, 0, 4, ok, ok, ok, None, 100, None, ok, ok, need, None) == -1
    assert lib.mla_decode_absorbed(G, 0, 0, ok, ok, ok, ok, 100, None, ok, ok, need, None) == -1
    wsu = lib.mla_up_proj_workspace(G, 0, 2, 3)
    assert wsu > 0
    assert lib.mla_up_proj(G, 0, 2, 3, *([ok] * 11), None, ok, wsu - 1, None) == -6
    assert lib.mla_up_proj(G, 0, 2, 3, *([ok] * 10), None, None, ok, wsu, None) == -1
    assert lib.mla_gemm(0, 0, 4, 4, ok, ok, ok, None) == -1
    assert lib.mla_gemm(0, 4, 4, 4, ok, bad, ok, None) == -2
    # absorbed prefill: K3 decode geometry and bf16 only; every pointer but g required; workspace checked
    wsa = lib.mla_attn_fwd_absorbed_workspace(G, 1, 8)
    assert wsa > 0 and lib.mla_attn_fwd_absorbed_workspace(ctypes.byref(_geom(m.TINY)), 1, 8) == 0
    absorbed = lambda **kw: [kw.get(n, ok) for n in ("Q", "W", "cache", "g", "O", "ml")]
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 0, *absorbed(), ok, wsa, None) == -1
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 8, *absorbed(cache=None), ok, wsa, None) == -1
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 8, *absorbed(ml=None), ok, wsa, None) == -1
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 8, *absorbed(O=bad), ok, wsa, None) == -2
    assert lib.mla_attn_fwd_absorbed(G, 1, 1, 8, *absorbed(), ok, wsa, None) == -3
    assert lib.mla_attn_fwd_absorbed(ctypes.byref(_geom(m.TINY)), 0, 1, 8, *absorbed(), ok, wsa, None) == -3
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 8, *absorbed(), ok, wsa - 1, None) == -6
    assert lib.mla_attn_fwd_absorbed(G, 0, 1, 8, *absorbed(g=None), None, wsa, None) == -6
    # workspace queries reject bad sizes with 0
    assert lib.mla_decode_workspace(G, 0, 0, 100) == 0
    assert lib.mla_up_proj_workspace(None, 0, 1, 1) == 0
    assert m.launch_count() == launches_before, "validation failures must launch nothing"


def test_binding_refuses_missing_library(tmp_path):
    import gated_mla_qk_b200 as m
    saved = m._lib
    try:
        m._lib = None
        with pytest.raises(ImportError):
            m.load_library(str(tmp_path / "nope.so"))
    finally:
        m._lib = saved
