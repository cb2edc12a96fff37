"""Python binding of libgmla.so (the C ABI in include/gmla.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, checks device, dtype, contiguity and element count (the
counts follow from the geometry and the leading sizes, as include/gmla.h
lays the tensors out), and passes raw device pointers and the current CUDA
stream to the library, which runs every step of the path in its own kernels.  There is no CPU or library fallback: if the shared object is
missing, importing the binding's functions raises.

Entry points (same names as the C ABI): ``mla_up_proj``, ``mla_attn_fwd``, ``mla_attn_fwd_train``,
``mla_attn_bwd``,
``qkclip_rescale``, ``mla_decode_absorbed``, ``mla_gemm``; plus the workspace
size queries, ``device_status`` and ``launch_count``.
"""
from __future__ import annotations

import ctypes
import os

from .synth import Geom, K3, TINY  # noqa: F401  (geometry type shared with callers)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgmla.so")

GMLA_BF16, GMLA_F32 = 0, 1
STATUS = {0: "GMLA_OK", -1: "GMLA_EINVAL", -2: "GMLA_EALIGN", -3: "GMLA_EUNSUPPORTED", -4: "GMLA_ECUDA",
          -5: "GMLA_ETIMEOUT", -6: "GMLA_EWORKSPACE"}

EXPORTS = ["mla_up_proj_workspace", "mla_up_proj", "mla_attn_fwd", "mla_attn_fwd_train", "mla_attn_bwd_workspace", "mla_attn_bwd", "qkclip_rescale", "mla_decode_workspace",
           "mla_decode_absorbed", "mla_decode_absorbed_noalloc", "mla_attn_fwd_absorbed_workspace",
           "mla_attn_fwd_absorbed", "mla_gemm", "gmla_device_status", "gmla_set_wait_limit_ns", "gmla_selftest_wait", "gmla_last_cuda_error", "gmla_strerror",
           "gmla_version", "gmla_launch_count"]


class GmlaError(RuntimeError):
    def __init__(self, fn: str, status: int, lib=None):
        msg = f"{fn} failed: {STATUS.get(status, status)}"
        if lib is not None:
            msg += f" ({lib.gmla_strerror(status).decode()})"
            if status == -4:
                msg += f", cudaError {lib.gmla_last_cuda_error()}"
        super().__init__(msg)
        self.status = status


class CGeom(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("d_model", ctypes.c_int), ("q_lora", ctypes.c_int), ("kv_lora", ctypes.c_int),
                ("d_c", ctypes.c_int), ("d_s", ctypes.c_int), ("d_v", ctypes.c_int), ("rms_eps", ctypes.c_float)]

    @classmethod
    def of(cls, g: Geom) -> "CGeom":
        return cls(g.H, g.d_model, g.q_lora, g.kv_lora, g.d_c, g.d_s, g.d_v, g.rms_eps)


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libgmla.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m gated_mla_qk_b200.build` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    G = ctypes.POINTER(CGeom)
    sig = {
        "mla_up_proj_workspace": (S, [G, I, I, I]),
        "mla_up_proj": (I, [G, I, I, I] + [P] * 12 + [P, S, P]),
        "mla_attn_fwd": (I, [G, I, I, I, P, P, P, P, P, P, P, P]),
        "mla_attn_fwd_train": (I, [G, I, I, I, P, P, P, P, P, P, P, P, P]),
        "mla_attn_bwd_workspace": (S, [G, I, I]),
        "mla_attn_bwd": (I, [G, I, I, I] + [P] * 13 + [P, S, P]),
        "qkclip_rescale": (I, [G, I, P, P, P, F, P, P, P]),
        "mla_decode_workspace": (S, [G, I, I, I]),
        "mla_decode_absorbed": (I, [G, I, I, P, P, P, P, I, P, P, P, S, P]),
        "mla_decode_absorbed_noalloc": (I, [G, I, I, P, P, P, P, I, P, P, P]),
        "mla_attn_fwd_absorbed_workspace": (S, [G, I, I]),
        "mla_attn_fwd_absorbed": (I, [G, I, I, I, P, P, P, P, P, P, P, S, P]),
        "mla_gemm": (I, [I, I, I, I, P, P, P, P]),
        "gmla_device_status": (I, [P]),
        "gmla_set_wait_limit_ns": (I, [ctypes.c_ulonglong]),
        "gmla_selftest_wait": (I, [P, P]),
        "gmla_last_cuda_error": (I, []),
        "gmla_strerror": (ctypes.c_char_p, [I]),
        "gmla_version": (I, []),
        "gmla_launch_count": (ctypes.c_ulonglong, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return GMLA_BF16
    if t.dtype == torch.float32:
        return GMLA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _require_cuda(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _ptr(t, name, dtype=None, numel=None):
    """Device pointer of `t` after checking it; `numel` is the element count the
    library will read or write through it (a wrong count would make a kernel
    run past the tensor, which the C ABI cannot see)."""
    if t is None:
        return None
    _require_cuda(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _rank(t, name, dims: int, layout: str):
    if t.dim() != dims:
        raise ValueError(f"{name} must be {layout}, got shape {tuple(t.shape)}")


def _attn_counts(geom: Geom, B: int, T: int) -> dict:
    """Element counts of the attention tensors for B x T tokens (layouts of include/gmla.h)."""
    BT, H = B * T, geom.H
    return dict(Q=BT * H * geom.d_qk, KC=BT * H * geom.d_c, kS=BT * geom.d_s, V=BT * H * geom.d_v,
                O=BT * H * geom.d_v, lse=BT * H)


def _decode_counts(geom: Geom, n: int, cache) -> dict:
    """Element counts of the decode tensors for n sequences; the cache holds whole rows of kv_lora + d_s values."""
    w = geom.kv_lora + geom.d_s
    if cache is not None and cache.numel() % w != 0:
        raise ValueError(f"cache has {cache.numel()} elements, not a whole number of {w}-wide rows")
    return dict(q=n * geom.H * geom.d_qk, W_UKV=geom.kv_lora * geom.H * (geom.d_c + geom.d_v),
                O=n * geom.H * geom.d_v)


def _check(fn, status):
    if status != 0:
        raise GmlaError(fn, status, _lib)


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------
def mla_up_proj_workspace(geom: Geom, dtype_code: int, B: int, T: int) -> int:
    return load_library().mla_up_proj_workspace(ctypes.byref(CGeom.of(geom)), dtype_code, B, T)


def mla_up_proj(geom: Geom, x, W_DQ, w_q, W_UQ, W_DKV, w_kv, W_UKV, Q, KC, kS, V, cache=None, workspace=None,
                stream=None):
    """Fill Q, KC, kS, V (and the latent cache if given) from x; see include/gmla.h."""
    lib = load_library()
    _rank(x, "x", 3, "[B, T, d_model]")
    B, T = x.shape[0], x.shape[1]
    dt = _dtype_code(x)
    need = mla_up_proj_workspace(geom, dt, B, T)
    if workspace is None:
        workspace = _torch().empty(need, dtype=_torch().uint8, device=x.device)
    g, M = geom, B * T
    args = ((x, "x", M * g.d_model), (W_DQ, "W_DQ", g.d_model * g.q_lora), (w_q, "w_q", g.q_lora),
            (W_UQ, "W_UQ", g.q_lora * g.H * g.d_qk), (W_DKV, "W_DKV", g.d_model * (g.kv_lora + g.d_s)),
            (w_kv, "w_kv", g.kv_lora), (W_UKV, "W_UKV", g.kv_lora * g.H * (g.d_c + g.d_v)),
            (Q, "Q", M * g.H * g.d_qk), (KC, "KC", M * g.H * g.d_c), (kS, "kS", M * g.d_s),
            (V, "V", M * g.H * g.d_v), (cache, "cache", M * (g.kv_lora + g.d_s)))
    _check("mla_up_proj", lib.mla_up_proj(
        ctypes.byref(CGeom.of(geom)), dt, B, T, *[_ptr(a, n, x.dtype, k) for a, n, k in args],
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def mla_attn_fwd(geom: Geom, Q, KC, kS, V, g, O, maxlogit, stream=None):
    """O <- sigmoid(g) * causal softmax(QK^T/sqrt(d_qk)) V; maxlogit[h] <- head max logit."""
    lib = load_library()
    torch = _torch()
    _rank(Q, "Q", 4, "[B, T, H, d_c + d_s]")
    B, T = Q.shape[0], Q.shape[1]
    dt = _dtype_code(Q)
    n = _attn_counts(geom, B, T)
    _check("mla_attn_fwd", lib.mla_attn_fwd(
        ctypes.byref(CGeom.of(geom)), dt, B, T, _ptr(Q, "Q", None, n["Q"]), _ptr(KC, "KC", Q.dtype, n["KC"]),
        _ptr(kS, "kS", Q.dtype, n["kS"]), _ptr(V, "V", Q.dtype, n["V"]), _ptr(g, "g", Q.dtype, n["O"]),
        _ptr(O, "O", Q.dtype, n["O"]), _ptr(maxlogit, "maxlogit", torch.float32, geom.H), _stream(stream)))


def mla_attn_fwd_train(geom: Geom, Q, KC, kS, V, g, O, maxlogit, lse=None, stream=None):
    """mla_attn_fwd with the output O kept in float32 (the training form); lse (optional) gets the row log-sum-exp."""
    lib = load_library()
    torch = _torch()
    _rank(Q, "Q", 4, "[B, T, H, d_c + d_s]")
    B, T = Q.shape[0], Q.shape[1]
    dt = _dtype_code(Q)
    n = _attn_counts(geom, B, T)
    _check("mla_attn_fwd_train", lib.mla_attn_fwd_train(
        ctypes.byref(CGeom.of(geom)), dt, B, T, _ptr(Q, "Q", None, n["Q"]), _ptr(KC, "KC", Q.dtype, n["KC"]),
        _ptr(kS, "kS", Q.dtype, n["kS"]), _ptr(V, "V", Q.dtype, n["V"]), _ptr(g, "g", Q.dtype, n["O"]),
        _ptr(O, "O", torch.float32, n["O"]), _ptr(lse, "lse", torch.float32, n["lse"]),
        _ptr(maxlogit, "maxlogit", torch.float32, geom.H), _stream(stream)))


def mla_attn_bwd_workspace(geom: Geom, B: int, T: int) -> int:
    return load_library().mla_attn_bwd_workspace(ctypes.byref(CGeom.of(geom)), B, T)


def mla_attn_bwd(geom: Geom, Q, KC, kS, V, g, O, lse, dO, dQ, dKC, dkS, dV, dg=None, workspace=None, stream=None):
    """Gradients (float32) of the loss through the gated attention: dQ, dKC, dkS (summed over heads), dV, dg."""
    lib = load_library()
    torch = _torch()
    _rank(Q, "Q", 4, "[B, T, H, d_c + d_s]")
    B, T = Q.shape[0], Q.shape[1]
    f32 = torch.float32
    if workspace is None:
        workspace = torch.empty(mla_attn_bwd_workspace(geom, B, T), dtype=torch.uint8, device=Q.device)
    n = _attn_counts(geom, B, T)
    _check("mla_attn_bwd", lib.mla_attn_bwd(
        ctypes.byref(CGeom.of(geom)), _dtype_code(Q), B, T, _ptr(Q, "Q", None, n["Q"]),
        _ptr(KC, "KC", Q.dtype, n["KC"]), _ptr(kS, "kS", Q.dtype, n["kS"]), _ptr(V, "V", Q.dtype, n["V"]),
        _ptr(g, "g", Q.dtype, n["O"]), _ptr(O, "O", f32, n["O"]), _ptr(lse, "lse", f32, n["lse"]),
        _ptr(dO, "dO", f32, n["O"]), _ptr(dQ, "dQ", f32, n["Q"]), _ptr(dKC, "dKC", f32, n["KC"]),
        _ptr(dkS, "dkS", f32, n["kS"]), _ptr(dV, "dV", f32, n["V"]), _ptr(dg, "dg", f32, n["O"]),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def qkclip_rescale(geom: Geom, W_UQ, W_UKV, maxlogit, tau: float, clipped=None, gamma=None, stream=None):
    """In-place QK-Clip of W_UQ / W_UKV for heads with maxlogit > tau."""
    lib = load_library()
    torch = _torch()
    dt = _dtype_code(W_UQ)
    H = geom.H
    _check("qkclip_rescale", lib.qkclip_rescale(
        ctypes.byref(CGeom.of(geom)), dt, _ptr(W_UQ, "W_UQ", None, geom.q_lora * H * geom.d_qk),
        _ptr(W_UKV, "W_UKV", W_UQ.dtype, geom.kv_lora * H * (geom.d_c + geom.d_v)),
        _ptr(maxlogit, "maxlogit", torch.float32, H), float(tau), _ptr(clipped, "clipped", torch.uint8, H),
        _ptr(gamma, "gamma", torch.float32, H), _stream(stream)))


def mla_decode_workspace(geom: Geom, dtype_code: int, n_seq: int, max_len: int) -> int:
    return load_library().mla_decode_workspace(ctypes.byref(CGeom.of(geom)), dtype_code, n_seq, max_len)


def mla_decode_absorbed(geom: Geom, q, W_UKV, cache, seq_offsets, max_len: int, g, O, workspace=None, stream=None):
    """Absorbed-latent decode of one query token per sequence; see include/gmla.h."""
    lib = load_library()
    torch = _torch()
    _rank(q, "q", 3, "[n_seq, H, d_c + d_s]")
    dt = _dtype_code(q)
    n = q.shape[0]
    need = mla_decode_workspace(geom, dt, n, max_len)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    c = _decode_counts(geom, n, cache)
    _check("mla_decode_absorbed", lib.mla_decode_absorbed(
        ctypes.byref(CGeom.of(geom)), dt, n, _ptr(q, "q", None, c["q"]), _ptr(W_UKV, "W_UKV", q.dtype, c["W_UKV"]),
        _ptr(cache, "cache", q.dtype), _ptr(seq_offsets, "seq_offsets", torch.int32, n + 1), int(max_len),
        _ptr(g, "g", q.dtype, c["O"]), _ptr(O, "O", q.dtype, c["O"]), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def mla_decode_absorbed_noalloc(geom: Geom, q, W_UKV, cache, seq_offsets, max_len: int, g, O, stream=None):
    """mla_decode_absorbed on the library's fixed 16 MiB device scratch (no workspace).

    For callers that cannot allocate device memory on their request path; see
    include/gmla.h for the size limit and the sharing rules of the scratch.
    """
    lib = load_library()
    torch = _torch()
    _rank(q, "q", 3, "[n_seq, H, d_c + d_s]")
    n = q.shape[0]
    c = _decode_counts(geom, n, cache)
    _check("mla_decode_absorbed_noalloc", lib.mla_decode_absorbed_noalloc(
        ctypes.byref(CGeom.of(geom)), _dtype_code(q), n, _ptr(q, "q", None, c["q"]),
        _ptr(W_UKV, "W_UKV", q.dtype, c["W_UKV"]), _ptr(cache, "cache", q.dtype),
        _ptr(seq_offsets, "seq_offsets", torch.int32, n + 1), int(max_len), _ptr(g, "g", q.dtype, c["O"]),
        _ptr(O, "O", q.dtype, c["O"]), _stream(stream)))


def mla_attn_fwd_absorbed_workspace(geom: Geom, B: int, T: int) -> int:
    return load_library().mla_attn_fwd_absorbed_workspace(ctypes.byref(CGeom.of(geom)), B, T)


def mla_attn_fwd_absorbed(geom: Geom, Q, W_UKV, cache, g, O, maxlogit, workspace=None, stream=None):
    """mla_attn_fwd's O and maxlogit computed on the latent cache (absorbed form); see include/gmla.h."""
    lib = load_library()
    torch = _torch()
    _rank(Q, "Q", 4, "[B, T, H, d_c + d_s]")
    B, T = Q.shape[0], Q.shape[1]
    if workspace is None:
        workspace = torch.empty(mla_attn_fwd_absorbed_workspace(geom, B, T), dtype=torch.uint8, device=Q.device)
    n = _attn_counts(geom, B, T)
    _check("mla_attn_fwd_absorbed", lib.mla_attn_fwd_absorbed(
        ctypes.byref(CGeom.of(geom)), _dtype_code(Q), B, T, _ptr(Q, "Q", None, n["Q"]),
        _ptr(W_UKV, "W_UKV", Q.dtype, geom.kv_lora * geom.H * (geom.d_c + geom.d_v)),
        _ptr(cache, "cache", Q.dtype, B * T * (geom.kv_lora + geom.d_s)), _ptr(g, "g", Q.dtype, n["O"]),
        _ptr(O, "O", Q.dtype, n["O"]), _ptr(maxlogit, "maxlogit", torch.float32, geom.H),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def mla_gemm(A, B, C, stream=None):
    """C <- A @ B (row-major), fp32 accumulation."""
    lib = load_library()
    _rank(A, "A", 2, "[M, K]")
    M, K = A.shape
    if B.dim() != 2 or B.shape[0] != K:
        raise ValueError(f"B has shape {tuple(B.shape)}, expected [{K}, N]")
    N = B.shape[1]
    _check("mla_gemm", lib.mla_gemm(_dtype_code(A), M, N, K, _ptr(A, "A"), _ptr(B, "B", A.dtype),
                                    _ptr(C, "C", A.dtype, M * N), _stream(stream)))


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device error status."""
    return load_library().gmla_device_status(_stream(stream))


def set_wait_limit_ns(ns: int = 0) -> None:
    """Limit of the kernels' device-side waits in nanoseconds (0: the 2 s default); see include/gmla.h."""
    _check("gmla_set_wait_limit_ns", load_library().gmla_set_wait_limit_ns(int(ns)))


def selftest_wait(elapsed, stream=None) -> None:
    """Launch the bounded-wait self-test; ``elapsed`` is a CUDA int64 tensor of 2 (see include/gmla.h)."""
    torch = _torch()
    _check("gmla_selftest_wait", load_library().gmla_selftest_wait(_ptr(elapsed, "elapsed", torch.int64, 2),
                                                                   _stream(stream)))


def launch_count() -> int:
    return int(load_library().gmla_launch_count())
