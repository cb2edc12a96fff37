"""Seeded synthetic inputs shaped like Kimi K3's gated MLA layer.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
consume exactly the arrays built here, so the two sides see the same bytes.

Every generator draws from ``numpy.random.default_rng(seed)`` in float32 and
then rounds to the workload's storage dtype (bf16 through torch's own
round-to-nearest-even cast).  Arrays come back as float32 numpy arrays whose
values are exactly representable in the storage dtype; ``to_torch`` turns
them into tensors of that dtype.

Geometry (Kimi K3 · Gated MLA · OpenModelAtlas, "All 20 steps" and the
parameter table; Gated MLA et NoPE, "Récapitulatif des couches Gated MLA"):
d = 7168, H = 96 heads, q_lora = 1536, kv_lora = 512, per-head content key
K^C 128, shared key k^S 64, value 128.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np


@dataclass(frozen=True)
class Geom:
    """Layer geometry. d_qk = d_c + d_s is the per-head query/key width."""

    H: int = 96
    d_model: int = 7168
    q_lora: int = 1536
    kv_lora: int = 512
    d_c: int = 128   # per-head content part of query and key (qk_nope_head_dim)
    d_s: int = 64    # shared key part k^S (qk_rope_head_dim, unrotated under NoPE)
    d_v: int = 128
    rms_eps: float = 1e-6

    @property
    def d_qk(self) -> int:
        return self.d_c + self.d_s

    def as_dict(self):
        return asdict(self)


K3 = Geom()
TINY = Geom(H=4, d_model=256, q_lora=128, kv_lora=64, d_c=32, d_s=16, d_v=32)


def round_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the storage dtype ("f32" or "bf16"), kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a
    if dtype == "bf16":
        import torch

        return torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def to_torch(a: np.ndarray, dtype: str, device="cpu"):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    return t.to(device)


def _normal(rng, shape, std=1.0):
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


# ---------------------------------------------------------------------------
# Attention-core workloads: Q, K^C, k^S, V, g drawn directly.
# ---------------------------------------------------------------------------
def attn_core(B: int, T: int, geom: Geom = K3, *, seed: int, hot_heads: int = 8,
              hot_scale: float = 3.0, gate: bool = True, dtype: str = "bf16"):
    """Q[B,T,H,d_qk], KC[B,T,H,d_c], kS[B,T,d_s], V[B,T,H,d_v], g[B,T,H*d_v] ~ N(0,1).

    Q and K^C of heads [0, hot_heads) are multiplied by ``hot_scale`` before
    rounding, which makes those heads' logits large (the clip's target case).
    """
    rng = np.random.default_rng(seed)
    H = geom.H
    Q = _normal(rng, (B, T, H, geom.d_qk))
    KC = _normal(rng, (B, T, H, geom.d_c))
    kS = _normal(rng, (B, T, geom.d_s))
    V = _normal(rng, (B, T, H, geom.d_v))
    g = _normal(rng, (B, T, H * geom.d_v)) if gate else None
    if hot_heads:
        Q[:, :, :hot_heads, :] *= np.float32(hot_scale)
        KC[:, :, :hot_heads, :] *= np.float32(hot_scale)
    out = dict(Q=Q, KC=KC, kS=kS, V=V, g=g)
    return {k: (None if v is None else round_storage(v, dtype)) for k, v in out.items()}


def attn_core_config(name: str):
    """The two attention-core workloads: B=2,T=2048 (hot x3) and B=1,T=16384 (hot x4)."""
    if name == "core_T2048":
        return attn_core(2, 2048, K3, seed=1, hot_heads=8, hot_scale=3.0)
    if name == "long_T16384":
        return attn_core(1, 16384, K3, seed=2, hot_heads=8, hot_scale=4.0)
    raise KeyError(name)


# ---------------------------------------------------------------------------
# Whole-layer workloads: x and the layer's weights.
# ---------------------------------------------------------------------------
def layer_weights(geom: Geom, rng, *, with_gate_out: bool):
    """Weights in math notation (y = x W, row-major [in, out]), N(0, 1/fan_in)."""
    d, H = geom.d_model, geom.H
    W = dict(
        W_DQ=_normal(rng, (d, geom.q_lora), 1.0 / np.sqrt(d)),
        W_UQ=_normal(rng, (geom.q_lora, H * geom.d_qk), 1.0 / np.sqrt(geom.q_lora)),
        W_DKV=_normal(rng, (d, geom.kv_lora + geom.d_s), 1.0 / np.sqrt(d)),
        W_UKV=_normal(rng, (geom.kv_lora, H * (geom.d_c + geom.d_v)), 1.0 / np.sqrt(geom.kv_lora)),
        w_q=np.ones(geom.q_lora, np.float32),
        w_kv=np.ones(geom.kv_lora, np.float32),
    )
    if with_gate_out:
        W["W_g"] = _normal(rng, (d, H * geom.d_v), 1.0 / np.sqrt(d))
        W["W_O"] = _normal(rng, (H * geom.d_v, d), 1.0 / np.sqrt(H * geom.d_v))
    return W


def scale_head_qk_columns(W: dict, geom: Geom, heads, factors):
    """Multiply head h's query columns in W_UQ (all d_qk) and its K^C columns in W_UKV."""
    for h, f in zip(heads, factors):
        f = np.float32(f)
        W["W_UQ"][:, h * geom.d_qk:(h + 1) * geom.d_qk] *= f
        c0 = h * (geom.d_c + geom.d_v)
        W["W_UKV"][:, c0:c0 + geom.d_c] *= f


def tiny_layer(seed: int = 0):
    """The tiny fp32 layer: B=1, T=64, geometry TINY, head scales [1,2,4,8], tau=10."""
    rng = np.random.default_rng(seed)
    geom = TINY
    x = _normal(rng, (1, 64, geom.d_model))
    W = layer_weights(geom, rng, with_gate_out=True)
    scale_head_qk_columns(W, geom, [0, 1, 2, 3], [1.0, 2.0, 4.0, 8.0])
    return dict(geom=geom, x=x, tau=10.0, dtype="f32", **W)


def k3_clip_layer(seed: int = 3, B: int = 4, T: int = 4096):
    """K3-sized clip workload: x[4,4096,7168], bf16; 12 seeded heads scaled by U(2,6); tau=100."""
    rng = np.random.default_rng(seed)
    geom = K3
    x = _normal(rng, (B, T, geom.d_model))
    W = layer_weights(geom, rng, with_gate_out=False)
    sel = np.random.default_rng(0)
    heads = sel.choice(geom.H, 12, replace=False)
    factors = sel.uniform(2.0, 6.0, size=12)
    scale_head_qk_columns(W, geom, heads, factors)
    out = dict(geom=geom, x=round_storage(x, "bf16"), tau=100.0, dtype="bf16",
               hot_heads=heads.tolist(), hot_factors=factors.tolist())
    for k, v in W.items():
        out[k] = round_storage(v, "bf16")
    return out


# ---------------------------------------------------------------------------
# Absorbed decode workload.
# ---------------------------------------------------------------------------
def decode_lengths(rng, n_seq: int, lo: int, hi: int) -> np.ndarray:
    """Context lengths: integers U[lo, hi], the first draw of the decode workload's stream."""
    return rng.integers(lo, hi + 1, size=n_seq).astype(np.int64)


def decode_batch(n_seq: int = 64, lo: int = 1024, hi: int = 8192, geom: Geom = K3,
                 seed: int = 4, gate: bool = False, dtype: str = "bf16"):
    """64 sequences with integer context lengths U[lo, hi]; latent cache [sum L, 576] ~ N(0,1).

    The cache is packed by sequence: rows seq_offsets[i] .. seq_offsets[i+1]-1
    belong to sequence i; each row is [c^KV (kv_lora) | k^S (d_s)].
    """
    rng = np.random.default_rng(seed)
    lens = decode_lengths(rng, n_seq, lo, hi)
    offsets = np.zeros(n_seq + 1, np.int64)
    offsets[1:] = np.cumsum(lens)
    total = int(offsets[-1])
    cache = _normal(rng, (total, geom.kv_lora + geom.d_s))
    q = _normal(rng, (n_seq, geom.H, geom.d_qk))
    W_UKV = _normal(rng, (geom.kv_lora, geom.H * (geom.d_c + geom.d_v)), 1.0 / np.sqrt(geom.kv_lora))
    g = _normal(rng, (n_seq, geom.H * geom.d_v)) if gate else None
    return dict(geom=geom, lens=lens, seq_offsets=offsets.astype(np.int32),
                cache=round_storage(cache, dtype), q=round_storage(q, dtype),
                W_UKV=round_storage(W_UKV, dtype),
                g=None if g is None else round_storage(g, dtype), dtype=dtype)
