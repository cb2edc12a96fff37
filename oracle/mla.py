"""Plain float64 CPU restatement of the gated MLA hot path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs use this module.  The CUDA library never calls it.

Sources (cited by page title and section):
  [OMA]  "Kimi K3 · Gated MLA · OpenModelAtlas" — the "All 20 steps" formula
         list, the parameter table and the quoted attention / projection code.
  [NOPE] "Gated MLA et NoPE" — the cache-size table ("Le principe") and the
         layer summary ("Récapitulatif des couches Gated MLA").
  [SOTA] "Anthology of the SOTA", record SOTA-131 (QK-Clip), "Source" and
         "Conditions" paragraphs.
  [FW]   "Kimi Qkclip" (Fireworks blog), section 3, "Training vs. Inference in
         Multi-Head Latent Attention": training materialises per-head keys,
         decoding works on the cached latent.

Notation follows [OMA]: x W with row-major weights W[in, out]; per head h the
query is [q^C_h (d_c) | q^S_h (d_s)], the key is K_h = [K^C_h | k^S] with k^S
shared by all heads, the value is V_h (d_v); S = Q K^T / sqrt(d_c + d_s).

Precision: every sum, exp and division here is float64.  Where the layer
stores an activation in its model dtype (each projection and norm output in
the quoted HF module), ``dtype="bf16"`` rounds that activation to bf16 with
round-to-nearest-even, as the module boundary does; ``dtype="f32"`` rounds to
float32.  The QK-Clip rescale is the one place where float32 arithmetic is the
definition (see ``qkclip``).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_round", "rms_norm", "up_proj", "attention", "attention_rows", "head_maxlogit",
    "attention_lse", "attention_backward", "qkclip", "decode_absorbed", "decode_materialised", "layer_forward",
]


# ---------------------------------------------------------------------------
# Storage rounding
# ---------------------------------------------------------------------------
def bf16_round(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as float32.

    bf16 keeps the float32 exponent and the top 7 stored mantissa bits, so
    rounding is done on the bit pattern: add half an ulp of the kept field
    (plus one if the kept field is odd, which breaks ties to even) and clear
    the dropped bits.  float64 input is rounded directly from its 52-bit
    mantissa (one rounding, no detour through float32).  Inputs are assumed
    finite and inside the float32 normal range.
    """
    a = np.asarray(a)
    if a.dtype == np.float64:
        u = a.view(np.uint64)
        drop = np.uint64(45)                       # 52 - 7 mantissa bits dropped
        lsb = (u >> drop) & np.uint64(1)
        u = (u + (np.uint64(1) << np.uint64(44)) - np.uint64(1) + lsb) & ~((np.uint64(1) << drop) - np.uint64(1))
        return u.view(np.float64).astype(np.float32)
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    u = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    """The module-boundary rounding of an activation, returned as float64."""
    if dtype == "bf16":
        return bf16_round(a).astype(np.float64)
    if dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    if dtype == "f64":
        return a
    raise ValueError(dtype)


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Up-projections  [OMA] "All 20 steps", query heads and key/value heads
# ---------------------------------------------------------------------------
def rms_norm(c, w, eps):
    """RMSNorm over the last axis: c / sqrt(mean(c^2) + eps) * w.

    The pages name the module (KimiRMSNorm on q_lora and kv_lora widths, [OMA]
    quoted ``__init__``) and the parameter table counts one weight per
    feature; the standard RMSNorm formula and eps = 1e-6 are this build's
    reading of an unstated detail.
    """
    c = _f64(c)
    ms = np.mean(c * c, axis=-1, keepdims=True)
    return c / np.sqrt(ms + eps) * _f64(w)


def up_proj(x, W_DQ, w_q, W_UQ, W_DKV, w_kv, W_UKV, geom, dtype="bf16"):
    """Queries, per-head content keys, the shared key and values from x.

    [OMA] "All 20 steps":
      c^Q = x W_DQ;            q = RMSNorm(c^Q) W_UQ, per head [q^C (d_c) | q^S (d_s)]
      [c^KV k^S] = x W_DKV;    c^KV = first kv_lora columns, k^S = last d_s columns
      [k^C v] = RMSNorm(c^KV) W_UKV, per head h: K^C_h = cols [0, d_c), V_h = cols [d_c, d_c+d_v)
    k^S is not normalised (the norm acts on c^KV only).  Returns float64
    arrays rounded at each module boundary to ``dtype``:
      Q [B,T,H,d_qk], KC [B,T,H,d_c], kS [B,T,d_s], V [B,T,H,d_v],
      cache [B,T,kv_lora+d_s] = [RMSNorm(c^KV) | k^S] (the latent a decoder keeps).
    """
    x = _f64(x)
    B, T, _ = x.shape
    H = geom.H
    c_Q = _store(x @ _f64(W_DQ), dtype)
    c_Q_hat = _store(rms_norm(c_Q, w_q, geom.rms_eps), dtype)
    q = _store(c_Q_hat @ _f64(W_UQ), dtype).reshape(B, T, H, geom.d_qk)

    ckv_ks = _store(x @ _f64(W_DKV), dtype)
    c_KV = ckv_ks[..., :geom.kv_lora]
    k_S = ckv_ks[..., geom.kv_lora:]
    c_KV_hat = _store(rms_norm(c_KV, w_kv, geom.rms_eps), dtype)
    kv = _store(c_KV_hat @ _f64(W_UKV), dtype).reshape(B, T, H, geom.d_c + geom.d_v)
    return dict(
        Q=q,
        KC=kv[..., :geom.d_c].copy(),
        kS=k_S.copy(),
        V=kv[..., geom.d_c:].copy(),
        cache=np.concatenate([c_KV_hat, k_S], axis=-1),
        c_Q=c_Q, c_Q_hat=c_Q_hat, c_KV=c_KV, c_KV_hat=c_KV_hat,
    )


# ---------------------------------------------------------------------------
# Causal attention with the output gate  [OMA] "All 20 steps", causal attention
# ---------------------------------------------------------------------------
def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _head_keys(KC, kS, b, h):
    """K_h = [K^C_h | k^S] for batch item b: [T, d_c + d_s]."""
    return np.concatenate([KC[b, :, h, :], kS[b]], axis=-1)


def attention(Q, KC, kS, V, g=None, *, heads=None, row_chunk=1024):
    """Causal gated attention and the per-head max logit.

    For each batch item b and head h ([OMA] "All 20 steps"):
      S = Q_h K_h^T / sqrt(d_qk)
      A[t, s] = exp S[t, s] / sum_{u <= t} exp S[t, u]   for s <= t, 0 for s > t
      O~_h = A V_h;  o = sigmoid(g) * reshape(O~)   (no gate when g is None)
    The max logit of head h is the largest scaled logit S[t, s] over all batch
    items and causal pairs s <= t — the statistic QK-Clip watches per head
    ([SOTA] "Source", "Conditions").  Masked pairs s > t are not logits.

    Rows are processed ``row_chunk`` at a time; each row's value depends only
    on that row, so the chunking is bookkeeping, not a reordering of any sum.
    Returns (O [B,T,H,d_v] float64, maxlogit [H] float64); heads not listed in
    ``heads`` are left as NaN.
    """
    B, T, H, d_qk = Q.shape
    d_v = V.shape[-1]
    scale = 1.0 / math.sqrt(d_qk)
    heads = range(H) if heads is None else heads
    O = np.full((B, T, H, d_v), np.nan)
    maxlogit = np.full(H, np.nan)
    for h in heads:
        m_h = -np.inf
        for b in range(B):
            K = _f64(_head_keys(KC, kS, b, h))
            Vh = _f64(V[b, :, h, :])
            for t0 in range(0, T, row_chunk):
                t1 = min(T, t0 + row_chunk)
                S = (_f64(Q[b, t0:t1, h, :]) @ K[:t1].T) * scale    # [rows, t1]
                causal = np.arange(t1)[None, :] <= np.arange(t0, t1)[:, None]
                S = np.where(causal, S, -np.inf)
                m_h = max(m_h, float(S.max()))
                m = S.max(axis=1, keepdims=True)
                P = np.exp(S - m)
                A = P / P.sum(axis=1, keepdims=True)
                O[b, t0:t1, h, :] = A @ Vh[:t1]
        maxlogit[h] = m_h
    if g is not None:
        O = O * _sigmoid(_f64(g).reshape(B, T, H, d_v))
    return O, maxlogit


def attention_rows(Q, KC, kS, V, g, rows):
    """Gated attention output for individual (b, t, h) rows: [len(rows), d_v].

    Same definition as ``attention`` evaluated one query row at a time, so a
    sample of a very long sequence can be checked without the whole T x T.
    Also returns each row's own max scaled logit over s <= t.
    """
    out, row_max = [], []
    d_qk = Q.shape[-1]
    scale = 1.0 / math.sqrt(d_qk)
    for (b, t, h) in rows:
        q = _f64(Q[b, t, h, :])
        K = np.concatenate([_f64(KC[b, :t + 1, h, :]), _f64(kS[b, :t + 1])], axis=-1)
        s = (K @ q) * scale
        row_max.append(float(s.max()))
        p = np.exp(s - s.max())
        o = (p / p.sum()) @ _f64(V[b, :t + 1, h, :])
        if g is not None:
            d_v = o.shape[-1]
            o = o * _sigmoid(_f64(g[b, t, h * d_v:(h + 1) * d_v]))
        out.append(o)
    return np.stack(out), np.array(row_max)


def head_maxlogit(Q, KC, kS, heads, *, row_chunk=2048):
    """max_{b, t, s <= t} S_h[t, s] for the listed heads (QK only, no softmax)."""
    B, T, H, d_qk = Q.shape
    scale = 1.0 / math.sqrt(d_qk)
    res = {}
    for h in heads:
        m_h = -np.inf
        for b in range(B):
            K = np.concatenate([_f64(KC[b, :, h, :]), _f64(kS[b])], axis=-1)
            for t0 in range(0, T, row_chunk):
                t1 = min(T, t0 + row_chunk)
                S = (_f64(Q[b, t0:t1, h, :]) @ K[:t1].T) * scale
                causal = np.arange(t1)[None, :] <= np.arange(t0, t1)[:, None]
                m_h = max(m_h, float(np.where(causal, S, -np.inf).max()))
        res[int(h)] = m_h
    return res


# ---------------------------------------------------------------------------
# Training: the row log-sum-exp the forward leaves for the backward, and the
# gradients of the forward above.  The pages run this layer in training (the
# clip exists for it: [SOTA] "Source"; [NOPE] "Un détail de précision
# numérique" keeps the forward's output in FP32 while training); k^S being one
# key part shared by every head ([OMA] "All 20 steps") makes its gradient a
# sum over heads.
# ---------------------------------------------------------------------------
def attention_lse(Q, KC, kS):
    """lse[b, t, h] = log sum_{s <= t} exp S_h[t, s], S the scaled logits."""
    B, T, H, d_qk = Q.shape
    scale = 1.0 / math.sqrt(d_qk)
    out = np.empty((B, T, H))
    causal = np.arange(T)[None, :] <= np.arange(T)[:, None]
    for b in range(B):
        for h in range(H):
            K = _f64(_head_keys(KC, kS, b, h))
            S = np.where(causal, (_f64(Q[b, :, h, :]) @ K.T) * scale, -np.inf)
            m = S.max(axis=1, keepdims=True)
            out[b, :, h] = (m + np.log(np.exp(S - m).sum(axis=1, keepdims=True)))[:, 0]
    return out


def attention_backward(Q, KC, kS, V, g, dO):
    """Gradients of the loss through o = sigmoid(g) * causal-softmax(Q K^T/sqrt(d_qk)) V.

    dO is dL/do [B, T, H*d_v].  Per batch item b and head h, with K_h =
    [K^C_h | k^S], A the causal softmax and O~ = A V_h (chain rule, in order):
      dO~     = dO * sigmoid(g)            dg = dO * O~ * sigmoid(g) (1 - sigmoid(g))
      dV_h    = A^T dO~                    dA = dO~ V_h^T
      dS      = A * (dA - rowsum(dA * A))  (softmax Jacobian; masked entries of A are 0)
      dQ_h    = dS K_h / sqrt(d_qk)        dK_h = dS^T Q_h / sqrt(d_qk)
    and dK_h splits into dK^C_h (its first d_c columns) and head h's share of
    dk^S (the rest); dk^S is the sum of the shares over the heads.
    Returns float64 (dQ [B,T,H,d_qk], dKC [B,T,H,d_c], dkS [B,T,d_s],
    dV [B,T,H,d_v], dg [B,T,H*d_v] or None when g is None).
    """
    B, T, H, d_qk = Q.shape
    d_c, d_v = KC.shape[-1], V.shape[-1]
    scale = 1.0 / math.sqrt(d_qk)
    dO = _f64(dO).reshape(B, T, H, d_v)
    gg = None if g is None else _f64(g).reshape(B, T, H, d_v)
    dQ = np.zeros((B, T, H, d_qk))
    dKC = np.zeros((B, T, H, d_c))
    dkS = np.zeros((B, T, d_qk - d_c))
    dV = np.zeros((B, T, H, d_v))
    dg = None if g is None else np.zeros((B, T, H, d_v))
    causal = np.arange(T)[None, :] <= np.arange(T)[:, None]
    for b in range(B):
        for h in range(H):
            K = _f64(_head_keys(KC, kS, b, h))
            Qh, Vh = _f64(Q[b, :, h, :]), _f64(V[b, :, h, :])
            S = np.where(causal, (Qh @ K.T) * scale, -np.inf)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            A = P / P.sum(axis=1, keepdims=True)
            Ot = A @ Vh
            if gg is None:
                dOt = dO[b, :, h, :]
            else:
                sg = _sigmoid(gg[b, :, h, :])
                dOt = dO[b, :, h, :] * sg
                dg[b, :, h, :] = dO[b, :, h, :] * Ot * sg * (1.0 - sg)
            dV[b, :, h, :] = A.T @ dOt
            dA = dOt @ Vh.T
            dS = A * (dA - (dA * A).sum(axis=1, keepdims=True))
            dQ[b, :, h, :] = (dS @ K) * scale
            dK = (dS.T @ Qh) * scale
            dKC[b, :, h, :] = dK[:, :d_c]
            dkS[b] += dK[:, d_c:]
    return dQ, dKC, dkS, dV, (None if dg is None else dg.reshape(B, T, H * d_v))


# ---------------------------------------------------------------------------
# QK-Clip  [SOTA] "Source": per head, when its max logit exceeds the
# threshold, rescale that head's query and key projection weights.
# ---------------------------------------------------------------------------
def qkclip(W_UQ, W_UKV, maxlogit, tau, geom, dtype="bf16"):
    """Rescale the clipped heads' query and key projection columns.

    A head h is clipped when maxlogit_h > tau (strictly; [SOTA] says the clip
    acts on heads whose max logit exceeds the threshold).  For a clipped head
    gamma_h = tau / maxlogit_h and
      W_UQ  columns of q^C_h  (h*d_qk + [0, d_c))           *= sqrt(gamma_h)
      W_UQ  columns of q^S_h  (h*d_qk + [d_c, d_qk))        *= gamma_h
      W_UKV columns of K^C_h  (h*(d_c+d_v) + [0, d_c))      *= sqrt(gamma_h)
    k^S (in W_DKV, shared by every head) and the V_h columns are untouched, so
    every logit of head h becomes gamma_h times its old value and the new max
    logit is tau.  How gamma is split between the per-head and the shared key
    part is not stated on the pages; this split is the one that scales all of
    S_h by gamma_h without touching a tensor other heads share.

    Arithmetic is float32 as stored weights are scaled in practice: gamma is
    one IEEE float32 division, sqrt(gamma) the correctly rounded float32
    square root, each new weight one float32 product rounded to the storage
    dtype (RNE).  Returns (W_UQ', W_UKV', clipped uint8 [H], gamma float32 [H]
    with 1 for unclipped heads); the inputs are not modified.
    """
    ml = np.asarray(maxlogit, dtype=np.float32)
    tau32 = np.float32(tau)
    WQ = np.array(W_UQ, dtype=np.float32, copy=True)
    WKV = np.array(W_UKV, dtype=np.float32, copy=True)
    H = geom.H
    clipped = np.zeros(H, np.uint8)
    gamma = np.ones(H, np.float32)

    def scaled(block, f):
        prod = (block.astype(np.float32) * np.float32(f)).astype(np.float32)
        return bf16_round(prod) if dtype == "bf16" else prod

    for h in range(H):
        if not (ml[h] > tau32):
            continue
        gam = np.float32(tau32 / ml[h])
        root = np.sqrt(gam, dtype=np.float32)
        clipped[h] = 1
        gamma[h] = gam
        q0 = h * geom.d_qk
        WQ[:, q0:q0 + geom.d_c] = scaled(WQ[:, q0:q0 + geom.d_c], root)
        WQ[:, q0 + geom.d_c:q0 + geom.d_qk] = scaled(WQ[:, q0 + geom.d_c:q0 + geom.d_qk], gam)
        k0 = h * (geom.d_c + geom.d_v)
        WKV[:, k0:k0 + geom.d_c] = scaled(WKV[:, k0:k0 + geom.d_c], root)
    return WQ, WKV, clipped, gamma


# ---------------------------------------------------------------------------
# Decode over the latent cache  [FW] section 3; [NOPE] "Le principe"
# ---------------------------------------------------------------------------
def _uk_uv(W_UKV, geom, h):
    w = _f64(W_UKV)
    c0 = h * (geom.d_c + geom.d_v)
    return w[:, c0:c0 + geom.d_c], w[:, c0 + geom.d_c:c0 + geom.d_c + geom.d_v]


def decode_absorbed(q, W_UKV, cache, seq_offsets, geom, g=None):
    """One query token per sequence attending over its whole cached latent.

    The cache row of token j is [c^KV_j (kv_lora) | k^S_j (d_s)] ([NOPE]
    "Le principe": 512 + 64 values per token).  Since K^C_{h,j} = c^KV_j W_UK,h
    with W_UK,h the K^C_h columns of W_UKV, q^C_h . K^C_{h,j} equals
    (q^C_h W_UK,h^T) . c^KV_j; the absorbed query is
      q~_h = [q^C_h W_UK,h^T | q^S_h]               (kv_lora + d_s)
      s_j  = q~_h . cache_j / sqrt(d_qk)            (the scale of the d_qk-wide head)
      u_h  = sum_j softmax(s)_j c^KV_j              (kv_lora)
      o_h  = u_h W_UV,h                             (d_v), then * sigmoid(g) if given.
    Every cached token is visible (the query is the newest position).  A
    sequence with no cached token has nothing to attend to; its output is the
    empty sum, 0 (a reading: the pages never decode an empty cache).
    Returns O [n_seq, H, d_v] float64.
    """
    q, cache = _f64(q), _f64(cache)
    n = q.shape[0]
    H = geom.H
    scale = 1.0 / math.sqrt(geom.d_qk)
    W = _f64(W_UKV).reshape(geom.kv_lora, H, geom.d_c + geom.d_v)
    W_UK = W[:, :, :geom.d_c]                      # [kv_lora, H, d_c]
    W_UV = W[:, :, geom.d_c:]                      # [kv_lora, H, d_v]
    O = np.zeros((n, H, geom.d_v))
    for i in range(n):
        C = cache[int(seq_offsets[i]):int(seq_offsets[i + 1])]          # [L, kv_lora + d_s]
        if C.shape[0] == 0:
            continue                                                      # empty cache: O[i] stays 0
        # q~_h = [q^C_h W_UK,h^T | q^S_h] for every head at once: [H, kv_lora + d_s]
        q_abs = np.concatenate([np.einsum("lhc,hc->hl", W_UK, q[i, :, :geom.d_c]), q[i, :, geom.d_c:]], axis=-1)
        s = (C @ q_abs.T) * scale                                         # [L, H]
        p = np.exp(s - s.max(axis=0, keepdims=True))
        p /= p.sum(axis=0, keepdims=True)
        u = p.T @ C[:, :geom.kv_lora]                                     # [H, kv_lora]
        O[i] = np.einsum("hl,lhv->hv", u, W_UV)
    if g is not None:
        O = O * _sigmoid(_f64(g).reshape(n, H, geom.d_v))
    return O


def decode_materialised(q, W_UKV, cache, seq_offsets, geom, g=None):
    """The same decode in the training form: build every head's keys and values.

    K_{h,j} = [c^KV_j W_UK,h | k^S_j], V_{h,j} = c^KV_j W_UV,h, then ordinary
    softmax attention of q_h over all cached positions ([FW] section 3: the
    training form materialises the per-head keys, decoding cannot afford to).
    An empty cache gives 0, as in ``decode_absorbed``.
    """
    q, cache = _f64(q), _f64(cache)
    n = q.shape[0]
    H = geom.H
    scale = 1.0 / math.sqrt(geom.d_qk)
    O = np.zeros((n, H, geom.d_v))
    for i in range(n):
        C = cache[int(seq_offsets[i]):int(seq_offsets[i + 1])]
        if C.shape[0] == 0:
            continue
        for h in range(H):
            W_UK, W_UV = _uk_uv(W_UKV, geom, h)
            K = np.concatenate([C[:, :geom.kv_lora] @ W_UK, C[:, geom.kv_lora:]], axis=-1)
            Vh = C[:, :geom.kv_lora] @ W_UV
            s = (K @ q[i, h]) * scale
            p = np.exp(s - s.max())
            O[i, h] = (p / p.sum()) @ Vh
    if g is not None:
        O = O * _sigmoid(_f64(g).reshape(n, H, geom.d_v))
    return O


# ---------------------------------------------------------------------------
# Whole layer  [OMA] "All 20 steps" end to end
# ---------------------------------------------------------------------------
def layer_forward(x, W, geom, dtype="f32"):
    """x -> Delta_attn: up-projections, causal attention, gate g = x W_g, output W_O.

    Returns a dict with the up-projection outputs, g, o (gated attention,
    [B,T,H*d_v]), maxlogit [H] and delta = o W_O.
    """
    up = up_proj(x, W["W_DQ"], W["w_q"], W["W_UQ"], W["W_DKV"], W["w_kv"], W["W_UKV"], geom, dtype)
    g = _store(_f64(x) @ _f64(W["W_g"]), dtype)
    O, ml = attention(up["Q"], up["KC"], up["kS"], up["V"], g)
    B, T = O.shape[:2]
    o = _store(O.reshape(B, T, -1), dtype)
    delta = o @ _f64(W["W_O"])
    return dict(up, g=g, o=o, maxlogit=ml, delta=delta)
