"""fp64 naive MLA decode and the facts it is pinned by -- test infrastructure.

Everything here follows the pages' definitions literally, in fp64, from the
same bf16 bit patterns the GPU receives (widened exactly).  No rounding happens
after widening.  See the package docstring for the sources and readings.
"""

from __future__ import annotations

import math

import numpy as np

D_C = 512
D_R = 64
D_H = 128


# --------------------------------------------------------------------------
# RoPE ("DeepSeek-V2 ... MLA" explainer, section 2.2.2: S = Q^T R_m^T R_n K)
# --------------------------------------------------------------------------

def rope_thetas(d: int = D_R, base: float = 10000.0) -> np.ndarray:
    """theta_i = base^(-2i/d) for pair i = 0 .. d/2-1 (original RoPE frequencies)."""
    return np.array([base ** (-2 * i / d) for i in range(d // 2)], dtype=np.float64)


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate the last axis of ``x`` (pairs (2i, 2i+1)) by angle pos * theta_i.

    ``pos`` broadcasts against x.shape[:-1].  y_{2i} = x_{2i} cos - x_{2i+1} sin,
    y_{2i+1} = x_{2i} sin + x_{2i+1} cos: the rotation matrix R_pos.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_thetas(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty(np.broadcast_shapes(x.shape, c.shape[:-1] + (d,)), dtype=np.float64)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


# --------------------------------------------------------------------------
# Cache footprint ("两张账" page, "第一张账"; reading notes, Method 1 table)
# --------------------------------------------------------------------------

def kv_elements_per_token_layer(kind: str, n_h: int = 128, d_h: int = D_H, n_g: int = 1,
                                d_c: int = D_C, d_r: int = D_R) -> int:
    """Cached elements per token per layer for MHA / GQA / MQA / MLA."""
    if kind == "mha":
        return 2 * n_h * d_h
    if kind == "gqa":
        return 2 * n_g * d_h
    if kind == "mqa":
        return 2 * d_h
    if kind == "mla":
        return d_c + d_r
    raise ValueError(kind)


def mla_equivalent_gqa_groups(d_h: int = D_H) -> float:
    """MLA cache expressed as GQA groups: (d_c + d_h^R) / (2 d_h) with d_c = 4 d_h, d_h^R = d_h/2."""
    return kv_elements_per_token_layer("mla", d_h=d_h, d_c=4 * d_h, d_r=d_h // 2) / (2 * d_h)


# --------------------------------------------------------------------------
# Naive decode ("两张账" page: the naive path rebuilds k^C and v^C from c^KV)
# --------------------------------------------------------------------------

def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def attend_naive(c_kv, k_rope_raw, q_nope, q_rope_raw, W_UK, W_UV, n_q: int,
                 scale: float | None = None, base: float = 10000.0, heads=None,
                 keep_probs: bool = False):
    """Decode step of one sequence in the naive form, fp64.

    c_kv [L, 512], k_rope_raw [L, 64] (unrotated), q_nope [n_q, H, 128],
    q_rope_raw [n_q, H, 64] (unrotated), W_UK / W_UV [H, 128, 512]; all fp64
    (already widened).  For every query j and head h:
      k^C_t = W^UK_h c_t, v^C_t = W^UV_h c_t            (per-head up-projections)
      k^R_t = R_t k_raw_t (shared by all heads), q^R = R_p q_raw, p = L - n_q + j
      s_t = [q_nope; q^R] . [k^C_t; k^R_t] * scale for t <= p
      P = softmax(s); out = sum_t P_t v^C_t; o_lat = sum_t P_t c_t; lse = log sum exp s.
    Returns out [n_q, H', 128], o_lat [n_q, H', 512], lse [n_q, H'] (+ probs).
    """
    c_kv, k_rope_raw = _f64(c_kv), _f64(k_rope_raw)
    q_nope, q_rope_raw = _f64(q_nope), _f64(q_rope_raw)
    L = c_kv.shape[0]
    H = q_nope.shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    scale = 1.0 / math.sqrt(D_H + D_R) if scale is None else scale
    if L < n_q:
        raise ValueError("each sequence must hold at least its n_q new tokens")
    k_R = rope(k_rope_raw, np.arange(L), base)                   # [L, 64]
    out = np.zeros((n_q, len(heads), D_H))
    o_lat = np.zeros((n_q, len(heads), D_C))
    lse = np.zeros((n_q, len(heads)))
    probs = {}
    for hi, h in enumerate(heads):
        Wk, Wv = _f64(W_UK[h]), _f64(W_UV[h])                    # [128, 512]
        k_C = c_kv @ Wk.T                                        # [L, 128]
        v_C = c_kv @ Wv.T                                        # [L, 128]
        for j in range(n_q):
            p = L - n_q + j
            q_R = rope(q_rope_raw[j, h], p, base)                 # [64]
            s = (k_C[:p + 1] @ q_nope[j, h] + k_R[:p + 1] @ q_R) * scale
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            P = e / z
            out[j, hi] = P @ v_C[:p + 1]
            o_lat[j, hi] = P @ c_kv[:p + 1]
            lse[j, hi] = m + math.log(z)
            if keep_probs:
                probs[(j, h)] = P
    if keep_probs:
        return out, o_lat, lse, probs
    return out, o_lat, lse


def attend_absorbed(c_kv, k_rope_raw, q_nope, q_rope_raw, W_UK, W_UV, n_q: int,
                    scale: float | None = None, base: float = 10000.0):
    """The same step in the absorbed form, fp64 (used only to pin the identity).

    q_abs,h = (W^UK_h)^T q_nope,h so that q_nope . k^C_t = q_abs . c_t; the
    output is aggregated in latent space and mapped by W^UV afterwards.
    """
    c_kv, k_rope_raw = _f64(c_kv), _f64(k_rope_raw)
    q_nope, q_rope_raw = _f64(q_nope), _f64(q_rope_raw)
    L = c_kv.shape[0]
    H = q_nope.shape[1]
    scale = 1.0 / math.sqrt(D_H + D_R) if scale is None else scale
    k_R = rope(k_rope_raw, np.arange(L), base)
    out = np.zeros((n_q, H, D_H))
    o_lat = np.zeros((n_q, H, D_C))
    lse = np.zeros((n_q, H))
    for h in range(H):
        Wk, Wv = _f64(W_UK[h]), _f64(W_UV[h])
        for j in range(n_q):
            p = L - n_q + j
            q_abs = Wk.T @ q_nope[j, h]                           # [512]
            q_R = rope(q_rope_raw[j, h], p, base)
            s = (c_kv[:p + 1] @ q_abs + k_R[:p + 1] @ q_R) * scale
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            o_lat[j, h] = (e / z) @ c_kv[:p + 1]
            out[j, h] = Wv @ o_lat[j, h]
            lse[j, h] = m + math.log(z)
    return out, o_lat, lse


# --------------------------------------------------------------------------
# Split-KV partials and their log-sum-exp merge
# --------------------------------------------------------------------------

def attend_partial_latent(c_kv, k_rope_raw, q_nope, q_rope_raw, W_UK, n_q: int, t0: int, t1: int,
                          scale: float | None = None, base: float = 10000.0):
    """Latent output and lse of every (j, h) over the key range [t0, t1) only.

    A query with no visible key in the range gets o = 0, lse = -inf.
    """
    c_kv, k_rope_raw = _f64(c_kv), _f64(k_rope_raw)
    q_nope, q_rope_raw = _f64(q_nope), _f64(q_rope_raw)
    L = c_kv.shape[0]
    H = q_nope.shape[1]
    scale = 1.0 / math.sqrt(D_H + D_R) if scale is None else scale
    k_R = rope(k_rope_raw, np.arange(L), base)
    o = np.zeros((n_q, H, D_C))
    lse = np.full((n_q, H), -np.inf)
    for h in range(H):
        Wk = _f64(W_UK[h])
        k_C = c_kv @ Wk.T
        for j in range(n_q):
            hi = min(t1, L - n_q + j + 1)
            if hi <= t0:
                continue
            q_R = rope(q_rope_raw[j, h], L - n_q + j, base)
            s = (k_C[t0:hi] @ q_nope[j, h] + k_R[t0:hi] @ q_R) * scale
            m = s.max()
            e = np.exp(s - m)
            o[j, h] = (e / e.sum()) @ c_kv[t0:hi]
            lse[j, h] = m + math.log(e.sum())
    return o, lse


def merge_partials(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Log-sum-exp merge over the split axis (axis 0).

    m = max_s lse_s; w_s = exp(lse_s - m); o = sum_s w_s o_s / sum_s w_s;
    lse = m + log sum_s w_s.  Splits with lse = -inf carry zero weight.
    """
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m[None])
    z = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / z[..., None]
    return o, m + np.log(z)


def up_project(o_lat: np.ndarray, W_UV: np.ndarray) -> np.ndarray:
    """out[t, h] = W^UV_h o_lat[t, h]  ([T, H, 512] -> [T, H, 128])."""
    return np.einsum("hdc,thc->thd", _f64(W_UV), _f64(o_lat))


def absorb_query(q_nope: np.ndarray, W_UK: np.ndarray) -> np.ndarray:
    """q_abs[t, h] = (W^UK_h)^T q_nope[t, h]  ([T, H, 128] -> [T, H, 512])."""
    return np.einsum("hdc,thd->thc", _f64(W_UK), _f64(q_nope))


# --------------------------------------------------------------------------
# Query side of the low-rank path (explainer 2.2.1.2: queries are compressed
# like K/V, a down-projection to c^Q then up-projections; q^C_t = W^UQ c^Q_t;
# 2.2.2: the decoupled per-head q^R)
# --------------------------------------------------------------------------

def query_up(c_q: np.ndarray, W_UQ: np.ndarray, W_QR: np.ndarray):
    """q^C[t, h] = W^UQ_h c^Q_t (128) and q^R[t, h] = W^QR_h c^Q_t (64, not yet rotated).

    c_q [T, d_c'], W_UQ [H, 128, d_c'], W_QR [H, 64, d_c'] -> ([T, H, 128], [T, H, 64]).
    Reading: both query parts come from the compressed query c^Q (the pages print
    q^C = W^UQ c^Q; the formula for q^R is lost, and "compressed the same way as
    K/V" is read as q^R also being an up-projection of c^Q).  The rotation R_p of
    q^R happens in the absorb step, at the query's position.
    """
    c_q = _f64(c_q)
    return (np.einsum("hdk,tk->thd", _f64(W_UQ), c_q, optimize=True),
            np.einsum("hdk,tk->thd", _f64(W_QR), c_q, optimize=True))
