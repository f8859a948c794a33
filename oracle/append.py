"""Bit-exact emulation of the latent-cache append -- test infrastructure.

What is appended ("两张账" page, "第一张账"; explainer section 2.2.2): only
c_t^KV (copied as is) and the shared key k_t^R, RoPE-rotated at the token's
position t, so no key rotation is needed when the cache is read.  One packed
row per token: columns 0..511 = c^KV, 512..575 = R_t k_raw.

The rotation is emulated in the kernel's own arithmetic so that results can be
compared bit for bit:
  * theta_i = base^(-2i/64) and the angle pos*theta_i in fp64, cos/sin from the
    C library in fp64, each rounded once to fp32 (round to nearest even);
  * y0 = fl32(fl32(x0*c) - fl32(x1*s)), y1 = fl32(fl32(x0*s) + fl32(x1*c)),
    every product and sum rounded to fp32 separately (no fused multiply-add);
  * y rounded to bf16 with round-to-nearest-even.
numpy float32 arithmetic rounds every operation to fp32 and never fuses.
"""

from __future__ import annotations

import math

import numpy as np

D_C = 512
D_R = 64
D_ROW = D_C + D_R


def rope_table_f32(positions, base: float = 10000.0, d: int = D_R):
    """(cos, sin) as fp32, shape [len(positions), d/2], from fp64 math.cos/math.sin."""
    thetas = [base ** (-2 * i / d) for i in range(d // 2)]
    positions = [int(p) for p in np.asarray(positions).reshape(-1)]
    uniq = sorted(set(positions))
    rows = {}
    for p in uniq:
        cs = np.empty(d // 2, dtype=np.float32)
        sn = np.empty(d // 2, dtype=np.float32)
        for i, th in enumerate(thetas):
            ang = float(p) * th
            cs[i] = np.float32(math.cos(ang))
            sn[i] = np.float32(math.sin(ang))
        rows[p] = (cs, sn)
    c = np.stack([rows[p][0] for p in positions]) if positions else np.empty((0, d // 2), np.float32)
    s = np.stack([rows[p][1] for p in positions]) if positions else np.empty((0, d // 2), np.float32)
    return c, s


def f32_to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    if np.any(~np.isfinite(y)):
        raise ValueError("non-finite value in the rotated key")
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def rotate_k_bits(k_raw_bits: np.ndarray, positions, base: float = 10000.0) -> np.ndarray:
    """Rotated k^R as bf16 bits, [n, 64], in the kernel's fp32 arithmetic."""
    k_raw_bits = np.asarray(k_raw_bits, dtype=np.uint16).reshape(-1, D_R)
    x = (k_raw_bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    c, s = rope_table_f32(positions, base)
    x0, x1 = x[:, 0::2], x[:, 1::2]
    y = np.empty_like(x)
    y[:, 0::2] = (x0 * c) - (x1 * s)
    y[:, 1::2] = (x0 * s) + (x1 * c)
    return f32_to_bf16_bits(y)


def append_rows(cache_bits: np.ndarray, seq_start, seq_idx, pos, c_kv_bits, k_raw_bits,
                base: float = 10000.0) -> np.ndarray:
    """Return a copy of ``cache_bits`` [cap, 576] with T tokens appended.

    Token i goes to row seq_start[seq_idx[i]] + pos[i]: c^KV into columns
    0..511 and R_pos k_raw into 512..575.  Rows not addressed stay untouched.
    """
    out = np.array(cache_bits, dtype=np.uint16, copy=True)
    seq_start = np.asarray(seq_start, dtype=np.int64)
    seq_idx = np.asarray(seq_idx, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    rows = seq_start[seq_idx] + pos
    if len(rows) and (rows.min() < 0 or rows.max() >= out.shape[0]):
        raise IndexError("append row outside the cache")
    out[rows, :D_C] = np.asarray(c_kv_bits, dtype=np.uint16).reshape(-1, D_C)
    out[rows, D_C:] = rotate_k_bits(k_raw_bits, pos, base)
    return out
