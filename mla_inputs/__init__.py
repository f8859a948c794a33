"""Seeded synthetic inputs for MLA absorbed decode.

This module is the one piece shared by the CUDA path's tests/benchmark and by
the CPU oracle.  It holds no attention arithmetic: it only turns a 64-bit seed
into bf16 bit patterns (and integer sequence lengths) with a counter-based
generator, so any row range of any tensor can be regenerated on its own.

Generator (each step is a published definition):
  * splitmix64 finaliser (Steele, Lea, Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014) applied to ``key + (k+1)*0x9E3779B97F4A7C15``
    gives the k-th 64-bit word of a stream; ``key`` mixes the seed and a
    per-tensor stream id.
  * uniform u = ((w >> 11) + 1) * 2^-53, in (0, 1].
  * Box-Muller (Box & Muller 1958): word pair (2k, 2k+1) gives
    r = sqrt(-2 ln u1), z_{2k} = r cos(2 pi u2), z_{2k+1} = r sin(2 pi u2).
  * value = sigma * z in fp64, rounded once to bf16 with round-to-nearest-even.

Workload shapes follow the five decode configurations of the DeepSeek-V2 MLA
description (V2-Lite: 16 heads of 128, d_c = 512, d_h^R = 64; V2: d_c = 4 d_h,
d_h^R = d_h / 2): c_KV, unrotated k^R, q_nope and q^R ~ N(0, 1); W^UK and W^UV
~ N(0, 1/512); RoPE base 10000.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

D_C = 512          # latent width d_c
D_R = 64           # decoupled RoPE width d_h^R
D_H = 128          # per-head width d_h
D_ROW = D_C + D_R  # cached elements per token per layer

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_STREAM_MUL = 0xD1B54A32D192ED03

# stream ids (one per tensor)
STREAM_C_KV = 1
STREAM_K_ROPE = 2
STREAM_Q_NOPE = 3
STREAM_Q_ROPE = 4
STREAM_W_UK = 5
STREAM_W_UV = 6
STREAM_LENGTHS = 7
STREAM_C_Q = 8
STREAM_W_UQ = 9
STREAM_W_QR = 10


def _mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _mix64_int(x: int) -> int:
    m = (1 << 64) - 1
    x &= m
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & m
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & m
    return x ^ (x >> 31)


def stream_key(seed: int, stream: int) -> int:
    return _mix64_int((seed ^ ((stream * _STREAM_MUL) & ((1 << 64) - 1))) & ((1 << 64) - 1))


def words(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """64-bit words start..start+count-1 of stream ``stream``."""
    key = np.uint64(stream_key(seed, stream))
    k = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + k * _GOLDEN)


def uniforms(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    w = words(seed, stream, start, count)
    return ((w >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (round to nearest, ties to even) in one step.

    Works on the fp64 bit pattern: the 52-bit mantissa is rounded to 7 bits,
    after which the value is exact in fp32 and its top 16 bits are the bf16.
    Only zero and the bf16 normal range are accepted (inputs here are scaled
    Gaussians, far from both ends of the range).
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    a = np.abs(x)
    nz = a != 0.0
    if np.any(nz & ((a < 2.0 ** -126) | (a >= 2.0 ** 127))):
        raise ValueError("value outside the bf16 normal range")
    b = x.view(np.uint64)
    drop = np.uint64(45)
    lsb = (b >> drop) & np.uint64(1)
    with np.errstate(over="ignore"):
        r = (b + (np.uint64((1 << 44) - 1) + lsb)) & ~np.uint64((1 << 45) - 1)
    f32 = r.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_chunk(seed, stream, start, count, sigma):
    first_pair = start // 2
    last_pair = (start + count - 1) // 2
    npair = last_pair - first_pair + 1
    u = uniforms(seed, stream, 2 * first_pair, 2 * npair).reshape(npair, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    ang = 2.0 * np.pi * u[:, 1]
    z = np.empty((npair, 2), dtype=np.float64)
    z[:, 0] = r * np.cos(ang)
    z[:, 1] = r * np.sin(ang)
    z = z.reshape(-1)[start - 2 * first_pair: start - 2 * first_pair + count]
    return f64_to_bf16_bits(sigma * z)


_CHUNK = 1 << 22


def normal_bf16(seed: int, stream: int, start: int, count: int, sigma: float = 1.0,
                threads: int | None = None) -> np.ndarray:
    """bf16 bit patterns of elements start..start+count-1 of a N(0, sigma^2) stream."""
    if count <= 0:
        return np.empty(0, dtype=np.uint16)
    if count <= _CHUNK:
        return _normal_chunk(seed, stream, start, count, sigma)
    out = np.empty(count, dtype=np.uint16)
    spans = [(o, min(_CHUNK, count - o)) for o in range(0, count, _CHUNK)]
    nthr = threads or min(32, os.cpu_count() or 1)

    def work(span):
        o, n = span
        out[o:o + n] = _normal_chunk(seed, stream, start + o, n, sigma)

    with ThreadPoolExecutor(max_workers=nthr) as ex:
        list(ex.map(work, spans))
    return out


@dataclasses.dataclass(frozen=True)
class MLAConfig:
    """One decode workload: B sequences, H heads, n_q new query tokens each."""
    name: str
    B: int
    H: int
    n_q: int
    L: int | None          # uniform context length (None: ragged)
    L_max: int = 0         # ragged: lengths uniform in [1, L_max]
    seed: int = 0
    rope_base: float = 10000.0

    @property
    def T(self) -> int:
        return self.B * self.n_q

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(D_H + D_R))


CONFIGS = {
    "tiny": MLAConfig("tiny", B=1, H=16, n_q=1, L=256, seed=0x4D4C4100),
    "v2lite": MLAConfig("v2lite", B=64, H=16, n_q=1, L=4096, seed=0x4D4C4101),
    "v2": MLAConfig("v2", B=32, H=128, n_q=1, L=8192, seed=0x4D4C4102),
    "ragged": MLAConfig("ragged", B=128, H=128, n_q=2, L=None, L_max=32768, seed=0x4D4C4103),
    "128k": MLAConfig("128k", B=4, H=128, n_q=1, L=131072, seed=0x4D4C4104),
}


def kv_lengths(cfg: MLAConfig) -> np.ndarray:
    """Per-sequence cached length L_b, counting the n_q tokens of this step.

    Ragged lengths are uniform integers in [1, L_max]; a length below n_q is
    raised to n_q so that every query sees at least one key.
    """
    if cfg.L is not None:
        return np.full(cfg.B, cfg.L, dtype=np.int64)
    u = uniforms(cfg.seed, STREAM_LENGTHS, 0, cfg.B)
    L = 1 + np.floor(u * cfg.L_max).astype(np.int64)
    L = np.minimum(L, cfg.L_max)
    return np.maximum(L, cfg.n_q)


def seq_starts(lengths: np.ndarray) -> np.ndarray:
    """Start row of each sequence in the packed token pool (sequences back to back)."""
    s = np.zeros(len(lengths), dtype=np.int64)
    if len(lengths) > 1:
        s[1:] = np.cumsum(lengths[:-1])
    return s


@dataclasses.dataclass
class SeqInputs:
    """Raw bf16 inputs of one sequence (bit patterns, uint16)."""
    b: int
    L: int
    c_kv: np.ndarray     # [L, 512]
    k_rope: np.ndarray   # [L, 64] before rotation
    q_nope: np.ndarray   # [n_q, H, 128]
    q_rope: np.ndarray   # [n_q, H, 64] before rotation


def weights(cfg: MLAConfig, which: str) -> np.ndarray:
    """W^UK or W^UV, [H, 128, 512] bf16 bits, ~N(0, 1/512)."""
    stream = {"uk": STREAM_W_UK, "uv": STREAM_W_UV}[which]
    n = cfg.H * D_H * D_C
    return normal_bf16(cfg.seed, stream, 0, n, 1.0 / np.sqrt(D_C)).reshape(cfg.H, D_H, D_C)


def compressed_queries(cfg: MLAConfig, d_cq: int):
    """Compressed queries and their up-projections, bf16 bits: c^Q [T, d_cq] ~ N(0, 1),
    W^UQ [H, 128, d_cq] and W^QR [H, 64, d_cq] ~ N(0, 1/d_cq) (so q^C and q^R are ~N(0, 1))."""
    cq = normal_bf16(cfg.seed, STREAM_C_Q, 0, cfg.T * d_cq).reshape(cfg.T, d_cq)
    sig = 1.0 / np.sqrt(d_cq)
    wuq = normal_bf16(cfg.seed, STREAM_W_UQ, 0, cfg.H * D_H * d_cq, sig).reshape(cfg.H, D_H, d_cq)
    wqr = normal_bf16(cfg.seed, STREAM_W_QR, 0, cfg.H * D_R * d_cq, sig).reshape(cfg.H, D_R, d_cq)
    return cq, wuq, wqr


def token_rows(cfg: MLAConfig, row0: int, nrows: int):
    """Rows row0..row0+nrows-1 of the packed pool: (c_kv [n,512], k_rope [n,64])."""
    c = normal_bf16(cfg.seed, STREAM_C_KV, row0 * D_C, nrows * D_C).reshape(nrows, D_C)
    k = normal_bf16(cfg.seed, STREAM_K_ROPE, row0 * D_R, nrows * D_R).reshape(nrows, D_R)
    return c, k


def queries(cfg: MLAConfig, t0: int = 0, nt: int | None = None):
    """Query rows t0..t0+nt-1 (t = b*n_q + j): (q_nope [nt,H,128], q_rope [nt,H,64])."""
    nt = cfg.T - t0 if nt is None else nt
    qn = normal_bf16(cfg.seed, STREAM_Q_NOPE, t0 * cfg.H * D_H, nt * cfg.H * D_H)
    qr = normal_bf16(cfg.seed, STREAM_Q_ROPE, t0 * cfg.H * D_R, nt * cfg.H * D_R)
    return qn.reshape(nt, cfg.H, D_H), qr.reshape(nt, cfg.H, D_R)


def sequence(cfg: MLAConfig, b: int, lengths: np.ndarray | None = None) -> SeqInputs:
    lengths = kv_lengths(cfg) if lengths is None else lengths
    starts = seq_starts(lengths)
    L = int(lengths[b])
    c, k = token_rows(cfg, int(starts[b]), L)
    qn, qr = queries(cfg, b * cfg.n_q, cfg.n_q)
    return SeqInputs(b, L, c, k, qn, qr)
