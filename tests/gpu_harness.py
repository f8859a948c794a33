"""Build seeded MLA decode problems on the GPU through the C ABI, and compare
with the fp64 oracle on chosen sequences (test helper, GPU tests only)."""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

import mla_inputs as mi
import mla_latent_kv_34_b200 as mla
from oracle import naive as on

NAN_BF16 = 0x7FC0  # quiet NaN pattern put in cache rows no sequence owns
BLOCK_TOKENS, BLOCK_BYTES = 128, 147456


def _block_index_map() -> np.ndarray:
    """[128, 576] uint16 offsets inside a cache block of (row r, column c), per the mla.h layout."""
    r = np.arange(BLOCK_TOKENS)[:, None]
    c = np.arange(576)[None, :]
    byte = (c // 64) * (BLOCK_TOKENS * 128) + r * 128 + ((((c % 64) // 8) ^ (r % 8)) * 16) + (c % 8) * 2
    return (byte // 2).astype(np.int64)


BLOCK_MAP = _block_index_map()


def unpack_rows(cache_u16: np.ndarray, blocks: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Logical [n, 576] rows (bf16 bits) of a blocked cache given as uint16 [cap_blocks, 36864]."""
    return cache_u16[np.asarray(blocks)[:, None], BLOCK_MAP[np.asarray(rows)]]


def pack_rows(cache_u16: np.ndarray, blocks: np.ndarray, rows: np.ndarray, values: np.ndarray) -> None:
    """Inverse of unpack_rows (in place)."""
    cache_u16[np.asarray(blocks)[:, None], BLOCK_MAP[np.asarray(rows)]] = values


def cache_u16(cache: torch.Tensor) -> np.ndarray:
    return cache.cpu().numpy().view(np.uint16).reshape(cache.shape[0], BLOCK_BYTES // 2)


def to_dev_bf16(bits: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def tol_excess(got: np.ndarray, ref: np.ndarray, atol=1e-2, rtol=1e-2) -> float:
    """max(|got - ref| - (atol + rtol |ref|)); <= 0 means every element is within tolerance."""
    return float((np.abs(got - ref) - (atol + rtol * np.abs(ref))).max())


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


@dataclasses.dataclass
class Problem:
    cfg: mi.MLAConfig
    lengths: np.ndarray
    tables: np.ndarray  # int32 [B, max_blocks] pool block of each tile of each sequence
    cache: torch.Tensor
    block_table: torch.Tensor
    kv_len: torch.Tensor
    q_nope: torch.Tensor
    q_rope: torch.Tensor
    q_pos: torch.Tensor
    W_UK: torch.Tensor
    W_UV: torch.Tensor
    rope_tab: torch.Tensor
    status: torch.Tensor

    @property
    def T(self):
        return self.cfg.T

    def absorb(self) -> torch.Tensor:
        return mla.absorb_q(self.q_nope, self.q_rope, self.q_pos, self.W_UK, self.rope_tab, dev_status=self.status)

    def decode(self, q, num_splits=0, lse=True, path="tc"):
        lse_out = torch.empty((self.T, self.cfg.H), dtype=torch.float32, device=q.device) if lse else None
        fn = mla.decode if path == "tc" else mla.decode_cudacore
        out = fn(q, self.cache, self.block_table, self.kv_len, self.W_UV, self.cfg.n_q, self.cfg.scale,
                 num_splits=num_splits, lse_out=lse_out, dev_status=self.status)
        return out, lse_out

    def oracle(self, b: int, heads=None):
        """fp64 naive oracle on sequence b: out [n_q, H', 128], o_lat, lse."""
        s = mi.sequence(self.cfg, b, self.lengths)
        f = mi.bf16_bits_to_f64
        Wk = mi.weights(self.cfg, "uk")
        Wv = mi.weights(self.cfg, "uv")
        return on.attend_naive(f(s.c_kv), f(s.k_rope), f(s.q_nope), f(s.q_rope), f(Wk), f(Wv),
                               self.cfg.n_q, scale=self.cfg.scale, base=self.cfg.rope_base, heads=heads)


def block_tables(lengths, gap_blocks: int = 0, slack_blocks: int = 2, shuffle_seed=None, extra_cols: int = 0):
    """Block tables of a pool holding every sequence: (tables int32 [B, max_blocks], cap_blocks, unowned blocks).

    Contiguous (default): sequences take consecutive blocks from block 0, ``gap_blocks`` apart, with
    ``slack_blocks`` spare blocks at the end.  Shuffled (``shuffle_seed``): every block of the pool,
    including about one unowned block per sequence, is placed by a seeded random permutation, so the
    blocks of a sequence are scattered and out of order.  ``extra_cols`` adds table columns past the
    longest sequence.  Every entry past a sequence's own blocks names an unowned block.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    nblk = (lengths + BLOCK_TOKENS - 1) // BLOCK_TOKENS
    max_blocks = int(nblk.max()) + extra_cols
    if shuffle_seed is None:
        starts = np.zeros(B, dtype=np.int64)
        if B > 1:
            starts[1:] = np.cumsum(nblk[:-1] + gap_blocks)
        cap = int(starts[-1] + nblk[-1]) + slack_blocks
        owned = np.zeros(cap, dtype=bool)
        tables = np.zeros((B, max_blocks), dtype=np.int32)
        for b in range(B):
            tables[b, :nblk[b]] = starts[b] + np.arange(nblk[b])
            owned[starts[b]:starts[b] + nblk[b]] = True
    else:
        cap = int(nblk.sum()) + B + slack_blocks
        perm = np.random.default_rng(shuffle_seed).permutation(cap).astype(np.int32)
        tables = np.zeros((B, max_blocks), dtype=np.int32)
        owned = np.zeros(cap, dtype=bool)
        k = 0
        for b in range(B):
            tables[b, :nblk[b]] = perm[k:k + nblk[b]]
            owned[perm[k:k + nblk[b]]] = True
            k += int(nblk[b])
    unowned = np.flatnonzero(~owned)
    assert len(unowned) > 0
    for b in range(B):
        n = max_blocks - int(nblk[b])
        tables[b, nblk[b]:] = unowned[np.arange(n) % len(unowned)]
    return tables, cap, unowned


def build_problem(cfg: mi.MLAConfig, lengths=None, slack_blocks: int = 2, dev="cuda",
                  chunk_rows: int = 1 << 16, gap_blocks: int = 0, shuffle_seed=None, extra_cols: int = 0) -> Problem:
    """Fill a paged cache with every sequence's tokens via mla_append_cache.

    Block tables come from ``block_tables`` (contiguous or shuffled).  Every byte not written by an
    append (the tails of last blocks and all unowned blocks) holds the bf16 NaN pattern, so a kernel
    that used a row outside a sequence, or a table entry past a sequence's blocks, would be noticed.
    """
    lengths = mi.kv_lengths(cfg) if lengths is None else np.asarray(lengths, dtype=np.int64)
    pool_starts = mi.seq_starts(lengths)            # rows in the generator's packed pool
    tables, cap_blocks, _ = block_tables(lengths, gap_blocks, slack_blocks, shuffle_seed, extra_cols)
    N = int(lengths.sum())
    cache = torch.full((cap_blocks, BLOCK_BYTES // 2), NAN_BF16, dtype=torch.int16, device=dev).view(torch.uint8)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rope_tab = mla.rope_table(int(lengths.max()), cfg.rope_base, dev)
    table_t = torch.from_numpy(tables).to(dev)
    # per-row (sequence, position) of the whole pool
    seq_of_row = np.repeat(np.arange(cfg.B, dtype=np.int32), lengths)
    pos_of_row = (np.arange(N, dtype=np.int64) - np.repeat(pool_starts, lengths)).astype(np.int32)
    for r0 in range(0, N, chunk_rows):
        n = min(chunk_rows, N - r0)
        c, k = mi.token_rows(cfg, r0, n)
        mla.append_cache(cache, table_t, torch.from_numpy(seq_of_row[r0:r0 + n]).to(dev),
                         torch.from_numpy(pos_of_row[r0:r0 + n]).to(dev), to_dev_bf16(c, dev),
                         to_dev_bf16(k, dev), rope_tab, status)
    qn, qr = mi.queries(cfg)
    q_pos = np.concatenate([lengths[b] - cfg.n_q + np.arange(cfg.n_q) for b in range(cfg.B)]).astype(np.int32)
    return Problem(cfg, lengths, tables, cache, table_t,
                   torch.from_numpy(lengths.astype(np.int32)).to(dev),
                   to_dev_bf16(qn, dev), to_dev_bf16(qr, dev), torch.from_numpy(q_pos).to(dev),
                   to_dev_bf16(mi.weights(cfg, "uk"), dev), to_dev_bf16(mi.weights(cfg, "uv"), dev),
                   rope_tab, status)
