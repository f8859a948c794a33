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
    starts: np.ndarray
    cache: torch.Tensor
    seq_start: torch.Tensor
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
        out = fn(q, self.cache, self.seq_start, self.kv_len, self.W_UV, self.cfg.n_q, self.cfg.scale,
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


def build_problem(cfg: mi.MLAConfig, lengths=None, slack_rows: int = 64, dev="cuda",
                  chunk_rows: int = 1 << 16, gap_rows: int = 0) -> Problem:
    """Fill a packed cache with every sequence's tokens via mla_append_cache.

    Sequences sit back to back from row 0 (or ``gap_rows`` apart); the gaps and
    ``slack_rows`` extra rows at the end hold NaN so that a kernel reading past
    a sequence would be noticed.
    """
    lengths = mi.kv_lengths(cfg) if lengths is None else np.asarray(lengths, dtype=np.int64)
    pool_starts = mi.seq_starts(lengths)            # rows in the generator's packed pool
    starts = pool_starts + gap_rows * np.arange(cfg.B, dtype=np.int64)
    N = int(lengths.sum())
    cap = N + gap_rows * cfg.B + slack_rows
    cache = torch.full((cap, mi.D_ROW), NAN_BF16, dtype=torch.int16, device=dev)
    cache = cache.view(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rope_tab = mla.rope_table(int(lengths.max()), cfg.rope_base, dev)
    seq_start = torch.from_numpy(starts).to(dev)
    # per-row (sequence, position) of the whole pool
    seq_of_row = np.repeat(np.arange(cfg.B, dtype=np.int32), lengths)
    pos_of_row = (np.arange(N, dtype=np.int64) - np.repeat(pool_starts, lengths)).astype(np.int32)
    for r0 in range(0, N, chunk_rows):
        n = min(chunk_rows, N - r0)
        c, k = mi.token_rows(cfg, r0, n)
        mla.append_cache(cache, seq_start, torch.from_numpy(seq_of_row[r0:r0 + n]).to(dev),
                         torch.from_numpy(pos_of_row[r0:r0 + n]).to(dev), to_dev_bf16(c, dev),
                         to_dev_bf16(k, dev), rope_tab, status)
    qn, qr = mi.queries(cfg)
    q_pos = np.concatenate([lengths[b] - cfg.n_q + np.arange(cfg.n_q) for b in range(cfg.B)]).astype(np.int32)
    return Problem(cfg, lengths, starts, cache, seq_start,
                   torch.from_numpy(lengths.astype(np.int32)).to(dev),
                   to_dev_bf16(qn, dev), to_dev_bf16(qr, dev), torch.from_numpy(q_pos).to(dev),
                   to_dev_bf16(mi.weights(cfg, "uk"), dev), to_dev_bf16(mi.weights(cfg, "uv"), dev),
                   rope_tab, status)
