"""Python binding of libmla_b200 (MLA weight-absorbed decode on B200).

Argument marshalling only: every function checks dtypes/shapes/devices of
torch tensors and calls the C ABI of ``include/mla.h`` with raw device
pointers and the current CUDA stream.  All arithmetic runs in the library's
CUDA kernels; there is no fallback of any kind.  Importing this module fails
loudly if the shared library has not been built
(``python mla_latent_kv_34_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os

import torch

D_C, D_R, D_H = 512, 64, 128
D_ROW = D_C + D_R
BLOCK_TOKENS = 128      # tokens per cache block
BLOCK_BYTES = 147456    # 9 chunks x [128 rows x 128 bytes]

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python mla_latent_kv_34_b200/build.py`")
lib = ctypes.CDLL(_LIB_PATH)

_p = ctypes.c_void_p
_i32, _i64, _f32, _f64, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_size_t

_SIGS = {
    "mla_abi_version": ([], _i32),
    "mla_status_string": ([_i32], ctypes.c_char_p),
    "mla_device_status_string": ([ctypes.c_int32], ctypes.c_char_p),
    "mla_rope_table_fill": ([_p, _i64, _f64], _i32),
    "mla_absorb_q": ([_p, _p, _p, _p, _p, _i64, _i32, _i32, _p, _p, _p], _i32),
    "mla_query_up": ([_p, _p, _p, _i32, _i32, _i32, _p, _p, _p, _p], _i32),
    "mla_query_absorb": ([_p, _p, _p, _p, _p, _p, _i64, _i32, _i32, _i32, _p, _p, _p], _i32),
    "mla_append_cache": ([_p, _i64, _p, _i32, _i32, _p, _p, _p, _p, _p, _i64, _i32, _p, _p], _i32),
    "mla_decode_workspace_bytes": ([_i32, _i32, _i32, _i32], _sz),
    "mla_decode": ([_p, _p, _i64, _p, _i32, _p, _p, _i32, _i32, _i32, _f32, _i32, _p, _sz, _p, _p, _p, _p], _i32),
    "mla_decode_attend": ([_p, _p, _i64, _p, _i32, _p, _i32, _i32, _i32, _f32, _i32, _p, _sz, _p, _p], _i32),
    "mla_decode_finish": ([_p, _i32, _p, _i32, _i32, _i32, _i32, _p, _sz, _p, _p, _p, _p], _i32),
    "mla_decode_static": ([_p, _p, _i64, _p, _i32, _p, _p, _i32, _i32, _i32, _f32, _i32, _p, _p, _p, _p], _i32),
    "mla_decode_cudacore_workspace_bytes": ([_i32, _i32, _i32, _i32], _sz),
    "mla_decode_cudacore": ([_p, _p, _i64, _p, _i32, _p, _p, _i32, _i32, _i32, _f32, _i32, _p, _sz, _p, _p, _p,
                             _p], _i32),
    "mla_splitkv_combine": ([_p, _p, _i32, _i32, _i32, _p, _p, _p, _p], _i32),
    "mla_prefill_workspace_bytes": ([_i32, _i32], _sz),
    "mla_prefill_naive": ([_p, _p, _p, _i64, _p, _i64, _p, _i32, _i32, _p, _p, _i32, _f32, _p, _sz, _p, _p, _p, _p],
                          _i32),
}
for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _ret

EXPORTED = tuple(_SIGS)


class MLAError(RuntimeError):
    pass


def _check(status: int) -> None:
    if status != 0:
        raise MLAError(f"mla status {status}: {lib.mla_status_string(status).decode()}")


def device_status_string(word: int) -> str:
    return lib.mla_device_status_string(int(word)).decode()


def _ptr(t: torch.Tensor | None, dtype=None, shape=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise MLAError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise MLAError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise MLAError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise MLAError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def rope_table(rope_len: int, base: float = 10000.0, device="cuda") -> torch.Tensor:
    """fp32 [rope_len, 64] table of (cos, sin) pairs, filled by the library on the host."""
    host = torch.empty((rope_len, D_R), dtype=torch.float32).pin_memory() if rope_len else \
        torch.empty((0, D_R), dtype=torch.float32)
    if rope_len:
        _check(lib.mla_rope_table_fill(host.data_ptr(), rope_len, float(base)))
    return host.to(device, non_blocking=False)


def absorb_q(q_nope, q_rope, pos, W_UK, rope_tab, q_out=None, dev_status=None, stream=None):
    """q_out[t, h] = [(W^UK_h)^T q_nope[t, h] | R_pos[t] q_rope[t, h]]  -> bf16 [T, H, 576]."""
    T, H = q_nope.shape[0], q_nope.shape[1]
    if q_out is None:
        q_out = torch.empty((T, H, D_ROW), dtype=torch.bfloat16, device=q_nope.device)
    _check(lib.mla_absorb_q(
        _ptr(q_nope, torch.bfloat16, (T, H, D_H), "q_nope"), _ptr(q_rope, torch.bfloat16, (T, H, D_R), "q_rope"),
        _ptr(pos, torch.int32, (T,), "pos"), _ptr(W_UK, torch.bfloat16, (H, D_H, D_C), "W_UK"),
        _ptr(rope_tab, torch.float32, None, "rope_table"), 0 if rope_tab is None else rope_tab.shape[0],
        T, H, _ptr(q_out, torch.bfloat16, (T, H, D_ROW), "q_out"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return q_out


def query_up(c_q, W_UQ, W_QR, q_nope=None, q_rope=None, dev_status=None, stream=None):
    """q^C[t, h] = W^UQ_h c^Q_t -> bf16 [T, H, 128] and q^R[t, h] = W^QR_h c^Q_t -> bf16 [T, H, 64] (not rotated)."""
    T, d_cq = c_q.shape
    H = W_UQ.shape[0]
    if q_nope is None:
        q_nope = torch.empty((T, H, D_H), dtype=torch.bfloat16, device=c_q.device)
    if q_rope is None:
        q_rope = torch.empty((T, H, D_R), dtype=torch.bfloat16, device=c_q.device)
    _check(lib.mla_query_up(
        _ptr(c_q, torch.bfloat16, (T, d_cq), "c_q"), _ptr(W_UQ, torch.bfloat16, (H, D_H, d_cq), "W_UQ"),
        _ptr(W_QR, torch.bfloat16, (H, D_R, d_cq), "W_QR"), T, H, d_cq,
        _ptr(q_nope, torch.bfloat16, (T, H, D_H), "q_nope"), _ptr(q_rope, torch.bfloat16, (T, H, D_R), "q_rope"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return q_nope, q_rope


def query_absorb(c_q, W_UQ, W_QR, W_UK, pos, rope_tab, q_out=None, dev_status=None, stream=None):
    """c^Q [T, d_cq] -> q_out bf16 [T, H, 576] = [(W^UK_h)^T (W^UQ_h c^Q) | R_pos (W^QR_h c^Q)] in one launch."""
    T, d_cq = c_q.shape
    H = W_UQ.shape[0]
    if q_out is None:
        q_out = torch.empty((T, H, D_ROW), dtype=torch.bfloat16, device=c_q.device)
    _check(lib.mla_query_absorb(
        _ptr(c_q, torch.bfloat16, (T, d_cq), "c_q"), _ptr(W_UQ, torch.bfloat16, (H, D_H, d_cq), "W_UQ"),
        _ptr(W_QR, torch.bfloat16, (H, D_R, d_cq), "W_QR"), _ptr(W_UK, torch.bfloat16, (H, D_H, D_C), "W_UK"),
        _ptr(pos, torch.int32, (T,), "pos"), _ptr(rope_tab, torch.float32, None, "rope_table"),
        0 if rope_tab is None else rope_tab.shape[0], T, H, d_cq,
        _ptr(q_out, torch.bfloat16, (T, H, D_ROW), "q_out"), _ptr(dev_status, torch.int32, None, "dev_status"),
        _stream(stream)))
    return q_out


def new_cache(cap_blocks: int, device="cuda") -> torch.Tensor:
    """An empty pool of cache blocks: uint8 [cap_blocks, BLOCK_BYTES] (layout in include/mla.h)."""
    return torch.empty((cap_blocks, BLOCK_BYTES), dtype=torch.uint8, device=device)


def contiguous_block_table(lengths, max_blocks: int | None = None, first_block: int = 0, gap_blocks: int = 0,
                           device="cuda") -> torch.Tensor:
    """int32 [B, max_blocks] table giving each sequence consecutive pool blocks, sequences back to back
    (``gap_blocks`` apart) from ``first_block``; unused entries are -1."""
    import numpy as np
    lengths = np.asarray(lengths, dtype=np.int64)
    nblk = (lengths + BLOCK_TOKENS - 1) // BLOCK_TOKENS
    mb = int(max(1, nblk.max() if len(nblk) else 1)) if max_blocks is None else max_blocks
    tab = np.full((len(lengths), mb), -1, dtype=np.int32)
    start = first_block
    for b, n in enumerate(nblk):
        tab[b, :n] = start + np.arange(n)
        start += int(n) + gap_blocks
    return torch.from_numpy(tab).to(device)


def _cache_ptr(cache):
    if cache.dim() != 2 or cache.shape[1] != BLOCK_BYTES:
        raise MLAError(f"cache must be uint8 [cap_blocks, {BLOCK_BYTES}]")
    return _ptr(cache, torch.uint8, None, "cache")


def _table(block_table, B=None):
    if block_table.dim() != 2 or (B is not None and block_table.shape[0] != B):
        raise MLAError("block_table must be int32 [B, max_blocks]")
    return _ptr(block_table, torch.int32, None, "block_table"), block_table.shape[1]


def append_cache(cache, block_table, seq_idx, pos, c_kv, k_rope, rope_tab, dev_status=None, stream=None):
    """Write c_kv [T,512] and R_pos k_rope [T,64] at token pos of sequence seq_idx
    (pool block block_table[seq_idx, pos // 128], row pos % 128)."""
    T = c_kv.shape[0]
    tp, mb = _table(block_table)
    _check(lib.mla_append_cache(
        _cache_ptr(cache), cache.shape[0], tp, block_table.shape[0], mb,
        _ptr(seq_idx, torch.int32, (T,), "seq_idx"), _ptr(pos, torch.int32, (T,), "pos"),
        _ptr(c_kv, torch.bfloat16, (T, D_C), "c_kv"), _ptr(k_rope, torch.bfloat16, (T, D_R), "k_rope"),
        _ptr(rope_tab, torch.float32, None, "rope_table"), rope_tab.shape[0], T,
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))


def decode_workspace_bytes(B: int, n_q: int, H: int, num_splits: int = 0) -> int:
    return int(lib.mla_decode_workspace_bytes(B, n_q, H, num_splits))


def decode(q, cache, block_table, kv_len, W_UV, n_q: int, scale: float, num_splits: int = 0,
           workspace=None, out=None, lse_out=None, dev_status=None, stream=None):
    """One absorbed decode step: out bf16 [B*n_q, H, 128] (and lse fp32 [B*n_q, H] if given)."""
    B = kv_len.shape[0]
    T, H = q.shape[0], q.shape[1]
    if T != B * n_q:
        raise MLAError("q rows must equal len(kv_len) * n_q")
    need = decode_workspace_bytes(B, n_q, H, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((T, H, D_H), dtype=torch.bfloat16, device=q.device)
    _check(lib.mla_decode(
        _ptr(q, torch.bfloat16, (T, H, D_ROW), "q"), _cache_ptr(cache), cache.shape[0], *_table(block_table, B),
        _ptr(kv_len, torch.int32, (B,), "kv_len"),
        _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), B, n_q, H, float(scale), num_splits,
        _ptr(workspace, None, None, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(out, torch.bfloat16, (T, H, D_H), "out"), _ptr(lse_out, torch.float32, (T, H), "lse_out"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return out


DECODE_STATIC_SCRATCH_BYTES = 32 << 20  # MLA_DECODE_STATIC_SCRATCH_BYTES


def decode_static(q, cache, block_table, kv_len, W_UV, n_q: int, scale: float, num_splits: int = 0,
                  out=None, lse_out=None, dev_status=None, stream=None):
    """``decode`` with the library's own scratch (no workspace; ``out`` must be given to avoid any allocation).

    Calls that can overlap on one device race on that scratch; the first call per device must precede any
    stream capture.
    """
    B = kv_len.shape[0]
    T, H = q.shape[0], q.shape[1]
    if T != B * n_q:
        raise MLAError("q rows must equal len(kv_len) * n_q")
    if out is None:
        out = torch.empty((T, H, D_H), dtype=torch.bfloat16, device=q.device)
    _check(lib.mla_decode_static(
        _ptr(q, torch.bfloat16, (T, H, D_ROW), "q"), _cache_ptr(cache), cache.shape[0], *_table(block_table, B),
        _ptr(kv_len, torch.int32, (B,), "kv_len"),
        _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), B, n_q, H, float(scale), num_splits,
        _ptr(out, torch.bfloat16, (T, H, D_H), "out"), _ptr(lse_out, torch.float32, (T, H), "lse_out"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return out


def decode_attend(q, cache, block_table, kv_len, n_q: int, scale: float, num_splits: int, workspace,
                  dev_status=None, stream=None):
    """Phase 1 of decode: per-piece partials into ``workspace``."""
    B = kv_len.shape[0]
    T, H = q.shape[0], q.shape[1]
    _check(lib.mla_decode_attend(
        _ptr(q, torch.bfloat16, (B * n_q, H, D_ROW), "q"), _cache_ptr(cache),
        cache.shape[0], *_table(block_table, B), _ptr(kv_len, torch.int32, (B,), "kv_len"),
        B, n_q, H, float(scale), num_splits, _ptr(workspace, None, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(dev_status, torch.int32, None, "dev_status"),
        _stream(stream)))


def decode_finish(block_table, kv_len, W_UV, n_q: int, num_splits: int, workspace, out, lse_out=None,
                  dev_status=None, stream=None):
    """Phase 2 of decode: merge the pieces, apply W^UV into ``out`` bf16 [B*n_q, H, 128]."""
    B = kv_len.shape[0]
    H = W_UV.shape[0]
    _check(lib.mla_decode_finish(
        _ptr(kv_len, torch.int32, (B,), "kv_len"), block_table.shape[1],
        _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), B, n_q, H, num_splits,
        _ptr(workspace, None, None, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(out, torch.bfloat16, (B * n_q, H, D_H), "out"), _ptr(lse_out, torch.float32, (B * n_q, H), "lse_out"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return out


def decode_cudacore(q, cache, block_table, kv_len, W_UV, n_q: int, scale: float, num_splits: int = 0,
                    workspace=None, out=None, lse_out=None, dev_status=None, stream=None):
    """The decode step on CUDA cores (second implementation, same results within fp32 rounding)."""
    B = kv_len.shape[0]
    T, H = q.shape[0], q.shape[1]
    if T != B * n_q:
        raise MLAError("q rows must equal len(kv_len) * n_q")
    if workspace is None:
        need = int(lib.mla_decode_cudacore_workspace_bytes(B, n_q, H, num_splits))
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((T, H, D_H), dtype=torch.bfloat16, device=q.device)
    _check(lib.mla_decode_cudacore(
        _ptr(q, torch.bfloat16, (T, H, D_ROW), "q"), _cache_ptr(cache), cache.shape[0], *_table(block_table, B),
        _ptr(kv_len, torch.int32, (B,), "kv_len"),
        _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), B, n_q, H, float(scale), num_splits,
        _ptr(workspace, None, None, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(out, torch.bfloat16, (T, H, D_H), "out"), _ptr(lse_out, torch.float32, (T, H), "lse_out"),
        _ptr(dev_status, torch.int32, None, "dev_status"), _stream(stream)))
    return out


def splitkv_combine(o_part, lse_part, W_UV=None, out=None, lse_out=None, stream=None):
    """Merge split partials o_part fp32 [T,H,S,512], lse_part fp32 [T,H,S]."""
    T, H, S = lse_part.shape
    if out is None:
        out = torch.empty((T, H, D_H) if W_UV is not None else (T, H, D_C),
                          dtype=torch.bfloat16 if W_UV is not None else torch.float32, device=o_part.device)
    _check(lib.mla_splitkv_combine(
        _ptr(o_part, torch.float32, (T, H, S, D_C), "o_part"), _ptr(lse_part, torch.float32, (T, H, S), "lse_part"),
        T, H, S, _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), _ptr(out, None, None, "out"),
        _ptr(lse_out, torch.float32, (T, H), "lse_out"), _stream(stream)))
    return out


def prefill_workspace_bytes(L: int, H: int) -> int:
    return int(lib.mla_prefill_workspace_bytes(L, H))


def prefill_naive(q_nope, q_rope, rope_tab, cache, blocks, L: int, W_UK, W_UV, scale: float,
                  workspace=None, out=None, lse_out=None, dev_status=None, stream=None):
    """Naive-form attention of the last n = len(q_nope) of a sequence's L cached tokens -> bf16 [n, H, 128].

    ``blocks``: int32 device tensor, the sequence's row of the block table (at least ceil(L / 128) entries).
    """
    n, H = q_nope.shape[0], q_nope.shape[1]
    if blocks.dim() != 1 or blocks.shape[0] * BLOCK_TOKENS < L:
        raise MLAError("blocks must be an int32 vector of at least ceil(L / 128) entries")
    need = prefill_workspace_bytes(L, H)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_nope.device)
    if out is None:
        out = torch.empty((n, H, D_H), dtype=torch.bfloat16, device=q_nope.device)
    _check(lib.mla_prefill_naive(
        _ptr(q_nope, torch.bfloat16, (n, H, D_H), "q_nope"), _ptr(q_rope, torch.bfloat16, (n, H, D_R), "q_rope"),
        _ptr(rope_tab, torch.float32, None, "rope_table"), rope_tab.shape[0], _cache_ptr(cache), cache.shape[0],
        _ptr(blocks, torch.int32, None, "blocks"), int(L), n, _ptr(W_UK, torch.bfloat16, (H, D_H, D_C), "W_UK"),
        _ptr(W_UV, torch.bfloat16, (H, D_H, D_C), "W_UV"), H, float(scale), _ptr(workspace, None, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(out, torch.bfloat16, (n, H, D_H), "out"),
        _ptr(lse_out, torch.float32, (n, H), "lse_out"), _ptr(dev_status, torch.int32, None, "dev_status"),
        _stream(stream)))
    return out
