"""The C-ABI library on the CPU: it loads, exports every declared symbol, its
host-side table matches the oracle's bit for bit, and host validation rejects
bad arguments before any CUDA call (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def mla():
    import mla_latent_kv_34_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(mla):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(mla.lib, n), n
    assert set(names) == set(mla.EXPORTED)
    assert mla.lib.mla_abi_version() == 2


def test_rope_table_matches_oracle_bitwise(mla):
    from oracle.append import rope_table_f32
    n = 3000
    host = np.empty((n, 64), dtype=np.float32)
    assert mla.lib.mla_rope_table_fill(host.ctypes.data_as(ctypes.c_void_p), n, 10000.0) == 0
    pos = list(range(0, n, 7)) + [n - 1]
    c, s = rope_table_f32(pos)
    np.testing.assert_array_equal(host[pos][:, 0::2], c)
    np.testing.assert_array_equal(host[pos][:, 1::2], s)


def test_status_strings(mla):
    assert mla.lib.mla_status_string(0) == b"ok"
    assert b"workspace" in mla.lib.mla_status_string(4)
    assert b"kv_len" in mla.lib.mla_device_status_string(4)
    assert mla.lib.mla_device_status_string(0) == b"ok"


def test_host_validation_rejects_bad_arguments(mla):
    L = mla.lib
    fake = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
    odd = ctypes.c_void_p(4098)
    # decode: null q, unsupported H / n_q / splits, bad scale, small workspace, bad pool / table sizes
    def dec(q=fake, cap=10, mb=4, B=1, n_q=1, H=16, scale=0.07, splits=0, ws_bytes=1 << 30):
        return L.mla_decode(q, fake, cap, fake, mb, fake, fake, B, n_q, H, scale, splits, fake, ws_bytes, fake, None,
                            None, None)
    assert dec(q=None) == 1
    assert dec(H=129) == 2
    assert dec(n_q=0) == 2
    assert dec(n_q=257) == 2
    assert dec(splits=300) == 2
    assert dec(scale=-1.0) == 1
    assert dec(q=odd) == 1
    assert dec(cap=0) == 1
    assert dec(mb=0) == 1
    assert dec(cap=1 << 31) == 1
    need = L.mla_decode_workspace_bytes(4, 2, 128, 3)
    assert need > 0
    assert dec(B=4, n_q=2, H=128, splits=3, ws_bytes=need - 1) == 4
    # empty batch is a no-op
    assert L.mla_decode(None, None, 0, None, 0, None, None, 0, 1, 16, 0.07, 0, None, 0, None, None, None, None) == 0
    # the two phases validate the same way
    assert L.mla_decode_attend(fake, fake, 10, fake, 0, fake, 1, 1, 16, 0.07, 0, fake, 1 << 30, None, None) == 1
    assert L.mla_decode_finish(fake, 0, fake, 1, 1, 16, 0, fake, 1 << 30, fake, None, None, None) == 1
    assert L.mla_decode_finish(None, 4, fake, 1, 1, 16, 0, fake, 1 << 30, fake, None, None, None) == 1
    # absorb / append / combine
    assert L.mla_absorb_q(fake, fake, None, fake, None, 0, 4, 0, fake, None, None) == 2
    assert L.mla_absorb_q(None, fake, None, fake, None, 0, 4, 16, fake, None, None) == 1
    assert L.mla_absorb_q(None, None, None, None, None, 0, 0, 16, None, None, None) == 0
    assert L.mla_append_cache(fake, 10, fake, 2, 4, fake, fake, fake, fake, None, 5, 3, None, None) == 1
    assert L.mla_append_cache(fake, -1, fake, 2, 4, fake, fake, fake, fake, fake, 5, 3, None, None) == 1
    assert L.mla_append_cache(fake, 10, fake, 2, 0, fake, fake, fake, fake, fake, 5, 3, None, None) == 1
    assert L.mla_append_cache(fake, 10, fake, 0, 4, fake, fake, fake, fake, fake, 5, 3, None, None) == 1
    assert L.mla_append_cache(fake, 10, None, 2, 4, fake, fake, fake, fake, fake, 5, 3, None, None) == 1
    assert L.mla_append_cache(None, 0, None, 0, 0, None, None, None, None, None, 0, 0, None, None) == 0
    assert L.mla_splitkv_combine(fake, fake, 4, 16, 0, None, fake, None, None) == 2
    assert L.mla_splitkv_combine(None, fake, 4, 16, 2, None, fake, None, None) == 1
    # naive prefill: empty chunk, chunk longer than the sequence, no heads, no block row, small workspace
    def pre(n=5, L=300, H=16, rope_len=1000, cap=4, blocks=fake, ws_bytes=1 << 30, scale=0.07):
        return L_.mla_prefill_naive(fake, fake, fake, rope_len, fake, cap, blocks, L, n, fake, fake, H, scale, fake,
                                    ws_bytes, fake, None, None, None)
    L_ = L
    assert L.mla_prefill_naive(None, None, None, 0, None, 0, None, 10, 0, None, None, 16, 0.07, None, 0, None, None,
                               None, None) == 0
    assert pre(n=11, L=10) == 1
    assert pre(H=0) == 2
    assert pre(L=2000) == 1          # past the RoPE table
    assert pre(blocks=None) == 1
    assert pre(cap=0) == 1
    assert pre(scale=0.0) == 1
    assert pre(ws_bytes=100) == 4
    assert L.mla_prefill_workspace_bytes(300, 16) == 2 * 300 * 16 * 128 * 2
    # fused query side: empty, bad d_cq, bad H, null W^UK, rope table missing with positions
    assert L.mla_query_absorb(None, None, None, None, None, None, 0, 0, 16, 1536, None, None, None) == 0
    assert L.mla_query_absorb(fake, fake, fake, fake, None, None, 0, 4, 16, 100, fake, None, None) == 2
    assert L.mla_query_absorb(fake, fake, fake, fake, None, None, 0, 4, 129, 1536, fake, None, None) == 2
    assert L.mla_query_absorb(fake, fake, fake, None, None, None, 0, 4, 16, 1536, fake, None, None) == 1
    assert L.mla_query_absorb(fake, fake, fake, fake, fake, None, 0, 4, 16, 1536, fake, None, None) == 1
    # query up-projection: empty, d_cq not a multiple of 64, no heads, null input
    assert L.mla_query_up(None, None, None, 0, 16, 1536, None, None, None, None) == 0
    assert L.mla_query_up(fake, fake, fake, 4, 16, 100, fake, fake, None, None) == 2
    assert L.mla_query_up(fake, fake, fake, 4, 0, 1536, fake, fake, None, None) == 2
    assert L.mla_query_up(fake, fake, fake, -1, 16, 1536, fake, fake, None, None) == 1
    assert L.mla_query_up(None, fake, fake, 4, 16, 1536, fake, fake, None, None) == 1


def test_workspace_sizes(mla):
    # tensor-core path: one slot per (sequence + work unit) and row group, any split count, plus the merged
    # latent output (bf16, rows rounded up to a multiple of 16).  Work units: CTA pairs (at most 74 / G per
    # group; 128 rows per slot), or with at most 32 query rows the one-SM kernel's CTAs (at most 148, one
    # group; 32 rows per slot)
    a = mla.decode_workspace_bytes(32, 1, 128, 1)
    assert a == mla.decode_workspace_bytes(32, 1, 128, 0) > 32 * 128 * 512 * 4
    assert mla.decode_workspace_bytes(32, 2, 128, 0) > a  # two row groups, 37 pairs each (exact sizes below)
    for B, n_q, H in [(32, 1, 128), (128, 2, 128), (1, 1, 16), (70, 1, 3), (1, 256, 128), (3, 100, 16),
                      (64, 1, 16), (5, 2, 16), (5, 3, 11), (2, 1, 33)]:
        G = (n_q * H + 127) // 128
        units = 148 if n_q * H <= 32 else max(1, 74 // G)
        rs = 32 if n_q * H <= 32 else 128  # rows per slot
        rows = G * (B + units) * rs
        T = B * n_q
        olat_rows = (T + 15) // 16 * 16
        head = -(-rows * 8 // 1024) * 1024
        want = -(-(head + rows * 512 * 4) // 1024) * 1024 + H * olat_rows * 1024
        assert mla.decode_workspace_bytes(B, n_q, H, 0) == want, (B, n_q, H)
        assert want >= rows * (8 + 512 * 4)
    # CUDA-core path: one fp32 partial per split
    c1 = mla.lib.mla_decode_cudacore_workspace_bytes(32, 1, 128, 1)
    c4 = mla.lib.mla_decode_cudacore_workspace_bytes(32, 1, 128, 4)
    assert c4 > 3.9 * c1 > 0
