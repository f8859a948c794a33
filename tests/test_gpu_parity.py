"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Tolerance (stated for the decode output): |gpu - ref| <= 1e-2 + 1e-2 |ref| per
element, with bf16 inputs and fp32 accumulation; in addition the relative L2
error over the compared block must stay below 1e-2 and lse within 2e-2
(absolute, natural-log units).  The append is compared bit for bit.
"""

import math

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import append as oapp
from oracle import naive as on

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 1e-2


@pytest.fixture(scope="module")
def H():
    import gpu_harness
    return gpu_harness


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_decode(prob, out, lse, seqs, heads=None, label=""):
    from gpu_harness import rel_l2, tol_excess
    cfg = prob.cfg
    got_all = out.float().cpu().numpy().reshape(cfg.B, cfg.n_q, cfg.H, mi.D_H)
    lse_all = lse.cpu().numpy().reshape(cfg.B, cfg.n_q, cfg.H)
    hs = list(range(cfg.H)) if heads is None else list(heads)
    for b in seqs:
        ref, _, ref_lse = prob.oracle(b, heads=hs)
        got = got_all[b][:, hs]
        ex = tol_excess(got, ref, ATOL, RTOL)
        assert ex <= 0, f"{label} seq {b} (L={prob.lengths[b]}): tolerance exceeded by {ex:.3e}"
        assert rel_l2(got, ref) < 1e-2, f"{label} seq {b}: rel L2 {rel_l2(got, ref):.3e}"
        assert np.abs(lse_all[b][:, hs] - ref_lse).max() < 2e-2, f"{label} seq {b}: lse"
        assert np.all(np.isfinite(got))


# ----------------------------------------------------------------- append

def test_append_bit_exact_with_canary(cuda_ok, H):
    """Appended rows equal the fp32 emulation bit for bit, in the pool blocks a shuffled block table names;
    no other byte changes."""
    dev = "cuda"
    import mla_latent_kv_34_b200 as mla
    cap_blocks = 80
    canary = np.full((cap_blocks, H.BLOCK_BYTES // 2), 0xA5A5, dtype=np.uint16)
    cache = torch.from_numpy(canary.view(np.int16).copy()).to(dev).view(torch.uint8)
    rng = np.random.default_rng(1)
    # 4 sequences x 8 blocks scattered over the 80-block pool, in no order
    tables = rng.permutation(cap_blocks)[:32].astype(np.int32).reshape(4, 8)
    T = 777
    seq_idx = rng.integers(0, 4, T).astype(np.int32)
    # distinct positions per sequence so no row is written twice
    pos = np.empty(T, dtype=np.int32)
    for s in range(4):
        idx = np.where(seq_idx == s)[0]
        pos[idx] = rng.choice(1000, len(idx), replace=False)
    c = mi.normal_bf16(77, 1, 0, T * 512).reshape(T, 512)
    k = mi.normal_bf16(77, 2, 0, T * 64).reshape(T, 64)
    tab = mla.rope_table(1000, 10000.0, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.append_cache(cache, torch.from_numpy(tables).to(dev), torch.from_numpy(seq_idx).to(dev),
                     torch.from_numpy(pos).to(dev), H.to_dev_bf16(c, dev), H.to_dev_bf16(k, dev), tab, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # logical rows from the oracle's fp32 emulation, placed per the documented block layout
    rows = np.concatenate([c, oapp.rotate_k_bits(k, pos)], axis=1)
    expect = canary.copy()
    blk = tables[seq_idx, pos // H.BLOCK_TOKENS]
    H.pack_rows(expect, blk, pos % H.BLOCK_TOKENS, rows)
    got = H.cache_u16(cache)
    np.testing.assert_array_equal(H.unpack_rows(got, blk, pos % H.BLOCK_TOKENS), rows)
    np.testing.assert_array_equal(got, expect)


def test_append_large_positions_bit_exact(cuda_ok, H):
    import mla_latent_kv_34_b200 as mla
    dev = "cuda"
    T = 512
    pos = (131071 - 255 * (T - 1 - np.arange(T, dtype=np.int64))).astype(np.int32)
    cap_blocks = int(pos.max()) // H.BLOCK_TOKENS + 1
    cache = mla.new_cache(cap_blocks, dev)
    c = mi.normal_bf16(78, 1, 0, T * 512).reshape(T, 512)
    k = mi.normal_bf16(78, 2, 0, T * 64).reshape(T, 64)
    tab = mla.rope_table(131072, 10000.0, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    table = torch.arange(cap_blocks, dtype=torch.int32, device=dev).flip(0).reshape(1, cap_blocks)
    mla.append_cache(cache, table, torch.zeros(T, dtype=torch.int32, device=dev),
                     torch.from_numpy(pos).to(dev), H.to_dev_bf16(c, dev), H.to_dev_bf16(k, dev), tab, st)
    blk = cap_blocks - 1 - pos // H.BLOCK_TOKENS
    got = H.unpack_rows(H.cache_u16(cache), blk, pos % H.BLOCK_TOKENS)
    np.testing.assert_array_equal(got[:, :512], c)
    np.testing.assert_array_equal(got[:, 512:], oapp.rotate_k_bits(k, pos))
    assert int(st.item()) == 0


def test_append_out_of_range_is_reported_and_skipped(cuda_ok, H):
    import mla_latent_kv_34_b200 as mla
    dev = "cuda"
    cache = torch.zeros((3, H.BLOCK_BYTES), dtype=torch.uint8, device=dev)
    tab = mla.rope_table(256, 10000.0, dev)
    c = torch.ones((3, 512), dtype=torch.bfloat16, device=dev)
    k = torch.ones((3, 64), dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    # table rows of 2 blocks; sequence 1's second entry (block 7) is outside the 3-block pool, and
    # position 300 of sequence 0 is past its row (300 // 128 = 2)
    table = torch.tensor([[0, 1], [2, 7]], dtype=torch.int32, device=dev)
    mla.append_cache(cache, table, torch.tensor([0, 1, 0], dtype=torch.int32, device=dev),
                     torch.tensor([3, 140, 300], dtype=torch.int32, device=dev), c, k, tab, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0x1
    # a sequence index outside the table's rows is reported, and its row is never read
    mla.append_cache(cache, table, torch.tensor([2, -1], dtype=torch.int32, device=dev),
                     torch.tensor([0, 0], dtype=torch.int32, device=dev), c[:2], k[:2], tab, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0x1
    u = H.cache_u16(cache)
    assert np.any(H.unpack_rows(u, [0], [3]) != 0)
    assert np.all(u[1:] == 0)
    st.zero_()
    mla.append_cache(cache, table, torch.tensor([0], dtype=torch.int32, device=dev),
                     torch.tensor([9], dtype=torch.int32, device=dev), c[:1], k[:1], tab[:5], st)
    torch.cuda.synchronize()
    assert int(st.item()) & 0x2


# ----------------------------------------------------------------- absorb

@pytest.mark.parametrize("T,Hh", [(1, 16), (37, 16), (32, 128), (256, 128), (5, 3)])
def test_absorb_q_matches_oracle(cuda_ok, H, T, Hh):
    import mla_latent_kv_34_b200 as mla
    dev = "cuda"
    cfg = mi.MLAConfig("absorb", B=T, H=Hh, n_q=1, L=10, seed=900 + T)
    qn, qr = mi.queries(cfg)
    Wk = mi.weights(cfg, "uk")
    pos = ((np.arange(T) * 7919) % 131072).astype(np.int32)
    tab = mla.rope_table(131072, 10000.0, dev)
    q = mla.absorb_q(H.to_dev_bf16(qn, dev), H.to_dev_bf16(qr, dev), torch.from_numpy(pos).to(dev),
                     H.to_dev_bf16(Wk, dev), tab)
    got = q.float().cpu().numpy()
    f = mi.bf16_bits_to_f64
    ref_abs = on.absorb_query(f(qn), f(Wk))
    ref_pe = on.rope(f(qr), pos[:, None])
    # one bf16 rounding of an fp32-accumulated value: relative 2^-8 plus tiny absolute
    assert np.all(np.abs(got[..., :512] - ref_abs) <= 1e-3 + 2 ** -8 * np.abs(ref_abs))
    assert np.all(np.abs(got[..., 512:] - ref_pe) <= 1e-6 + 2 ** -7 * np.abs(ref_pe))
    # rope part is bit-identical to the append arithmetic
    exp_bits = oapp.rotate_k_bits(qr.reshape(-1, 64), np.repeat(pos, Hh)).reshape(T, Hh, 64)
    np.testing.assert_array_equal(_bits(q)[..., 512:], exp_bits)
    # pos = NULL copies q^R as given
    q2 = mla.absorb_q(H.to_dev_bf16(qn, dev), H.to_dev_bf16(qr, dev), None, H.to_dev_bf16(Wk, dev), tab)
    np.testing.assert_array_equal(_bits(q2)[..., 512:], qr)


# ----------------------------------------------------------------- decode

def test_decode_tiny_full(cuda_ok, H):
    prob = H.build_problem(mi.CONFIGS["tiny"])
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    _check_decode(prob, out, lse, [0], label="tiny")


@pytest.mark.parametrize("L,n_q,Hh", [(1, 1, 16), (2, 2, 16), (3, 2, 128), (64, 1, 128), (65, 2, 128),
                                      (127, 1, 1), (128, 1, 128), (200, 2, 100), (1000, 1, 64), (129, 2, 64),
                                      (257, 2, 128)])
def test_decode_edge_shapes(cuda_ok, H, L, n_q, Hh):
    cfg = mi.MLAConfig("edge", B=2, H=Hh, n_q=n_q, L=L, seed=1000 + L + Hh)
    prob = H.build_problem(cfg, lengths=[L, max(n_q, L // 2 + 1)])
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    _check_decode(prob, out, lse, [0, 1], label=f"edge L={L}")


@pytest.mark.parametrize("n_q,Hh,L", [(4, 32, 700), (8, 16, 300), (16, 8, 2000), (3, 128, 260), (5, 64, 5)])
def test_decode_multi_token_queries(cuda_ok, H, n_q, Hh, L):
    """n_q > 2 new tokens per sequence (multi-token / speculative decode): query j sees keys up to
    L - n_q + j; rows of several query tokens share one 128-row group (or span groups)."""
    cfg = mi.MLAConfig("multi", B=3, H=Hh, n_q=n_q, L=L, seed=2000 + 17 * n_q + Hh)
    prob = H.build_problem(cfg, lengths=[L, max(n_q, L // 3), max(n_q, L - 1)])
    q = prob.absorb()
    out, lse = prob.decode(q)
    ref_out, ref_lse = prob.decode(q, num_splits=3, path="cudacore")
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
    # With a handful of keys the output is a short weighted sum of large W^UV c rows, so the two
    # paths' independent bf16 rounding of P shows at ~1e-2 absolute; each path is held to the
    # parity bar against the oracle below, so their difference is bounded by twice that bar.
    assert np.all(np.abs(a - b) <= 2 * (ATOL + RTOL * np.abs(b)))
    _check_decode(prob, out, lse, [0, 1, 2], label=f"n_q={n_q}")


@pytest.mark.parametrize("n_q,Hh,L", [(32, 16, 600), (100, 8, 400), (256, 16, 700), (64, 128, 300),
                                      (150, 4, 500)])
def test_decode_prefill_chunks(cuda_ok, H, n_q, Hh, L):
    """Chunks of up to 256 new tokens per sequence in the absorbed form (the arithmetic favours it
    over the naive form below about 340 tokens); query j sees keys up to L - n_q + j.  T = 2 n_q query
    rows: 300 rows span two 256-row blocks of the merged latent output, the second a partial one."""
    cfg = mi.MLAConfig("chunk", B=2, H=Hh, n_q=n_q, L=L, seed=3000 + n_q + Hh)
    prob = H.build_problem(cfg, lengths=[L, max(n_q, L // 2)], shuffle_seed=n_q)
    q = prob.absorb()
    out, lse = prob.decode(q)
    ref_out, _ = prob.decode(q, num_splits=2, path="cudacore")
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2 * (ATOL + RTOL * np.abs(b)))
    _check_decode(prob, out, lse, [0, 1], heads=range(0, Hh, max(1, Hh // 8)), label=f"chunk n_q={n_q}")


def test_decode_small_ragged_full(cuda_ok, H):
    cfg = mi.MLAConfig("ragged-small", B=12, H=128, n_q=2, L=None, L_max=700, seed=77)
    prob = H.build_problem(cfg)
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    _check_decode(prob, out, lse, range(cfg.B), heads=range(0, 128, 5), label="ragged-small")


@pytest.mark.parametrize("splits", [1, 2, 7, 32])
def test_decode_split_invariance(cuda_ok, H, splits):
    """Tensor-core path with at most `splits` CTA pairs per row group (so sequences
    are cut into 1 .. many pieces) against the CUDA-core path and the oracle."""
    cfg = mi.MLAConfig("splits", B=3, H=32, n_q=2, L=None, L_max=3000, seed=55)
    prob = H.build_problem(cfg)
    q = prob.absorb()
    ref_out, ref_lse = prob.decode(q, num_splits=4, path="cudacore")
    out, lse = prob.decode(q, num_splits=splits)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
    # same math up to summation order and the bf16 rounding of P
    assert np.all(np.abs(a - b) <= 2e-3 + 2 ** -6 * np.abs(b))
    assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() < 1e-3
    _check_decode(prob, out, lse, [0, 2], label=f"splits={splits}")


@pytest.mark.parametrize("B,Hh,n_q,L_max,splits,shuffle", [(7, 16, 2, 1500, 0, 3), (3, 4, 1, 700, 0, None),
                                                          (5, 11, 2, 2000, 3, 5), (1, 1, 1, 5, 0, None),
                                                          (40, 16, 1, 600, 1, 7), (6, 32, 1, 2600, 0, 9),
                                                          (4, 16, 2, 300, 200, None), (20, 16, 1, 900, 0, 11),
                                                          (100, 8, 2, 400, 0, 13)])
def test_decode_few_rows_one_sm_kernel(cuda_ok, H, B, Hh, n_q, L_max, splits, shuffle):
    """At most 32 query rows (n_q * H): the one-SM kernel (tokens as the MMA's M side, both contractions on
    one SM), with shuffled block tables and NaN canaries in unowned blocks, against the CUDA-core path and
    the oracle; one work unit per SM down to a single one, and more units than tiles.  The batch sizes
    also take the merge through 1, 2, 8 and 16 threads per row."""
    cfg = mi.MLAConfig("one-sm", B=B, H=Hh, n_q=n_q, L=None, L_max=L_max, seed=700 + B + Hh + n_q)
    prob = H.build_problem(cfg, shuffle_seed=shuffle)
    q = prob.absorb()
    ref_out, ref_lse = prob.decode(q, num_splits=3, path="cudacore")
    out, lse = prob.decode(q, num_splits=splits)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    assert torch.isfinite(out.float()).all()
    a, b = out.float().cpu().numpy(), ref_out.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2 * (ATOL + RTOL * np.abs(b)))
    assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() < 2e-2
    _check_decode(prob, out, lse, range(min(B, 6)), label=f"one-sm B={B} H={Hh} n_q={n_q}")


def test_decode_ignores_rows_outside_sequences(cuda_ok, H):
    """NaN rows between and after sequences never leak into any result."""
    cfg = mi.MLAConfig("gaps", B=5, H=128, n_q=2, L=None, L_max=400, seed=66)
    prob = H.build_problem(cfg, gap_blocks=3)
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    assert torch.isfinite(out.float()).all()
    _check_decode(prob, out, lse, range(cfg.B), heads=range(0, 128, 7), label="gaps")


def test_decode_tensor_core_matches_cuda_core_path(cuda_ok, H):
    cfg = mi.MLAConfig("paths", B=6, H=128, n_q=1, L=None, L_max=5000, seed=91)
    prob = H.build_problem(cfg)
    q = prob.absorb()
    out_c, lse_c = prob.decode(q, path="cudacore")
    out_t, lse_t = prob.decode(q)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    a, b = out_t.float().cpu().numpy(), out_c.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2e-3 + 2 ** -6 * np.abs(b))
    assert np.abs(lse_t.cpu().numpy() - lse_c.cpu().numpy()).max() < 1e-3


@pytest.mark.parametrize("name,seqs,heads", [
    ("v2lite", [0, 63], None),
    ("v2", [0, 31], range(0, 128, 9)),
    ("128k", [3], range(0, 128, 31)),
])
def test_decode_full_size_sampled(cuda_ok, H, name, seqs, heads):
    cfg = mi.CONFIGS[name]
    prob = H.build_problem(cfg)
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    _check_decode(prob, out, lse, seqs, heads=heads, label=name)
    # every row finite, lse >= log(1)
    assert torch.isfinite(out.float()).all()


def test_decode_ragged_full_size_sampled(cuda_ok, H):
    cfg = mi.CONFIGS["ragged"]
    prob = H.build_problem(cfg)
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    L = prob.lengths
    pick = sorted({int(np.argmin(L)), int(np.argmax(L)), 0, 77})
    _check_decode(prob, out, lse, pick, heads=range(0, 128, 16), label="ragged")
    assert torch.isfinite(out.float()).all()


def test_decode_reports_short_kv_len(cuda_ok, H):
    cfg = mi.MLAConfig("short", B=2, H=16, n_q=2, L=10, seed=3)
    prob = H.build_problem(cfg)
    prob.kv_len[1] = 1
    prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) & 0x4


# ----------------------------------------------------------------- paged cache

def test_decode_paged_shuffled_tables_match_contiguous_and_oracle(cuda_ok, H):
    """Sequences whose blocks are scattered over the pool in random order, with table entries past each
    sequence's blocks naming NaN-filled unowned blocks: the same results, bit for bit, as the contiguous
    layout (the kernels compute tile by tile, wherever the tile lives) and within the bar of the oracle."""
    cfg = mi.MLAConfig("paged", B=9, H=128, n_q=2, L=None, L_max=1300, seed=4242)
    flat = H.build_problem(cfg)
    paged = H.build_problem(cfg, shuffle_seed=7, extra_cols=3)
    assert not np.array_equal(paged.tables[:, 0], flat.tables[:, 0])
    q = flat.absorb()
    out_f, lse_f = flat.decode(q)
    out_p, lse_p = paged.decode(q)
    torch.cuda.synchronize()
    assert int(flat.status.item()) == 0 and int(paged.status.item()) == 0
    assert torch.equal(out_f, out_p) and torch.equal(lse_f, lse_p)
    _check_decode(paged, out_p, lse_p, range(cfg.B), heads=range(0, 128, 11), label="paged")
    out_c, _ = paged.decode(q, num_splits=2, path="cudacore")
    torch.cuda.synchronize()
    assert int(paged.status.item()) == 0
    a, b = out_p.float().cpu().numpy(), out_c.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2e-3 + 2 ** -6 * np.abs(b))


def test_decode_paged_v2_time_shape_sampled(cuda_ok, H):
    """V2-shaped workload on a shuffled pool (512 blocks of 32 sequences in random order)."""
    cfg = mi.CONFIGS["v2"]
    prob = H.build_problem(cfg, shuffle_seed=11)
    out, lse = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    _check_decode(prob, out, lse, [5, 30], heads=range(3, 128, 25), label="v2 paged")


def test_decode_table_overflow_and_bad_entry_are_reported(cuda_ok, H):
    """A sequence longer than its table row is not processed (zero rows, lse -inf, ROW_RANGE); the others
    are unaffected.  A table entry outside the pool is reported and never dereferenced."""
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("overflow", B=3, H=16, n_q=1, L=None, L_max=600, seed=8)
    prob = H.build_problem(cfg, lengths=[300, 200, 130])
    q = prob.absorb()
    kv = prob.kv_len.clone()
    kv[1] = 3 * 128 + 1  # needs 4 blocks; the rows hold 3
    lse = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    out = mla.decode(q, prob.cache, prob.block_table, kv, prob.W_UV, cfg.n_q, cfg.scale, lse_out=lse,
                     dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0x1
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    _check_decode(prob, out, lse, [0, 2], label="overflow")
    prob.status.zero_()
    bad = prob.block_table.clone()
    bad[2, 1] = prob.cache.shape[0] + 5
    mla.decode(q, prob.cache, bad, prob.kv_len, prob.W_UV, cfg.n_q, cfg.scale, lse_out=lse, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0x1


# ----------------------------------------------------------------- combine

@pytest.mark.parametrize("with_wuv", [False, True])
def test_splitkv_combine_matches_oracle_merge(cuda_ok, H, with_wuv):
    import mla_latent_kv_34_b200 as mla
    dev = "cuda"
    T, Hh, S = 5, 8, 6
    rng = np.random.default_rng(4)
    o = rng.standard_normal((T, Hh, S, 512)).astype(np.float32)
    lse = (rng.standard_normal((T, Hh, S)) * 3).astype(np.float32)
    lse[0, 0, :] = -np.inf
    lse[0, 0, 2] = 1.5          # one live split
    lse[1, 1, 3:] = -np.inf     # empty splits
    Wv = mi.normal_bf16(9, 6, 0, Hh * 128 * 512, 1 / math.sqrt(512)).reshape(Hh, 128, 512)
    lse_out = torch.empty((T, Hh), dtype=torch.float32, device=dev)
    out = mla.splitkv_combine(torch.from_numpy(o).to(dev), torch.from_numpy(lse).to(dev),
                              W_UV=H.to_dev_bf16(Wv, dev) if with_wuv else None, lse_out=lse_out)
    ref_o, ref_lse = on.merge_partials(np.moveaxis(o, 2, 0).astype(np.float64), np.moveaxis(lse, 2, 0))
    np.testing.assert_allclose(lse_out.cpu().numpy(), ref_lse, rtol=1e-5, atol=1e-5)
    if with_wuv:
        ref = on.up_project(ref_o, mi.bf16_bits_to_f64(Wv))
        got = out.float().cpu().numpy()
        assert np.all(np.abs(got - ref) <= 1e-3 + 2 ** -7 * np.abs(ref))
    else:
        np.testing.assert_allclose(out.cpu().numpy(), ref_o, rtol=1e-5, atol=1e-6)
