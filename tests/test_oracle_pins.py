"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU)."""

import json
import math
import os

import numpy as np
import pytest

import oracle_pins as pins
from oracle import append as oapp
from oracle import naive as on

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("check", pins.ALL_SINGLE, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(on.attend_naive)


def test_absorbed_equals_naive():
    pins.check_absorbed_identity(on.attend_naive, on.attend_absorbed)


def test_softmax_rows_sum_to_one():
    c, kr, qn, qr, Wk, Wv = pins.rand_problem(40, 3, 2, 7)
    _, _, lse, probs = on.attend_naive(c, kr, qn, qr, Wk, Wv, 2, keep_probs=True)
    for (j, h), P in probs.items():
        assert len(P) == 40 - 2 + j + 1
        assert np.all(P >= 0)
        assert abs(math.fsum(P) - 1.0) < 1e-14


def test_rope_is_a_rotation_with_relative_positions():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in ((0, 0), (3, 11), (1000, 17), (131071, 5)):
        qm, kn = on.rope(q, m), on.rope(k, n)
        assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-12
        # <R_m q, R_n k> = <q, R_{n-m} k>  (S = Q^T R_m^T R_n K)
        assert abs(qm @ kn - q @ on.rope(k, n - m)) < 1e-9
        np.testing.assert_allclose(on.rope(qm, -m), q, atol=1e-9)
    np.testing.assert_array_equal(on.rope(q, 0), q)


def test_splitkv_merge_equals_full():
    L, n_q, H = 50, 2, 2
    c, kr, qn, qr, Wk, Wv = pins.rand_problem(L, H, n_q, 9)
    _, o_full, lse_full = on.attend_naive(c, kr, qn, qr, Wk, Wv, n_q)
    for cuts in ((0, 50), (0, 7, 50), (0, 1, 20, 49, 50), (0, 13, 26, 39, 50)):
        parts = [on.attend_partial_latent(c, kr, qn, qr, Wk, n_q, a, b)
                 for a, b in zip(cuts[:-1], cuts[1:])]
        o, lse = on.merge_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        np.testing.assert_allclose(o, o_full, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, lse_full, rtol=1e-13, atol=1e-13)


def test_up_project_and_absorb_query_shapes():
    c, kr, qn, qr, Wk, Wv = pins.rand_problem(4, 3, 1, 10)
    q_abs = on.absorb_query(qn, Wk)
    for h in range(3):
        np.testing.assert_allclose(q_abs[0, h] @ c[2], qn[0, h] @ (Wk[h] @ c[2]), rtol=1e-12)
        np.testing.assert_allclose(on.up_project(c[None, None, 1].repeat(3, 1), Wv)[0, h],
                                   Wv[h] @ c[1], rtol=1e-12)


def test_cache_footprint_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "cache_footprint.json")))
    d_h = 128
    for kind, row in g["table_per_layer"].items():
        for n in (1, 2, 8, 16, 128):
            vals = {"n_h": n, "n_g": n, "d_h": d_h}
            expect = row["coef"] * math.prod(vals[f] for f in row["factors"])
            got = on.kv_elements_per_token_layer(kind, n_h=n, n_g=n, d_h=d_h,
                                                 d_c=g["d_c_over_d_h"] * d_h,
                                                 d_r=int(g["d_h_R_over_d_h"] * d_h))
            assert got == expect, (kind, n)
    assert on.mla_equivalent_gqa_groups() == g["mla_equivalent_gqa_groups"]
    v = g["v2lite"]
    assert v["d_c"] + v["d_h_R"] == on.kv_elements_per_token_layer("mla") == 576
    # bf16 storage: 1152 bytes per token per layer
    assert 2 * on.kv_elements_per_token_layer("mla") == 1152
    # MLA / MHA element ratio at 16 and 128 heads
    assert abs(576 / on.kv_elements_per_token_layer("mha", n_h=16) - 0.140625) < 1e-15
    assert abs(576 / on.kv_elements_per_token_layer("mha", n_h=128) - 0.017578125) < 1e-15


# ------------------------------ append emulation ------------------------------

def _bits(a):
    return np.asarray(a, dtype=np.uint16)


def test_append_position_zero_is_identity():
    from mla_inputs import normal_bf16
    k = normal_bf16(1, 2, 0, 64 * 10).reshape(10, 64)
    np.testing.assert_array_equal(oapp.rotate_k_bits(k, [0] * 10), k)


def test_append_rotation_within_one_bf16_ulp_of_fp64():
    from mla_inputs import bf16_bits_to_f64, f64_to_bf16_bits, normal_bf16
    n = 2000
    pos = (np.arange(n) * 977) % 131072
    k = normal_bf16(5, 2, 0, 64 * n).reshape(n, 64)
    got = oapp.rotate_k_bits(k, pos).astype(np.int32)
    ref = f64_to_bf16_bits(on.rope(bf16_bits_to_f64(k), pos)).astype(np.int32)
    # same sign => bit patterns of neighbouring bf16 values differ by 1
    diff = np.abs(got - ref)
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.99
    # norm preserved to bf16 accuracy
    x = bf16_bits_to_f64(k)
    y = bf16_bits_to_f64(got.astype(np.uint16))
    rel = np.abs(np.linalg.norm(y, axis=1) / np.linalg.norm(x, axis=1) - 1)
    assert rel.max() < 2 ** -8


def test_append_rows_land_where_addressed_and_nowhere_else():
    from mla_inputs import normal_bf16
    cap = 40
    canary = np.full((cap, 576), 0xA5A5, dtype=np.uint16)
    seq_start = np.array([0, 10, 25])
    seq_idx = np.array([0, 2, 1, 2])
    pos = np.array([3, 0, 9, 14])
    c = normal_bf16(3, 1, 0, 4 * 512).reshape(4, 512)
    k = normal_bf16(3, 2, 0, 4 * 64).reshape(4, 64)
    out = oapp.append_rows(canary, seq_start, seq_idx, pos, c, k)
    rows = [3, 25, 19, 39]
    for i, r in enumerate(rows):
        np.testing.assert_array_equal(out[r, :512], c[i])
        np.testing.assert_array_equal(out[r, 512:], oapp.rotate_k_bits(k[i:i + 1], [pos[i]])[0])
    untouched = np.setdiff1d(np.arange(cap), rows)
    assert np.all(out[untouched] == 0xA5A5)
    with pytest.raises(IndexError):
        oapp.append_rows(canary, seq_start, np.array([2]), np.array([15]), c[:1], k[:1])


def test_rope_table_matches_closed_values():
    c, s = oapp.rope_table_f32([0, 1, 100])
    assert np.all(c[0] == 1.0) and np.all(s[0] == 0.0)
    assert c[1, 0] == np.float32(math.cos(1.0)) and s[1, 0] == np.float32(math.sin(1.0))
    assert s[2, 16] == np.float32(math.sin(100 * 0.01))


def test_query_up_selection_closed_form():
    pins.check_query_up_selection(on.query_up)


def test_query_up_then_absorb_equals_precomposed():
    pins.check_query_absorb_precomposed(on.query_up, on.absorb_query)
