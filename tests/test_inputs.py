"""The seeded input generator: determinism, sub-range regeneration, rounding."""

from fractions import Fraction

import numpy as np

import mla_inputs as mi


def test_subrange_equals_slice_of_full_range():
    full = mi.normal_bf16(42, 3, 0, 5001)
    for a, n in ((0, 1), (1, 7), (2, 2), (999, 1000), (4997, 4)):
        np.testing.assert_array_equal(mi.normal_bf16(42, 3, a, n), full[a:a + n])


def test_threaded_large_generation_matches_chunks():
    n = (1 << 22) + 12345
    big = mi.normal_bf16(7, 1, 100, n)
    np.testing.assert_array_equal(big[:1000], mi.normal_bf16(7, 1, 100, 1000))
    np.testing.assert_array_equal(big[-1000:], mi.normal_bf16(7, 1, 100 + n - 1000, 1000))


def test_streams_and_seeds_differ():
    a = mi.normal_bf16(1, 1, 0, 100)
    assert not np.array_equal(a, mi.normal_bf16(1, 2, 0, 100))
    assert not np.array_equal(a, mi.normal_bf16(2, 1, 0, 100))


def test_moments_are_standard_normal():
    x = mi.bf16_bits_to_f64(mi.normal_bf16(9, 4, 0, 400000))
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    w = mi.bf16_bits_to_f64(mi.normal_bf16(9, 5, 0, 400000, 1 / np.sqrt(512)))
    assert abs(w.std() * np.sqrt(512) - 1.0) < 0.01


def _exact_rne_bf16(v: float) -> int:
    """Round-to-nearest-even to 8 significant bits by exact rational arithmetic."""
    if v == 0.0:
        return 0x8000 if np.signbit(v) else 0
    sign = 0x8000 if v < 0 else 0
    f = Fraction(abs(v))
    e = 0
    while f >= 2:
        f /= 2
        e += 1
    while f < 1:
        f *= 2
        e -= 1
    scaled = f * 128  # in [128, 256)
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    if lo == 256:
        lo, e = 128, e + 1
    return sign | ((e + 127) << 7) | (lo - 128)


def test_f64_to_bf16_rounding_is_exact_rne():
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000))
    # ties and near-ties around representable bf16 values
    for m in range(128, 256, 7):
        base = m / 128.0
        ulp = 1 / 128.0
        vals += [base + ulp / 2, base + ulp / 2 + 2 ** -40, base + ulp / 2 - 2 ** -40, -(base + ulp / 2)]
    got = mi.f64_to_bf16_bits(np.array(vals))
    exp = np.array([_exact_rne_bf16(v) for v in vals], dtype=np.uint16)
    np.testing.assert_array_equal(got, exp)


def test_ragged_lengths_in_range_and_clamped():
    cfg = mi.CONFIGS["ragged"]
    L = mi.kv_lengths(cfg)
    assert len(L) == 128 and L.min() >= 2 and L.max() <= 32768
    assert np.array_equal(L, mi.kv_lengths(cfg))
    s = mi.seq_starts(L)
    assert s[0] == 0 and np.all(np.diff(s) == L[:-1])


def test_sequence_rows_are_pool_rows():
    cfg = mi.MLAConfig("t", B=3, H=2, n_q=2, L=None, L_max=50, seed=5)
    L = mi.kv_lengths(cfg)
    s = mi.seq_starts(L)
    seq = mi.sequence(cfg, 2, L)
    c, k = mi.token_rows(cfg, 0, int(L.sum()))
    np.testing.assert_array_equal(seq.c_kv, c[s[2]:s[2] + L[2]])
    np.testing.assert_array_equal(seq.k_rope, k[s[2]:s[2] + L[2]])
    qn, qr = mi.queries(cfg)
    np.testing.assert_array_equal(seq.q_nope, qn[4:6])
