"""Checks that pin the fp64 oracle to facts fixed by the pages and by mathematics.

Each check takes the decode function under test (signature of
``oracle.naive.attend_naive``) so that the same check can be run against the
real oracle (must pass) and against oracles with a planted mistake (some check
must fail).  Sources: the MLA pages -- "两张账" (chenyuan1125.github.io),
section "第一张账"; the xinfinite.net explainer, sections 2.2.1.1 and 2.2.2.
"""

from __future__ import annotations

import math

import numpy as np

from mla_inputs import MLAConfig, bf16_bits_to_f64, normal_bf16

D_C, D_R, D_H = 512, 64, 128
SCALE = 1.0 / math.sqrt(192.0)


def rand_problem(L: int, H: int, n_q: int, seed: int):
    """Small random problem with the workloads' distributions (bf16 values, as fp64)."""
    g = lambda s, n, sig=1.0: bf16_bits_to_f64(normal_bf16(seed, s, 0, n, sig))
    c = g(11, L * D_C).reshape(L, D_C)
    kr = g(12, L * D_R).reshape(L, D_R)
    qn = g(13, n_q * H * D_H).reshape(n_q, H, D_H)
    qr = g(14, n_q * H * D_R).reshape(n_q, H, D_R)
    Wk = g(15, H * D_H * D_C, 1 / math.sqrt(D_C)).reshape(H, D_H, D_C)
    Wv = g(16, H * D_H * D_C, 1 / math.sqrt(D_C)).reshape(H, D_H, D_C)
    return c, kr, qn, qr, Wk, Wv


def check_single_token(attend) -> None:
    """L = 1: softmax over one key is 1, so out = W^UV c_0 and lse = s_0."""
    c, kr, qn, qr, Wk, Wv = rand_problem(1, 3, 1, 101)
    out, o_lat, lse = attend(c, kr, qn, qr, Wk, Wv, 1)[:3]
    for h in range(3):
        np.testing.assert_allclose(out[0, h], Wv[h] @ c[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o_lat[0, h], c[0], rtol=1e-12, atol=1e-12)


def check_constant_values(attend) -> None:
    """All c_t equal: whatever the scores, the output is W^UV c (weights sum to 1)."""
    c, kr, qn, qr, Wk, Wv = rand_problem(9, 2, 2, 102)
    c[:] = c[0]
    out = attend(c, kr, qn, qr, Wk, Wv, 2)[0]
    for j in range(2):
        for h in range(2):
            np.testing.assert_allclose(out[j, h], Wv[h] @ c[0], rtol=1e-11, atol=1e-12)


def check_zero_query(attend) -> None:
    """q = 0: all scores are 0, the softmax is uniform over the visible keys."""
    L = 7
    c, kr, qn, qr, Wk, Wv = rand_problem(L, 2, 1, 103)
    qn[:] = 0.0
    qr[:] = 0.0
    out, o_lat, lse = attend(c, kr, qn, qr, Wk, Wv, 1)[:3]
    for h in range(2):
        np.testing.assert_allclose(o_lat[0, h], c.mean(axis=0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out[0, h], Wv[h] @ c.mean(axis=0), rtol=1e-11, atol=1e-12)
        assert abs(lse[0, h] - math.log(L)) < 1e-12


def check_scale_closed_form(attend) -> None:
    """Two keys, W^UK = [I | 0] so k^C_t = c_t[:128], q^R = 0.

    s_t = a c_t[0] / sqrt(192); p_0 = 1 / (1 + exp(s_1 - s_0)); the output is
    W^UV (p_0 c_0 + p_1 c_1) and lse = log(e^{s_0} + e^{s_1}).
    """
    c, kr, qn, qr, Wk, Wv = rand_problem(2, 1, 1, 104)
    Wk[:] = 0.0
    Wk[0, :, :D_H] = np.eye(D_H)
    qn[:] = 0.0
    qr[:] = 0.0
    a = 3.0
    qn[0, 0, 0] = a
    c[0, 0], c[1, 0] = 1.5, -0.75
    s0, s1 = a * 1.5 * SCALE, a * -0.75 * SCALE
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    out, o_lat, lse = attend(c, kr, qn, qr, Wk, Wv, 1)[:3]
    np.testing.assert_allclose(o_lat[0, 0], p0 * c[0] + (1 - p0) * c[1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out[0, 0], Wv[0] @ (p0 * c[0] + (1 - p0) * c[1]), rtol=1e-11, atol=1e-13)
    assert abs(lse[0, 0] - math.log(math.exp(s0) + math.exp(s1))) < 1e-12


def check_rope_closed_form(attend) -> None:
    """Only the RoPE channel is active (q_nope = 0).

    With the query at position p = L - 1 and keys at t = 0..L-1:
      q^R = e_{2i}, k_raw = e_{2i}   ->  s_t = cos((t - p) theta_i) / sqrt(192)
      q^R = e_{2i+1}, k_raw = e_{2i} ->  s_t = sin((t - p) theta_i) / sqrt(192)
    with theta_i = 10000^(-2i/64): theta_0 = 1, theta_16 = 0.01.  lse of a
    query is log sum_t exp(s_t), which fixes every s_t for these inputs.
    """
    L = 5
    p = L - 1
    for i, theta in ((0, 1.0), (16, 0.01), (31, 10000.0 ** (-62 / 64))):
        for which in ("cos", "sin"):
            c, kr, qn, qr, Wk, Wv = rand_problem(L, 1, 1, 105 + i)
            qn[:] = 0.0
            qr[:] = 0.0
            kr[:] = 0.0
            kr[:, 2 * i] = 1.0
            qr[0, 0, 2 * i + (1 if which == "sin" else 0)] = 1.0
            f = math.cos if which == "cos" else math.sin
            s = np.array([f((t - p) * theta) * SCALE for t in range(L)])
            lse = attend(c, kr, qn, qr, Wk, Wv, 1)[2]
            assert abs(lse[0, 0] - math.log(np.exp(s).sum())) < 1e-12, (i, which)
            o_lat = attend(c, kr, qn, qr, Wk, Wv, 1)[1]
            w = np.exp(s - s.max())
            w /= w.sum()
            np.testing.assert_allclose(o_lat[0, 0], w @ c, rtol=1e-11, atol=1e-13)


def check_causal_within_pair(attend) -> None:
    """n_q = 2: query 0 (position L-2) must not see key L-1; query 1 sees it."""
    L = 6
    c, kr, qn, qr, Wk, Wv = rand_problem(L, 2, 2, 106)
    out_a = attend(c, kr, qn, qr, Wk, Wv, 2)[0]
    c2, kr2 = c.copy(), kr.copy()
    c2[L - 1] *= -5.0
    kr2[L - 1] += 3.0
    out_b = attend(c2, kr2, qn, qr, Wk, Wv, 2)[0]
    np.testing.assert_allclose(out_a[0], out_b[0], rtol=1e-13, atol=1e-14)
    assert np.abs(out_a[1] - out_b[1]).max() > 1e-3


def brute_force(c, kr, qn, qr, Wk, Wv, n_q, base=10000.0):
    """Scalar-loop attention for tiny inputs: plain Python floats, math.fsum, no numpy.

    Builds every head's full key [k^C; R_t k_raw] and value v^C explicitly,
    exponentiates the raw scores (no max shift) and normalises by the sum.
    """
    L = len(c)
    H = len(qn[0])
    c = [[float(v) for v in row] for row in c]
    kr = [[float(v) for v in row] for row in kr]
    half = D_R // 2
    th = [base ** (-2 * i / D_R) for i in range(half)]

    def rot(x, pos):
        y = [0.0] * D_R
        for i in range(half):
            a = pos * th[i]
            y[2 * i] = x[2 * i] * math.cos(a) - x[2 * i + 1] * math.sin(a)
            y[2 * i + 1] = x[2 * i] * math.sin(a) + x[2 * i + 1] * math.cos(a)
        return y

    out = [[None] * H for _ in range(n_q)]
    lse = [[None] * H for _ in range(n_q)]
    for h in range(H):
        Wk_h = [[float(v) for v in row] for row in Wk[h]]
        Wv_h = [[float(v) for v in row] for row in Wv[h]]
        keys, vals = [], []
        for t in range(L):
            kc = [math.fsum(Wk_h[d][i] * c[t][i] for i in range(D_C)) for d in range(D_H)]
            vc = [math.fsum(Wv_h[d][i] * c[t][i] for i in range(D_C)) for d in range(D_H)]
            keys.append(kc + rot(kr[t], t))
            vals.append(vc)
        for j in range(n_q):
            p = L - n_q + j
            q = [float(v) for v in qn[j][h]] + rot([float(v) for v in qr[j][h]], p)
            e = []
            for t in range(p + 1):
                s = math.fsum(q[d] * keys[t][d] for d in range(D_H + D_R)) / math.sqrt(D_H + D_R)
                e.append(math.exp(s))
            z = math.fsum(e)
            out[j][h] = [math.fsum(e[t] * vals[t][d] for t in range(p + 1)) / z for d in range(D_H)]
            lse[j][h] = math.log(z)
    return np.array(out), np.array(lse)


def check_brute_force(attend, cases=((1, 1), (3, 1), (5, 2), (8, 2))) -> None:
    for L, n_q in cases:
        c, kr, qn, qr, Wk, Wv = rand_problem(L, 2, n_q, 200 + L)
        # keep the raw-exp brute force well inside fp64 range
        out, _, lse = attend(c, kr, qn, qr, Wk, Wv, n_q)[:3]
        bout, blse = brute_force(c, kr, qn, qr, Wk, Wv, n_q)
        np.testing.assert_allclose(out, bout, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse, blse, rtol=1e-12, atol=1e-12)


def check_absorbed_identity(attend, absorbed) -> None:
    """The absorbed and naive forms agree algebraically (fp64, random inputs)."""
    for L, n_q, H in ((1, 1, 2), (37, 2, 3), (130, 1, 2)):
        args = rand_problem(L, H, n_q, 300 + L)
        a = attend(*args, n_q)[:3]
        b = absorbed(*args, n_q)
        for x, y in zip(a, b):
            np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-13)


ALL_SINGLE = (check_single_token, check_constant_values, check_zero_query,
              check_scale_closed_form, check_rope_closed_form,
              check_causal_within_pair, check_brute_force)


# ---------------------------------------------------------------- query side (q^C, q^R from c^Q)

def query_weights(H: int, d_cq: int, seed: int):
    """Random W^UQ [H,128,d_cq], W^QR [H,64,d_cq] with variance 1/d_cq, and c^Q ~ N(0,1) rows."""
    g = lambda s, n, sig=1.0: bf16_bits_to_f64(normal_bf16(seed, s, 0, n, sig))
    Wuq = g(21, H * D_H * d_cq, 1 / math.sqrt(d_cq)).reshape(H, D_H, d_cq)
    Wqr = g(22, H * D_R * d_cq, 1 / math.sqrt(d_cq)).reshape(H, D_R, d_cq)
    return Wuq, Wqr


def check_query_up_selection(query_up) -> None:
    """Selection weights give slices of c^Q in closed form.

    Head h's W^UQ_h picks columns (7h + d + 1) mod d_c' (d = 0..127) and W^QR_h
    picks columns (5h + 2i + 3) mod d_c' (i = 0..63): one 1 per row, so
    q^C[t, h, d] = c^Q[t, (7h + d + 1) mod d_c'] and likewise for q^R.  A
    transposed weight, a head read from another head's weights, or the two
    projections swapped all give different slices.
    """
    T, H, d_cq = 3, 4, 320
    rng = np.random.default_rng(17)
    cq = rng.standard_normal((T, d_cq))
    Wuq = np.zeros((H, D_H, d_cq))
    Wqr = np.zeros((H, D_R, d_cq))
    for h in range(H):
        Wuq[h, np.arange(D_H), (7 * h + np.arange(D_H) + 1) % d_cq] = 1.0
        Wqr[h, np.arange(D_R), (5 * h + 2 * np.arange(D_R) + 3) % d_cq] = 1.0
    qn, qr = query_up(cq, Wuq, Wqr)
    assert qn.shape == (T, H, D_H) and qr.shape == (T, H, D_R)
    for h in range(H):
        np.testing.assert_array_equal(qn[:, h], cq[:, (7 * h + np.arange(D_H) + 1) % d_cq])
        np.testing.assert_array_equal(qr[:, h], cq[:, (5 * h + 2 * np.arange(D_R) + 3) % d_cq])


def check_query_absorb_precomposed(query_up, absorb_query) -> None:
    """Query path then absorption equals the precomposed matrix (W^UK_h)^T W^UQ_h applied to c^Q.

    The precomposed product is formed here with one matmul per head, a different
    order of the same sums, so a dropped head, a wrong contraction axis or a
    transposed factor shows as a mismatch far above fp64 rounding.
    """
    T, H, d_cq = 5, 3, 192
    Wuq, Wqr = query_weights(H, d_cq, 31)
    _, _, _, _, Wk, _ = rand_problem(1, H, 1, 32)
    cq = bf16_bits_to_f64(normal_bf16(33, 1, 0, T * d_cq)).reshape(T, d_cq)
    qn, qr = query_up(cq, Wuq, Wqr)
    q_abs = absorb_query(qn, Wk)
    for h in range(H):
        M = Wk[h].T @ Wuq[h]                                   # [512, d_cq]
        np.testing.assert_allclose(q_abs[:, h], cq @ M.T, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(qr[:, h], cq @ Wqr[h].T, rtol=1e-12, atol=1e-13)
