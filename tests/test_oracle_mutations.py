"""Plant a mistake in the oracle (on the CPU) and check that a pin catches it.

Each mutation below is a plausible slip in an attention implementation; the
pins of ``oracle_pins`` must reject every one of them.
"""

import functools
import math

import numpy as np
import pytest

import oracle_pins as pins
from oracle import naive as on

_real_rope = on.rope


def _rope_half_split(x, pos, base=10000.0):
    # pairs (i, i + d/2) instead of adjacent dims
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * on.rope_thetas(d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _rope_reversed(x, pos, base=10000.0):
    return _real_rope(x, -np.asarray(pos), base)


def _rope_query_pos_plus_one(x, pos, base=10000.0):
    # the query is rotated at L - n_q + j + 1 (keys keep their positions);
    # a shift of every position together is invisible to RoPE by design
    if np.ndim(pos) == 0:
        pos = pos + 1
    return _real_rope(x, pos, base)


def _rope_base_wrong(x, pos, base=10000.0):
    return _real_rope(x, pos, 1000.0)


def _rope_dropped(x, pos, base=10000.0):
    return np.zeros(np.broadcast_shapes(np.shape(x), np.shape(pos) + (np.shape(x)[-1],)))


def _no_causal(c, kr, qn, qr, Wk, Wv, n_q, **kw):
    outs = [on.attend_naive(c, kr, qn[j:j + 1], qr[j:j + 1], Wk, Wv, 1, **kw) for j in range(n_q)]
    return tuple(np.concatenate([o[i] for o in outs], axis=0) for i in range(3))


def _swap_uk_uv(c, kr, qn, qr, Wk, Wv, n_q, **kw):
    return on.attend_naive(c, kr, qn, qr, Wv, Wk, n_q, **kw)


def _transposed_wuk(c, kr, qn, qr, Wk, Wv, n_q, **kw):
    # apply W^UK with its 128x128 leading block transposed (a mixed-up index)
    Wk2 = Wk.copy()
    Wk2[:, :, :128] = np.swapaxes(Wk[:, :, :128], 1, 2)
    return on.attend_naive(c, kr, qn, qr, Wk2, Wv, n_q, **kw)


MUTATIONS = {
    "scale_1_over_sqrt128": (functools.partial(on.attend_naive, scale=1 / math.sqrt(128)), None),
    "scale_missing": (functools.partial(on.attend_naive, scale=1.0), None),
    "rope_half_split": (on.attend_naive, _rope_half_split),
    "rope_reversed_direction": (on.attend_naive, _rope_reversed),
    "rope_query_position_off_by_one": (on.attend_naive, _rope_query_pos_plus_one),
    "rope_wrong_base": (on.attend_naive, _rope_base_wrong),
    "rope_term_dropped": (on.attend_naive, _rope_dropped),
    "no_causal_mask_within_pair": (_no_causal, None),
    "w_uk_w_uv_swapped": (_swap_uk_uv, None),
    "w_uk_index_transposed": (_transposed_wuk, None),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(name, monkeypatch):
    attend, rope_impl = MUTATIONS[name]
    if rope_impl is not None:
        monkeypatch.setattr(on, "rope", rope_impl)
    caught = []
    # cheap checks first; brute force last
    for check in pins.ALL_SINGLE:
        try:
            check(attend)
        except (AssertionError, ValueError):
            caught.append(check.__name__)
            break
    assert caught, f"no pin caught mutation {name}"


# ---------------------------------------------------------------- query side

def _qup_transposed(cq, Wuq, Wqr):
    # the square leading block of each head's W^UQ used transposed
    W2 = Wuq.copy()
    W2[:, :, :128] = np.swapaxes(Wuq[:, :, :128], 1, 2)
    return on.query_up(cq, W2, Wqr)


def _qup_head_shift(cq, Wuq, Wqr):
    # head h reads head h+1's weights
    return on.query_up(cq, np.roll(Wuq, -1, axis=0), np.roll(Wqr, -1, axis=0))


def _qup_rope_from_content(cq, Wuq, Wqr):
    # q^R taken from the first 64 rows of W^UQ instead of W^QR
    return on.query_up(cq, Wuq, Wuq[:, :64])


def _qup_dropped_column(cq, Wuq, Wqr):
    # the last column of c^Q left out of the contraction
    cq2 = np.array(cq, dtype=np.float64)
    cq2[:, -1] = 0.0
    return on.query_up(cq2, Wuq, Wqr)


QUERY_MUTATIONS = {
    "w_uq_index_transposed": _qup_transposed,
    "query_head_shifted": _qup_head_shift,
    "q_rope_from_w_uq": _qup_rope_from_content,
    "c_q_last_column_dropped": _qup_dropped_column,
}


@pytest.mark.parametrize("name", sorted(QUERY_MUTATIONS))
def test_query_pins_reject_planted_mistake(name):
    mutated = QUERY_MUTATIONS[name]
    caught = False
    for check in (pins.check_query_up_selection,
                  lambda f: pins.check_query_absorb_precomposed(f, on.absorb_query)):
        try:
            check(mutated)
        except AssertionError:
            caught = True
            break
    assert caught, f"no query-side pin caught mutation {name}"
