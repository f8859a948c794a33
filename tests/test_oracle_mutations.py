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
