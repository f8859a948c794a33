"""Naive-form prefill attention (mla_prefill_naive) against the fp64 oracle's naive form.

The oracle's attend_naive with n_q = n is exactly a prefill chunk: query j of the chunk sits at
position L - n + j and sees keys 0 .. L - n + j.  Same parity bar as the decode.  The sequence's
cache blocks are scattered over the pool (a shuffled block table, NaN in every unowned block).
"""

import numpy as np
import pytest
import torch

import mla_inputs as mi

pytestmark = pytest.mark.gpu
ATOL, RTOL = 1e-2, 1e-2


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness
    return gpu_harness


def _prefill(H, L, n, heads, seed):
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("prefill", B=1, H=heads, n_q=n, L=L, seed=seed)
    prob = H.build_problem(cfg, shuffle_seed=seed)
    lse = torch.empty((n, heads), dtype=torch.float32, device="cuda")
    out = mla.prefill_naive(prob.q_nope, prob.q_rope, prob.rope_tab, prob.cache, prob.block_table[0], L, prob.W_UK,
                            prob.W_UV, cfg.scale, lse_out=lse, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0, mla.device_status_string(int(prob.status.item()))
    return prob, out, lse


@pytest.mark.parametrize("L,n,heads", [(300, 300, 2), (1000, 400, 4), (129, 1, 1), (2500, 640, 2), (128, 128, 8),
                                       (777, 333, 16), (1100, 1024, 1), (64, 64, 128), (1500, 341, 3)])
def test_prefill_naive_matches_oracle(H, L, n, heads):
    prob, out, lse = _prefill(H, L, n, heads, 5000 + L + n + heads)
    ref, _, ref_lse = prob.oracle(0)
    got = out.float().cpu().numpy()
    excess = np.abs(got - ref) - (ATOL + RTOL * np.abs(ref))
    assert excess.max() <= 0, f"max excess {excess.max():.3e}"
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-2
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 2e-2


def test_prefill_naive_agrees_with_absorbed_decode(H):
    """n = 16 new tokens: the naive chunk path and the absorbed decode compute the same attention."""
    import mla_latent_kv_34_b200 as mla
    L, n, heads = 600, 16, 32
    prob, out, _ = _prefill(H, L, n, heads, 77)
    dec, _ = prob.decode(prob.absorb())
    torch.cuda.synchronize()
    a, b = out.float().cpu().numpy(), dec.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= 2 * (ATOL + RTOL * np.abs(b)))


def test_prefill_naive_reports_bad_block_entry(H):
    """A block entry outside the pool is reported (and never dereferenced)."""
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("prefill-bad", B=1, H=2, n_q=50, L=300, seed=31)
    prob = H.build_problem(cfg)
    blocks = prob.block_table[0].clone()
    blocks[1] = -3
    mla.prefill_naive(prob.q_nope, prob.q_rope, prob.rope_tab, prob.cache, blocks, 300, prob.W_UK, prob.W_UV,
                      cfg.scale, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0x1
