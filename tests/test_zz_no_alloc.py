"""mla_decode_static (library-owned scratch, no allocation) against mla_decode.

Collected last on purpose: it must pass both alone and after every other test
has used the device.  Two calls in a row reuse the same scratch; both must
agree with the workspace-taking entry point within the decode tolerance
|a - b| <= 1e-2 + 1e-2 |b| (they run the same kernels, so in practice they are
identical).  A third case fills the scratch to its documented limit and is
checked against the fp64 oracle.
"""

import ctypes

import numpy as np
import pytest
import torch

import mla_inputs as mi

ATOL, RTOL = 1e-2, 1e-2


def test_no_alloc_limit_matches_the_library():
    """The Python copy of the scratch size agrees with the library: the largest V2-shaped batch whose
    workspace fits is accepted by host validation, the next one is refused before any launch (no GPU
    needed: validation fails, or passes only as far as the null-pointer check)."""
    import mla_latent_kv_34_b200 as mla
    lim = mla.DECODE_STATIC_SCRATCH_BYTES
    assert mla.decode_workspace_bytes(32, 1, 128) <= lim < mla.decode_workspace_bytes(33, 1, 128)
    st = mla.lib.mla_decode_static(None, None, 0, None, 0, None, None, 33, 1, 128, ctypes.c_float(0.07), 0,
                                   None, None, None, None)
    assert st == 4, mla.lib.mla_status_string(st).decode()
    # B = 32 fits: validation moves on to the arguments (null q) instead of refusing the size
    st = mla.lib.mla_decode_static(None, None, 0, None, 0, None, None, 32, 1, 128, ctypes.c_float(0.07), 0,
                                   None, None, None, None)
    assert st == 1, mla.lib.mla_status_string(st).decode()
    # few heads (the one-SM path, 32 rows per slot): a V2-Lite-sized batch fits as well
    assert mla.decode_workspace_bytes(64, 1, 16) <= lim
    st = mla.lib.mla_decode_static(None, None, 0, None, 0, None, None, 64, 1, 16, ctypes.c_float(0.07), 0,
                                   None, None, None, None)
    assert st == 1, mla.lib.mla_status_string(st).decode()


@pytest.mark.gpu
def test_no_alloc_decode_matches_decode_twice(cuda_ok):
    import gpu_harness as H
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("no-alloc", B=20, H=128, n_q=1, L=None, L_max=1500, seed=91)
    assert mla.decode_workspace_bytes(cfg.B, cfg.n_q, cfg.H) <= mla.DECODE_STATIC_SCRATCH_BYTES
    prob = H.build_problem(cfg)
    q = prob.absorb()
    ref, ref_lse = prob.decode(q)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    ref_np, ref_lse_np = ref.float().cpu().numpy(), ref_lse.cpu().numpy()
    outs = [torch.empty_like(ref) for _ in range(2)]
    lses = [torch.empty_like(ref_lse) for _ in range(2)]
    for o, l in zip(outs, lses):
        mla.decode_static(q, prob.cache, prob.block_table, prob.kv_len, prob.W_UV, cfg.n_q, cfg.scale,
                          out=o, lse_out=l, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    for k in range(2):
        got = outs[k].float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.all(np.abs(got - ref_np) <= ATOL + RTOL * np.abs(ref_np)), f"call {k}"
        assert np.abs(lses[k].cpu().numpy() - ref_lse_np).max() < 2e-2, f"call {k} lse"


@pytest.mark.gpu
def test_no_alloc_decode_at_the_scratch_limit_matches_oracle(cuda_ok):
    """B = 32, H = 128 fills the scratch to the limit (the last slots and the merged-output tiles at its
    end are in use); sampled rows against the fp64 oracle, the same check the parity tests use."""
    import gpu_harness as H
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("no-alloc-limit", B=32, H=128, n_q=1, L=None, L_max=400, seed=92)
    assert mla.decode_workspace_bytes(cfg.B, cfg.n_q, cfg.H) <= mla.DECODE_STATIC_SCRATCH_BYTES
    prob = H.build_problem(cfg, shuffle_seed=3)
    q = prob.absorb()
    out = torch.empty((cfg.T, cfg.H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    mla.decode_static(q, prob.cache, prob.block_table, prob.kv_len, prob.W_UV, cfg.n_q, cfg.scale,
                      out=out, lse_out=lse, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    got_all = out.float().cpu().numpy()
    lse_all = lse.cpu().numpy()
    heads = list(range(0, 128, 13))
    for b in (0, 17, 31):
        ref, _, ref_lse = prob.oracle(b, heads=heads)
        got = got_all[b][None][:, heads]
        assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)), f"seq {b}"
        assert np.abs(lse_all[b][heads] - ref_lse[0]).max() < 2e-2


@pytest.mark.gpu
def test_no_alloc_decode_few_heads_matches_oracle(cuda_ok):
    """Few heads (n_q * H <= 32: the one-SM attend kernel, 32 rows per workspace slot) through the
    library-owned scratch: the same result as mla_decode and the oracle on sampled sequences."""
    import gpu_harness as H
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("no-alloc-few", B=64, H=16, n_q=2, L=None, L_max=900, seed=93)
    assert mla.decode_workspace_bytes(cfg.B, cfg.n_q, cfg.H) <= mla.DECODE_STATIC_SCRATCH_BYTES
    prob = H.build_problem(cfg, shuffle_seed=4)
    q = prob.absorb()
    ref, ref_lse = prob.decode(q)
    out = torch.empty_like(ref)
    lse = torch.empty_like(ref_lse)
    mla.decode_static(q, prob.cache, prob.block_table, prob.kv_len, prob.W_UV, cfg.n_q, cfg.scale,
                      out=out, lse_out=lse, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    a, b = out.float().cpu().numpy(), ref.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= ATOL + RTOL * np.abs(b))
    got_all = a.reshape(cfg.B, cfg.n_q, cfg.H, 128)
    lse_all = lse.cpu().numpy().reshape(cfg.B, cfg.n_q, cfg.H)
    for bb in (0, 31, 63):
        ref_o, _, ref_l = prob.oracle(bb)
        assert np.all(np.abs(got_all[bb] - ref_o) <= ATOL + RTOL * np.abs(ref_o)), f"seq {bb}"
        assert np.abs(lse_all[bb] - ref_l).max() < 2e-2
