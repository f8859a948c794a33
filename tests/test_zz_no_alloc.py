"""mla_decode_static (library-owned scratch, no allocation) against mla_decode.

Collected last on purpose: it must pass both alone and after every other test
has used the device.  Two calls in a row reuse the same scratch; both must
agree with the workspace-taking entry point within the decode tolerance
|a - b| <= 1e-2 + 1e-2 |b| (they run the same kernels, so in practice they are
identical).
"""

import ctypes

import numpy as np
import pytest
import torch

import mla_inputs as mi

ATOL, RTOL = 1e-2, 1e-2


def test_no_alloc_rejects_oversized_shape():
    """A shape whose partials exceed the static scratch is refused before any launch (no GPU needed)."""
    import mla_latent_kv_34_b200 as mla
    assert mla.decode_workspace_bytes(54, 1, 128) > mla.DECODE_STATIC_SCRATCH_BYTES
    assert mla.decode_workspace_bytes(53, 1, 128) <= mla.DECODE_STATIC_SCRATCH_BYTES
    st = mla.lib.mla_decode_static(None, None, 0, None, None, None, 54, 1, 128, ctypes.c_float(0.07), 0,
                                   None, None, None, None)
    assert st == 4, mla.lib.mla_status_string(st).decode()


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
        mla.decode_static(q, prob.cache, prob.seq_block, prob.kv_len, prob.W_UV, cfg.n_q, cfg.scale,
                          out=o, lse_out=l, dev_status=prob.status)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    for k in range(2):
        got = outs[k].float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.all(np.abs(got - ref_np) <= ATOL + RTOL * np.abs(ref_np)), f"call {k}"
        assert np.abs(lses[k].cpu().numpy() - ref_lse_np).max() < 2e-2, f"call {k} lse"
