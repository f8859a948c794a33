"""Query up-projections (q^C = W^UQ c^Q, q^R = W^QR c^Q) on the GPU against the fp64 oracle.

The MLA explainer (2.2.1.2) compresses queries like keys and values; the
library's ``mla_query_up`` produces exactly the inputs of ``mla_absorb_q``.
Tolerance of the projection: one bf16 rounding of an fp32 tensor-core sum,
|gpu - ref| <= 2^-8 |ref| + 1e-4 (half a bf16 ulp is at most 2^-8 of the value;
the fp32 accumulation over d_c' <= 1536 terms adds far less than 1e-4).  The
chained check (c^Q -> q -> decode) is held to the decode parity bar.
"""

import numpy as np
import pytest
import torch

import mla_inputs as mi
from oracle import naive as on

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gpu_harness
    return gpu_harness


def _run(H, T, nh, d_cq, seed):
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("qup", B=T, H=nh, n_q=1, L=1, seed=seed)
    cq, wuq, wqr = mi.compressed_queries(cfg, d_cq)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    qn, qr = mla.query_up(H.to_dev_bf16(cq, "cuda"), H.to_dev_bf16(wuq, "cuda"), H.to_dev_bf16(wqr, "cuda"),
                          dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    f = mi.bf16_bits_to_f64
    ref_n, ref_r = on.query_up(f(cq), f(wuq), f(wqr))
    return qn.float().cpu().numpy(), qr.float().cpu().numpy(), ref_n, ref_r


@pytest.mark.parametrize("T,nh,d_cq", [(1, 1, 64), (17, 16, 1536), (32, 128, 1536), (130, 3, 576),
                                       (200, 8, 128), (256, 128, 1536)])
def test_query_up_matches_oracle(H, T, nh, d_cq):
    got_n, got_r, ref_n, ref_r = _run(H, T, nh, d_cq, 4000 + T + nh + d_cq)
    for got, ref, name in ((got_n, ref_n, "q^C"), (got_r, ref_r, "q^R")):
        assert got.shape == ref.shape, name
        bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-4
        assert not bad.any(), f"{name}: {int(bad.sum())} elements off, first at {np.argwhere(bad)[0].tolist()}"


def test_query_up_chain_to_decode(H):
    """c^Q -> mla_query_up -> mla_absorb_q -> mla_decode against the oracle attention on the
    oracle's own fp64 q^C, q^R (the GPU rounds q^C and q^R to bf16 once, like any stored query)."""
    import mla_latent_kv_34_b200 as mla
    d_cq = 1536
    cfg = mi.MLAConfig("qup-chain", B=3, H=32, n_q=2, L=None, L_max=900, seed=4242)
    prob = H.build_problem(cfg)
    cq, wuq, wqr = mi.compressed_queries(cfg, d_cq)
    qn, qr = mla.query_up(H.to_dev_bf16(cq, "cuda"), H.to_dev_bf16(wuq, "cuda"), H.to_dev_bf16(wqr, "cuda"),
                          dev_status=prob.status)
    q = mla.absorb_q(qn, qr, prob.q_pos, prob.W_UK, prob.rope_tab, dev_status=prob.status)
    out, lse = prob.decode(q)
    torch.cuda.synchronize()
    assert int(prob.status.item()) == 0
    f = mi.bf16_bits_to_f64
    ref_qn, ref_qr = on.query_up(f(cq), f(wuq), f(wqr))
    Wk, Wv = f(mi.weights(cfg, "uk")), f(mi.weights(cfg, "uv"))
    got = out.float().cpu().numpy().reshape(cfg.B, cfg.n_q, cfg.H, 128)
    for b in range(cfg.B):
        s = mi.sequence(cfg, b, prob.lengths)
        rows = slice(b * cfg.n_q, (b + 1) * cfg.n_q)
        ref, _, _ = on.attend_naive(f(s.c_kv), f(s.k_rope), ref_qn[rows], ref_qr[rows], Wk, Wv, cfg.n_q,
                                    scale=cfg.scale, base=cfg.rope_base)
        assert np.all(np.abs(got[b] - ref) <= 1e-2 + 1e-2 * np.abs(ref)), f"sequence {b}"
        assert np.linalg.norm(got[b] - ref) / np.linalg.norm(ref) < 1e-2


@pytest.mark.parametrize("T,nh,d_cq", [(1, 1, 64), (17, 16, 1536), (32, 128, 1536), (130, 3, 576),
                                       (200, 8, 128), (256, 128, 1536), (64, 5, 192)])
def test_query_absorb_is_query_up_then_absorb(H, T, nh, d_cq):
    """The fused c^Q -> q_abs call equals mla_query_up followed by mla_absorb_q bit for bit, and the
    oracle's fp64 chain W^UK^T (W^UQ c^Q), R_pos (W^QR c^Q) within one bf16 rounding of each step."""
    import mla_latent_kv_34_b200 as mla
    cfg = mi.MLAConfig("qabs", B=T, H=nh, n_q=1, L=1, seed=6000 + T + nh + d_cq)
    cq, wuq, wqr = mi.compressed_queries(cfg, d_cq)
    wuk = mi.weights(cfg, "uk")
    dev = "cuda"
    pos = ((np.arange(T) * 7919 + 3) % 131072).astype(np.int32)
    tab = mla.rope_table(131072, 10000.0, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cq_d, wuq_d, wqr_d, wuk_d = (H.to_dev_bf16(x, dev) for x in (cq, wuq, wqr, wuk))
    pos_d = torch.from_numpy(pos).to(dev)
    fused = mla.query_absorb(cq_d, wuq_d, wqr_d, wuk_d, pos_d, tab, dev_status=status)
    qn, qr = mla.query_up(cq_d, wuq_d, wqr_d, dev_status=status)
    two = mla.absorb_q(qn, qr, pos_d, wuk_d, tab, dev_status=status)
    unrot = mla.query_absorb(cq_d, wuq_d, wqr_d, wuk_d, None, tab, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(fused.view(torch.int16), two.view(torch.int16))
    # pos = NULL: the RoPE part is q^R as rounded, not rotated
    assert torch.equal(unrot[..., 512:].view(torch.int16), qr.view(torch.int16))
    f = mi.bf16_bits_to_f64
    ref_n, ref_r = on.query_up(f(cq), f(wuq), f(wqr))
    ref_abs = on.absorb_query(ref_n, f(wuk))
    ref_pe = on.rope(ref_r, pos[:, None])
    got = fused.float().cpu().numpy()
    # Rigorous bounds: q^C (and q^R) are rounded to bf16 once, a relative error of at most u = 2^-8 (bf16
    # keeps 8 significant bits); through W^UK that is at most u sum_i |W^UK[i, c]| |q^C_i|; the output is
    # rounded once more (at most u |value|, taken as u (1 + 2^-6) |ref|); fp32 sums add far less than 1e-5.
    u = 2.0 ** -8
    prop = u * np.einsum("hic,thi->thc", np.abs(f(wuk)), np.abs(ref_n))
    assert np.all(np.abs(got[..., :512] - ref_abs) <= prop + u * (1 + 2 ** -6) * np.abs(ref_abs) + 1e-5)
    # RoPE part: a rotation of the rounded pair, so the pair's rounding error stays within u (|x0| + |x1|)
    pair = np.abs(ref_r[..., 0::2]) + np.abs(ref_r[..., 1::2])
    prop_r = u * np.repeat(pair, 2, axis=-1)
    assert np.all(np.abs(got[..., 512:] - ref_pe) <= prop_r + u * (1 + 2 ** -6) * np.abs(ref_pe) + 1e-5)
