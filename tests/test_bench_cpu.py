"""Host-side arithmetic of bench.py, checked on the CPU with stand-ins for the device calls."""

import contextlib
import os
import sys
import types

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import mla_inputs as mi  # noqa: E402


def _fake_torch():
    class Graph:
        def replay(self):
            pass

    t = types.SimpleNamespace(**{k: getattr(torch, k) for k in ("from_numpy", "empty", "zeros", "bfloat16",
                                                                 "int16", "int32")})
    t.cuda = types.SimpleNamespace(CUDAGraph=Graph, synchronize=lambda: None,
                                   graph=lambda g, capture_error_mode=None: contextlib.nullcontext())
    return t


def test_query_up_measurement_bytes_and_shapes():
    calls = []

    def query_up(cq, wuq, wqr, q_nope=None, q_rope=None, dev_status=None):
        calls.append((tuple(cq.shape), tuple(wuq.shape), tuple(wqr.shape), tuple(q_nope.shape),
                      tuple(q_rope.shape)))

    mla = types.SimpleNamespace(query_up=query_up, device_status_string=str)
    cfg = mi.MLAConfig("small", B=4, H=8, n_q=2, L=64, seed=5)
    d_cq = 256
    us = 2.0
    r = bench.measure_query_up(_fake_torch(), mla, cfg, "cpu", lambda g, n: [us * 1e-3] * n, 7,
                               {"hbm_gbs": 1000.0}, d_cq)
    T, H = cfg.T, cfg.H
    assert calls[0] == ((T, d_cq), (H, 128, d_cq), (H, 64, d_cq), (T, H, 128), (T, H, 64))
    want = H * 192 * d_cq * 2 + T * d_cq * 2 + T * H * 192 * 2
    assert r["algorithmic_bytes"] == want
    assert r["launches"] == 7 and r["us_per_launch"] == us
    assert np.isclose(r["achieved"], want / (us * 1e-6) / 1e9, rtol=1e-3)
    assert np.isclose(r["frac"], r["achieved"] / 1000.0, rtol=1e-3)


def test_reference_arm_line_carries_the_contract_keys():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line with the
    contract's keys, its own cpu_baseline and an e2e object with no host-device traffic."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--config", "tiny"], cwd=root, capture_output=True, text=True,
                         timeout=300, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_clock_window_keeps_only_samples_inside_it():
    import datetime as dt
    lines = []
    t = dt.datetime(2026, 1, 1, 12, 0, 0)
    for k in range(10):
        ts = (t + dt.timedelta(milliseconds=100 * k)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        reason = "Active" if k == 9 else "Not Active"
        lines.append(f"{ts}, 0, {1000 + k}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {reason}\n")
    r = bench.ClockSampler.parse(lines, t + dt.timedelta(milliseconds=250), t + dt.timedelta(milliseconds=650))
    assert r["samples"] == 4 and r["sm_mhz"] == 1004.5 and r["reasons"] == []
    r = bench.ClockSampler.parse(lines)
    assert r["samples"] == 10 and r["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler.parse(lines, t + dt.timedelta(seconds=5)) is None


def test_step_bytes_count_inputs_and_outputs_only():
    cfg = mi.CONFIGS["v2"]
    c = bench.step_counts(cfg, mi.kv_lengths(cfg))
    T, H = cfg.T, cfg.H
    want = (c["sum_L"] * 1152 + 2 * H * 128 * 512 * 2 + T * H * 192 * 2 + T * H * 128 * 2 + T * 576 * 4)
    assert c["step_bytes"] == want
    assert c["core_flops"] == 2 * H * 1088 * c["sum_L"]


def test_both_oracle_arms_sample_the_same_way():
    """cpu_baseline and the reference arm share one sample plan and one rate definition."""
    cfg = mi.CONFIGS["ragged"]
    L = mi.kv_lengths(cfg)
    plans = [bench.oracle_sample_plan(cfg, L, i) for i in range(2 * cfg.B + 3)]
    assert [p[0] for p in plans[:cfg.B]] == list(range(cfg.B))
    assert all(len(h) == bench.ORACLE_HEADS for _, h in plans)
    assert plans[cfg.B][1][0] == bench.ORACLE_HEADS
    r = bench.oracle_rate_line(cfg, L, [2.0, 2.0], [1000, 3000])
    c = bench.step_counts(cfg, L)
    assert np.isclose(r["full_step_s"], 4.0 / 4000 * c["sum_L"] * cfg.H)
    assert np.isclose(r["value"], c["step_bytes"] / r["full_step_s"] / 1e12)


def test_packed_upload_buffer_holds_every_input_at_aligned_offsets():
    """The end-to-end leg uploads a step's inputs as one buffer: every tensor keeps its dtype, shape and
    bytes, and starts on a 256-byte boundary (the library needs 16)."""
    g = torch.Generator().manual_seed(3)
    like = {"c_kv": torch.randn((5, 512), generator=g).bfloat16(), "pos": torch.arange(7, dtype=torch.int32),
            "q_rope": torch.randn((3, 2, 64), generator=g).bfloat16(), "seq_idx": torch.zeros(1, dtype=torch.int32)}
    buf, views = bench.packed(torch, like, "cpu", False)
    base = buf.data_ptr()
    for k, t in like.items():
        v = views[k]
        assert v.dtype == t.dtype and v.shape == t.shape
        assert (v.data_ptr() - base) % 256 == 0
        v.copy_(t)
    for k, t in like.items():  # no view overlaps another
        assert torch.equal(views[k], t)
    assert buf.numel() == sum((t.numel() * t.element_size() + 255) // 256 * 256 for t in like.values())
