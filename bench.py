#!/usr/bin/env python
"""Benchmark of one MLA weight-absorbed decode step on B200.

A step is the whole hot path over one batch: append the step's n_q new tokens
to the latent cache (mla_append_cache), absorb W^UK into the queries
(mla_absorb_q), attend against the cache (mla_decode_attend) and merge the
split partials + apply W^UV (mla_decode_finish).  Inputs are seeded synthetic
tensors of the configuration's shapes (mla_inputs); the cache is filled before
timing and stays resident in HBM.  L2 is flushed (a 256 MiB write) between
timed steps.

  python bench.py [--config ragged] [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  The headline workload is the ragged serving
batch (the largest single-GPU configuration); at N = 1 the other 128-head
workloads (V2-shaped and 128K) are measured the same way into `per_config`.
With --gpus N > 1 (torchrun), every rank runs its own batch (weak scaling, no
data-path collective); timing is the max over ranks.  --impl reference times
the fp64 CPU oracle on bounded samples of the same workload.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_inputs as mi  # noqa: E402

METRIC = "MLA absorbed decode: µs/step, TB/s & TFLOP/s as % of B200 roofline"
UNIT = "TB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# kernels each C-ABI call of the step launches
KERNELS_PER_STEP = {"append": 1, "absorb": 1, "attend": 1, "finish": 2}
CORE_SOURCES = ["mla_latent_kv_34_b200/csrc/decode_tc.cu", "mla_latent_kv_34_b200/csrc/sm100.cuh"]
CLOCK_WINDOW_S = 1.0   # the clock sampler needs about a second of load to see several samples
ORACLE_HEADS = 16      # heads per oracle sample (both the cpu_baseline and the reference arm)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 200 for the CUDA path; 20 oracle samples for --impl reference)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="ragged", choices=sorted(mi.CONFIGS),
                    help="headline workload (default: ragged, the largest single-GPU configuration)")
    ap.add_argument("--extra-configs", default="v2,128k",
                    help="comma-separated configurations also measured (N=1 only) into the line's per_config "
                         "object; empty to skip")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-query-up", action="store_true",
                    help="skip the separate timing of the compressed-query up-projection")
    ap.add_argument("--query-rank", type=int, default=1536, help="d_c' of the query up-projection timing")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds of the oracle samples")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the separate timing of prefill chunks (naive vs absorbed form)")
    ap.add_argument("--prefill-config", default="v2",
                    help="workload whose first sequence the prefill chunks are timed on (N=1 only)")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ workload arithmetic

def step_counts(cfg: mi.MLAConfig, lengths: np.ndarray) -> dict:
    """Algorithmic bytes / FLOPs of one step: the minimum traffic of the step's inputs and outputs.

    The absorbed query q_abs (written by absorb_q, read by the attend kernel) is an intermediate of
    this implementation and is not counted; nor are the split partials.
    """
    H, T, n_q = cfg.H, cfg.T, cfg.n_q
    sum_L = int(lengths.sum())
    cache = sum_L * mi.D_ROW * 2  # cached rows read (block padding is not counted)
    weights = 2 * H * mi.D_H * mi.D_C * 2
    q_in = T * H * (mi.D_H + mi.D_R) * 2
    out = T * H * mi.D_H * 2
    new_rows = T * mi.D_ROW * 2 * 2              # raw rows read + packed rows written
    core_flops = 2 * n_q * H * (mi.D_ROW + mi.D_C) * sum_L
    proj_flops = 2 * 2 * T * H * mi.D_H * mi.D_C  # absorb + up-projection
    return {
        "sum_L": sum_L,
        "core_bytes": cache,                      # per cached token: 1152 B
        "core_flops": core_flops,                 # per cached token: 2 n_q H (576 + 512)
        "step_bytes": cache + weights + q_in + out + new_rows,
        "step_flops": core_flops + proj_flops,
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(config_name: str, launch_units: int):
    """DRAM bytes per launch of the core kernel from a committed ncu summary, if current."""
    p = os.path.join(ROOT, "profiles", "decode_core_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != source_hash(CORE_SOURCES):
        return None
    ent = d.get("per_config", {}).get(config_name)
    if not ent:
        return None
    # scaled by cached tokens processed when captured on a smaller case
    return float(ent["dram_bytes_per_launch"]) * launch_units / float(ent["units"])


def roofline_of(counts: dict, core_ms: float, peaks: dict, peak_src: str, traffic) -> dict:
    """Roofline of the attend kernel: min(HBM, bf16 tensor) bound, burst peaks (the kernel is timed alone)."""
    core_s = core_ms * 1e-3
    t_bytes = counts["core_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_flops = counts["core_flops"] / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_bytes >= t_flops else "tensor"
    if bound == "hbm":
        achieved, peak, unit = counts["core_bytes"] / core_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = counts["core_flops"] / core_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    return {
        "kernel": "mla_decode_attend", "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
        "frac": round(achieved / peak, 4), "peak_source": f"{peak_src} (burst)", "traffic": traffic,
        "algorithmic_bytes": counts["core_bytes"], "algorithmic_flops": counts["core_flops"],
        "us_per_launch": round(core_ms * 1e3, 3),
        "tflops_achieved": round(counts["core_flops"] / core_s / 1e12, 2),
        "hbm_gbs_achieved": round(counts["core_bytes"] / core_s / 1e9, 1),
        "frac_vs_sustained_tensor": round(
            max(t_bytes, counts["core_flops"] / (peaks["bf16_tflops_sustained"] * 1e12)) / core_s, 4),
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons; the summary keeps the samples whose
    timestamps fall inside the window marked by mark_start() / mark_end()."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    @staticmethod
    def parse(lines, t0=None, t1=None):
        rows = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                row = {"ts": ts, "sm": float(parts[2]), "max": float(parts[3]), "power": float(parts[4]),
                       "hw": parts[6], "hwt": parts[7], "swt": parts[8], "pcap": parts[9]}
            except ValueError:
                continue
            if (t0 is None or ts >= t0) and (t1 is None or ts <= t1):
                rows.append(row)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                            ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["max"] for r in rows),
                "power_w_max": max(r["power"] for r in rows), "samples": len(rows), "reasons": sorted(reasons)}

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.parse(lines, self.t0, self.t1)


# ------------------------------------------------------------------ distributed plumbing

class Dist:
    """One process per GPU (torchrun env vars); NCCL for the barrier and the max / sum reductions.

    backend="gloo" runs the same plumbing on CPU ranks (used by the multi-process tests).
    """

    def __init__(self, gpus: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = False
        if gpus > 1 and self.world != gpus:
            raise SystemExit(f"--gpus {gpus} needs torchrun with {gpus} processes (WORLD_SIZE={self.world})")

    def _device(self, torch):
        return torch.device("cuda", self.local_rank) if self.backend == "nccl" else torch.device("cpu")

    def init(self, torch):
        if self.backend == "nccl":
            torch.cuda.set_device(self.local_rank)
        if self.world > 1:
            import torch.distributed as dist
            kw = {"device_id": self._device(torch)} if self.backend == "nccl" else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = True

    def barrier(self, torch):
        if self.pg:
            import torch.distributed as dist
            if self.backend == "nccl":
                dist.barrier(device_ids=[self.local_rank])
            else:
                dist.barrier()

    def reduce(self, torch, value: float, op: str) -> float:
        if not self.pg:
            return value
        import torch.distributed as dist
        t = torch.tensor([value], dtype=torch.float64, device=self._device(torch))
        dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def rank_config(base: mi.MLAConfig, rank: int) -> mi.MLAConfig:
    """Each rank decodes its own batch of the same shape (weak scaling): only the seed differs."""
    return mi.MLAConfig(**{**base.__dict__, "seed": base.seed + 7919 * rank})


def aggregate(dist, torch, step_ms: list, step_bytes: float) -> tuple:
    """Weak scaling: each rank times its own batch; the job's time per step is the slowest rank's,
    its work the sum over ranks.  Returns (ms_per_step, TB/s of the whole job)."""
    total_ms = dist.reduce(torch, sum(step_ms), "max")
    ms_per_step = total_ms / len(step_ms)
    bytes_all = dist.reduce(torch, float(step_bytes), "sum")
    return ms_per_step, bytes_all / (ms_per_step * 1e-3) / 1e12


def workload_name(cfg: mi.MLAConfig) -> str:
    return (f"{cfg.name}: B={cfg.B} H={cfg.H} n_q={cfg.n_q} "
            f"L={'U[1,%d]' % cfg.L_max if cfg.L is None else cfg.L} d_c=512 d_R=64 d_h=128")


# ------------------------------------------------------------------ our arm

def block_table(cfg: mi.MLAConfig, lengths: np.ndarray, n_blocks: int, torch, dev):
    """The pool's blocks handed to the sequences in a seeded random order (a paged cache as a serving
    runtime leaves it after sequences have come and gone): int32 [B, max_blocks]."""
    nblk = (lengths + 127) // 128
    perm = np.random.default_rng(cfg.seed).permutation(n_blocks).astype(np.int32)
    tab = np.zeros((cfg.B, int(nblk.max())), dtype=np.int32)
    k = 0
    for b in range(cfg.B):
        tab[b, :nblk[b]] = perm[k:k + nblk[b]]
        k += int(nblk[b])
    return torch.from_numpy(tab).to(dev)


def build_state(torch, mla, cfg: mi.MLAConfig, dev):
    lengths = mi.kv_lengths(cfg)
    starts = mi.seq_starts(lengths)  # rows of the generator's packed pool
    N = int(lengths.sum())
    nblk = (lengths + mla.BLOCK_TOKENS - 1) // mla.BLOCK_TOKENS

    def dbf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    cache = torch.zeros((int(nblk.sum()), mla.BLOCK_BYTES), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rope = mla.rope_table(int(lengths.max()), cfg.rope_base, dev)
    table = block_table(cfg, lengths, int(nblk.sum()), torch, dev)
    seq_of_row = np.repeat(np.arange(cfg.B, dtype=np.int32), lengths)
    pos_of_row = (np.arange(N, dtype=np.int64) - np.repeat(starts, lengths)).astype(np.int32)
    chunk = 1 << 18
    for r0 in range(0, N, chunk):
        n = min(chunk, N - r0)
        c, k = mi.token_rows(cfg, r0, n)
        mla.append_cache(cache, table, torch.from_numpy(seq_of_row[r0:r0 + n]).to(dev),
                         torch.from_numpy(pos_of_row[r0:r0 + n]).to(dev), dbf(c), dbf(k), rope, status)
    # the step's new tokens: the last n_q rows of every sequence
    new_rows = np.concatenate([starts[b] + lengths[b] - cfg.n_q + np.arange(cfg.n_q) for b in range(cfg.B)])
    new_c = np.concatenate([mi.token_rows(cfg, int(r), 1)[0] for r in new_rows])
    new_k = np.concatenate([mi.token_rows(cfg, int(r), 1)[1] for r in new_rows])
    new_seq = np.repeat(np.arange(cfg.B, dtype=np.int32), cfg.n_q)
    new_pos = pos_of_row[new_rows].astype(np.int32)
    qn, qr = mi.queries(cfg)
    host = {  # pinned host copies of the per-step inputs (for the end-to-end leg)
        "c_kv": torch.from_numpy(new_c.view(np.int16)).view(torch.bfloat16).pin_memory(),
        "k_rope": torch.from_numpy(new_k.view(np.int16)).view(torch.bfloat16).pin_memory(),
        "seq_idx": torch.from_numpy(new_seq).pin_memory(),
        "pos": torch.from_numpy(new_pos).pin_memory(),
        "q_nope": torch.from_numpy(qn.view(np.int16)).view(torch.bfloat16).pin_memory(),
        "q_rope": torch.from_numpy(qr.view(np.int16)).view(torch.bfloat16).pin_memory(),
    }
    devt = {k: v.to(dev) for k, v in host.items()}
    T, H = cfg.T, cfg.H
    st = {
        "lengths": lengths, "cache": cache, "status": status, "rope": rope, "block_table": table,
        "kv_len": torch.from_numpy(lengths.astype(np.int32)).to(dev),
        "W_UK": dbf(mi.weights(cfg, "uk")), "W_UV": dbf(mi.weights(cfg, "uv")),
        "host": host, "dev": devt,
        "q_abs": torch.empty((T, H, mi.D_ROW), dtype=torch.bfloat16, device=dev),
        "out": torch.empty((T, H, mi.D_H), dtype=torch.bfloat16, device=dev),
        "out_host": torch.empty((T, H, mi.D_H), dtype=torch.bfloat16).pin_memory(),
        "ws": torch.empty(mla.decode_workspace_bytes(cfg.B, cfg.n_q, H, 0), dtype=torch.uint8, device=dev),
    }
    torch.cuda.synchronize()
    return st


def step_append(mla, cfg, st):
    d = st["dev"]
    mla.append_cache(st["cache"], st["block_table"], d["seq_idx"], d["pos"], d["c_kv"], d["k_rope"], st["rope"],
                     st["status"])


def step_absorb(mla, cfg, st):
    d = st["dev"]
    mla.absorb_q(d["q_nope"], d["q_rope"], d["pos"], st["W_UK"], st["rope"], q_out=st["q_abs"],
                 dev_status=st["status"])


def step_attend(mla, cfg, st):
    mla.decode_attend(st["q_abs"], st["cache"], st["block_table"], st["kv_len"], cfg.n_q, cfg.scale, 0, st["ws"],
                      dev_status=st["status"])


def step_finish(mla, cfg, st):
    mla.decode_finish(st["block_table"], st["kv_len"], st["W_UV"], cfg.n_q, 0, st["ws"], st["out"],
                      dev_status=st["status"])


STEP_PARTS = {"append": step_append, "absorb_q": step_absorb, "decode_attend": step_attend,
              "decode_finish": step_finish}


def run_step(mla, cfg, st):
    for f in STEP_PARTS.values():
        f(mla, cfg, st)


def make_timer(torch, flush):
    """time_graph(g, n): n replays of graph g, each after an L2 flush, timed by CUDA events on the current
    stream (the one the graph's launches go to)."""
    def time_graph(g, n):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for i in range(n):
            flush.zero_()
            ev[i][0].record()
            g.replay()
            ev[i][1].record()
        torch.cuda.synchronize()
        return [e[0].elapsed_time(e[1]) for e in ev]
    return time_graph


def measure_query_up(torch, mla, cfg, dev, time_graph, n, peaks, d_cq, W_UK=None):
    """Time the compressed-query side alone, each as a CUDA graph after an L2 flush: mla_query_up
    (c^Q [T, d_c'] -> q^C, q^R) and, with W_UK, mla_query_absorb (c^Q -> the absorbed query in one launch,
    which replaces mla_query_up + mla_absorb_q).  Neither is part of the step (its queries arrive as q^C, q^R).
    Algorithmic bytes: the weights read once, c^Q in, the outputs out.
    """
    cq, wuq, wqr = mi.compressed_queries(cfg, d_cq)

    def dbf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    cq_d, wuq_d, wqr_d = dbf(cq), dbf(wuq), dbf(wqr)
    T, H = cfg.T, cfg.H
    qn = torch.empty((T, H, mi.D_H), dtype=torch.bfloat16, device=dev)
    qr = torch.empty((T, H, mi.D_R), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def timed(run):
        for _ in range(3):
            run()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            run()
        torch.cuda.synchronize()
        us = 1e3 * statistics.mean(time_graph(g, n))
        torch.cuda.synchronize()
        del g
        return us

    def line(kernel, us, nbytes, **extra):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"kernel": kernel, "d_cq": d_cq, "T": T, "H": H, "launches": n, "us_per_launch": round(us, 3),
                "algorithmic_bytes": nbytes, "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), **extra}

    us = timed(lambda: mla.query_up(cq_d, wuq_d, wqr_d, q_nope=qn, q_rope=qr, dev_status=status))
    nbytes = H * (mi.D_H + mi.D_R) * d_cq * 2 + T * d_cq * 2 + T * H * (mi.D_H + mi.D_R) * 2
    res = line("mla_query_up", us, nbytes, note="timed alone, L2 flushed before each launch; not part of the step")
    if W_UK is not None:
        pos = torch.arange(T, dtype=torch.int32, device=dev)
        tab = mla.rope_table(max(T, 1), cfg.rope_base, dev)
        qa = torch.empty((T, H, mi.D_ROW), dtype=torch.bfloat16, device=dev)
        us = timed(lambda: mla.query_absorb(cq_d, wuq_d, wqr_d, W_UK, pos, tab, q_out=qa, dev_status=status))
        nbytes = (H * (mi.D_H + mi.D_R) * d_cq * 2 + H * mi.D_H * mi.D_C * 2 + T * d_cq * 2 + T * H * mi.D_ROW * 2)
        res["fused"] = line("mla_query_absorb", us, nbytes,
                            note="c^Q -> absorbed query in one launch (= mla_query_up + mla_absorb_q)")
    if int(status.item()) != 0:
        return {"error": "device status " + mla.device_status_string(int(status.item()))}
    return res


def prefill_flops(L: int, n: int, H: int) -> dict:
    """Algorithmic FLOPs of the last n of L tokens of one sequence attending causally, in both forms.

    naive: rebuild k^C and v^C of every key and head (2 x 128 x 512 MACs), then 192 + 128 MACs per
    (query, visible key, head).  absorbed: W^UK into each query and W^UV after (2 x 128 x 512 MACs per
    (query, head)), then 576 + 512 MACs per (query, visible key, head).
    """
    visible = n * (L - n) + n * (n + 1) // 2
    return {"naive": 2 * (L * H * 2 * 128 * 512 + visible * H * (192 + 128)),
            "absorbed": 2 * (n * H * 2 * 128 * 512 + visible * H * (576 + 512))}


def measure_prefill(torch, mla, cfg, st, dev, time_graph, steps, peaks, chunks=(64, 128, 256, 512, 1024)):
    """Time one prefill chunk of n new tokens at the end of sequence 0 in both forms: mla_prefill_naive
    (decompress + attend) and, for n <= 256, the absorbed path (absorb_q + decode with n_q = n).  Each is a
    CUDA graph timed alone with L2 flushed before each launch; not part of the step."""
    L = int(st["lengths"][0])
    H = cfg.H
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    row = st["block_table"][0].contiguous()
    table1 = row.reshape(1, -1)
    kv1 = torch.full((1,), L, dtype=torch.int32, device=dev)
    res = {"L": L, "H": H, "launches": steps, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "chunks": []}

    def dbf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    def timed(run):
        for _ in range(3):
            run()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            run()
        torch.cuda.synchronize()
        us = 1e3 * statistics.mean(time_graph(g, steps))
        del g
        return us

    ws_naive = torch.empty(mla.prefill_workspace_bytes(L, H), dtype=torch.uint8, device=dev)
    for n in chunks:
        if n > L:
            continue
        qcfg = mi.MLAConfig("prefill", B=1, H=H, n_q=n, L=L, seed=cfg.seed + 991)
        qn_bits, qr_bits = mi.queries(qcfg)
        qn, qr = dbf(qn_bits), dbf(qr_bits)
        out = torch.empty((n, H, mi.D_H), dtype=torch.bfloat16, device=dev)
        f = prefill_flops(L, n, H)
        ent = {"n": n}
        us = timed(lambda: mla.prefill_naive(qn, qr, st["rope"], st["cache"], row, L, st["W_UK"], st["W_UV"],
                                             cfg.scale, workspace=ws_naive, out=out, dev_status=status))
        ent["naive_us"] = round(us, 2)
        ent["naive_tflops"] = round(f["naive"] / (us * 1e-6) / 1e12, 1)
        if n <= 256:
            pos = torch.arange(L - n, L, dtype=torch.int32, device=dev)
            qa = torch.empty((n, H, mi.D_ROW), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(mla.decode_workspace_bytes(1, n, H), dtype=torch.uint8, device=dev)

            def absorbed():
                mla.absorb_q(qn, qr, pos, st["W_UK"], st["rope"], q_out=qa, dev_status=status)
                mla.decode(qa, st["cache"], table1, kv1, st["W_UV"], n, cfg.scale, workspace=ws, out=out,
                           dev_status=status)
            us = timed(absorbed)
            ent["absorbed_us"] = round(us, 2)
            ent["absorbed_tflops"] = round(f["absorbed"] / (us * 1e-6) / 1e12, 1)
            ent["faster"] = "naive" if ent["naive_us"] < ent["absorbed_us"] else "absorbed"
        res["chunks"].append(ent)
    if int(status.item()) != 0:
        return {"error": "device status " + mla.device_status_string(int(status.item()))}
    res["note"] = ("naive: decompress k^C, v^C of all L keys then causal attention; absorbed: absorb_q + the "
                   "decode kernels with n_q = n (n <= 256); timed alone, L2 flushed before each launch")
    return res


def _check_status(mla, st):
    if int(st["status"].item()) != 0:
        raise SystemExit(f"device status {mla.device_status_string(int(st['status'].item()))}")


def e2e_serial(torch, mla, cfg, st, steps, flush) -> float:
    """End to end, one step at a time on one stream: upload, the step's library calls, read-back; each
    step after an L2 flush.  Mean ms per step."""
    h, d = st["host"], st["dev"]
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ee[i][0].record()
        for k in h:
            d[k].copy_(h[k], non_blocking=True)
        run_step(mla, cfg, st)
        st["out_host"].copy_(st["out"], non_blocking=True)
        ee[i][1].record()
    torch.cuda.synchronize()
    return sum(e[0].elapsed_time(e[1]) for e in ee) / steps


def packed(torch, like: dict, device, pin: bool):
    """One contiguous uint8 buffer with a 256-byte-aligned view per tensor of `like` (same dtypes and
    shapes), so a step's inputs move in one copy."""
    offs, total = {}, 0
    for k, t in like.items():
        offs[k] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8, device=device, pin_memory=pin)
    views = {k: buf[offs[k]:offs[k] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for k, t in like.items()}
    return buf, views


def e2e_pipelined(torch, mla, cfg, st, steps):
    """End to end as a serving loop runs it: step k's inputs go up (one copy of one packed pinned buffer)
    on one copy stream into one of two device input sets while step k-1 computes, and step k's output
    comes back on another copy stream into one of two pinned host buffers while step k+1 computes.  The
    step's library calls are replayed from a CUDA graph per input set.  Every upload and read-back is
    inside the timed region (events from before the first upload to after the last read-back).  Returns
    (mean ms per step, bytes uploaded per step)."""
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    host_buf, host_views = packed(torch, st["host"], "cpu", True)
    for k, v in st["host"].items():
        host_views[k].copy_(v)
    dev_bufs, dev_sets = zip(*(packed(torch, st["dev"], st["out"].device, False) for _ in range(2)))
    out_sets = [st["out"], torch.empty_like(st["out"])]
    host_out = [st["out_host"], torch.empty_like(st["out_host"]).pin_memory()]
    graphs = []
    for b in range(2):
        dev_bufs[b].copy_(host_buf)
        view = dict(st, dev=dev_sets[b], out=out_sets[b])
        run_step(mla, cfg, view)  # warm
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            run_step(mla, cfg, view)
        graphs.append(g)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(comp)
    s_in.wait_event(start)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i - 2 has read this input set
            dev_bufs[b].copy_(host_buf, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])  # step i - 2's output has been read back
        graphs[b].replay()
        ev_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            host_out[b].copy_(out_sets[b], non_blocking=True)
            ev_out[b].record(s_out)
    comp.wait_stream(s_out)
    end.record(comp)
    torch.cuda.synchronize()
    del graphs
    return start.elapsed_time(end) / steps, host_buf.numel()


def measure_workload(torch, mla, dist, cfg, dev, args, flush, sampler=None, headline=False) -> dict:
    """Build one workload, then time its step (CUDA graph of the 5 launches), each part alone, and the
    end-to-end leg through the public API from pinned host buffers.  All timings are CUDA events on the
    launching stream with an L2 flush before every replay; the step time is the max over ranks."""
    st = build_state(torch, mla, cfg, dev)
    counts = step_counts(cfg, st["lengths"])
    time_graph = make_timer(torch, flush)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        run_step(mla, cfg, st)
    torch.cuda.synchronize()
    _check_status(mla, st)

    # The step is replayed from a CUDA graph (the library's calls neither allocate nor synchronise), so
    # the device runs its launches back to back and host launch overhead stays out of the numbers.
    # Each kernel is also captured alone and timed the same way for the per-kernel split.
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            fn()
        return g

    g_step = capture(lambda: run_step(mla, cfg, st))
    g_parts = {name: capture(lambda f=f: f(mla, cfg, st)) for name, f in STEP_PARTS.items()}
    torch.cuda.synchronize()
    time_graph(g_step, 2)
    dist.barrier(torch)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_start()
    t_start = time.perf_counter()
    step_ms = time_graph(g_step, args.steps)
    if sampler:
        # keep the same load on the GPU until the sampler has seen about a second of it (a short timed
        # region alone would fall between two nvidia-smi samples); these replays are not timed
        while time.perf_counter() - t_start < CLOCK_WINDOW_S:
            time_graph(g_step, 20)
        sampler.mark_end()
    loaded_s = time.perf_counter() - t_start
    dist.barrier(torch)
    part_ms = {name: time_graph(g, args.steps) for name, g in g_parts.items()}
    _check_status(mla, st)
    del g_step, g_parts
    core_ms = dist.reduce(torch, statistics.mean(part_ms["decode_attend"]), "max")
    ms_per_step, value = aggregate(dist, torch, step_ms, counts["step_bytes"])
    bytes_all = dist.reduce(torch, float(counts["step_bytes"]), "sum")
    flops_all = dist.reduce(torch, float(counts["step_flops"]), "sum")
    tokens_all = dist.reduce(torch, float(counts["sum_L"]), "sum")

    e2e = None
    if not args.no_e2e:
        d2h = st["out_host"].numel() * st["out_host"].element_size()
        dist.barrier(torch)
        torch.cuda.synchronize()
        serial_ms = e2e_serial(torch, mla, cfg, st, args.steps, flush)
        dist.barrier(torch)
        torch.cuda.synchronize()
        pipe_ms, h2d = e2e_pipelined(torch, mla, cfg, st, args.steps)
        dist.barrier(torch)
        e2e_ms = dist.reduce(torch, pipe_ms, "max")
        e2e = {"value": round(bytes_all / (e2e_ms * 1e-3) / 1e12, 4), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "mode": "pipelined: every step's inputs (one packed pinned buffer) are copied up and its output "
                       "read back inside the timed region, on two copy streams with double-buffered device inputs "
                       "and outputs, so step k+1's upload and step k's read-back overlap step k's kernels (the "
                       "step's library calls replayed from a graph); no L2 flush (each workload's cache is larger "
                       "than L2, tiny excepted); serial_ms_per_step: one step at a time, six copies, eager calls, "
                       "L2 flushed",
               "serial_ms_per_step": round(dist.reduce(torch, serial_ms, "max"), 5)}
    _check_status(mla, st)

    peaks, peak_src = load_peaks()
    roofline = roofline_of(counts, core_ms, peaks, peak_src, traffic_for(cfg.name, counts["sum_L"]))
    step_roof_s = max(counts["step_bytes"] / (peaks["hbm_gbs"] * 1e9),
                      counts["step_flops"] / (peaks["bf16_tflops"] * 1e12))
    res = {
        "workload": workload_name(cfg), "lengths": st["lengths"], "counts": counts,
        "ms_per_step": ms_per_step, "value": value, "loaded_s": loaded_s,
        "us_per_step": round(ms_per_step * 1e3, 2),
        "kernel_us": {name: round(1e3 * statistics.mean(v), 2) for name, v in part_ms.items()},
        "tflops": round(flops_all / (ms_per_step * 1e-3) / 1e12, 2),
        "cache_tokens_per_s": round(tokens_all / (ms_per_step * 1e-3), 1),
        "step_roofline_frac": round(step_roof_s / (ms_per_step * 1e-3), 4),
        "roofline": roofline, "e2e": e2e,
    }
    if dist.world == 1 and not args.no_prefill and cfg.name == args.prefill_config:
        try:
            res["prefill"] = measure_prefill(torch, mla, cfg, st, dev, time_graph, min(args.steps, 50), peaks)
        except Exception as e:  # reported in the line; the step's numbers stand on their own
            res["prefill"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if headline and dist.world == 1 and not args.no_query_up:
        try:
            res["query_up"] = measure_query_up(torch, mla, cfg, dev, time_graph, min(args.steps, 1000), peaks,
                                               args.query_rank, W_UK=st["W_UK"])
        except Exception as e:  # reported in the line; the step's numbers above stand on their own
            res["query_up"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    del st
    torch.cuda.empty_cache()
    return res


def run_ours(args, dist):
    import torch
    dist.init(torch)
    import mla_latent_kv_34_b200 as mla
    dev = torch.device("cuda", dist.local_rank)
    cfg = rank_config(mi.CONFIGS[args.config], dist.rank)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = None if args.no_clocks else ClockSampler(uuid)
    if sampler:
        sampler.start()
    try:
        head = measure_workload(torch, mla, dist, cfg, dev, args, flush, sampler, headline=True)
    finally:
        clocks = sampler.stop() if sampler else None
    if clocks is not None:
        clocks["window"] = (f"the timed steps plus untimed replays of the same step graph, "
                            f"{head['loaded_s']:.2f} s of load in all")
    per_config = {}
    prefill = head.get("prefill")
    extras = [c for c in args.extra_configs.split(",") if c and c != args.config] if dist.world == 1 else []
    for name in extras:
        r = measure_workload(torch, mla, dist, rank_config(mi.CONFIGS[name], dist.rank), dev, args, flush)
        per_config[name] = {k: r[k] for k in ("workload", "us_per_step", "kernel_us", "tflops",
                                              "cache_tokens_per_s", "step_roofline_frac", "roofline", "e2e")}
        per_config[name]["value"] = round(r["value"], 4)
        if "prefill" in r:
            prefill = r["prefill"]
        per_config[name]["unit"] = UNIT

    counts = head["counts"]
    line = {
        "metric": METRIC, "value": round(head["value"], 4), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(head["ms_per_step"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, mla_inputs)",
        "config": {"workload": head["workload"], "B": cfg.B, "H": cfg.H, "n_q": cfg.n_q, "sum_L": counts["sum_L"],
                   "step": "append + absorb_q + decode_attend + decode_finish (merge, W^UV)",
                   "cache": "paged: pool blocks handed to the sequences in a seeded random order",
                   "l2": "flushed between timed steps (256 MiB write)",
                   "launch": "each timed step is one CUDA graph replay of the 5 library launches",
                   "parallelism": f"dp{args.gpus} (replicas)"},
        "us_per_step": head["us_per_step"], "kernel_us": head["kernel_us"], "tflops": head["tflops"],
        "cache_tokens_per_s": head["cache_tokens_per_s"], "step_roofline_frac": head["step_roofline_frac"],
        "roofline": head["roofline"], "e2e": head["e2e"],
        "gpu_launches": sum(KERNELS_PER_STEP.values()) * args.steps,
        "clocks": clocks,
    }
    if per_config:
        line["per_config"] = per_config
    if "query_up" in head:
        line["query_up"] = head["query_up"]
    if prefill is not None:
        line["prefill"] = prefill
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, head["lengths"], args.cpu_seconds)
    dist.close()
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the oracle as baseline / reference arm
#
# Both the cpu_baseline of our line and the reference arm time the SAME thing: the fp64 naive oracle on
# samples of the workload, each sample = one sequence, a block of ORACLE_HEADS heads, all its query
# tokens.  Samples cycle through the sequences (and head blocks) in a fixed order.  The oracle's cost is
# linear in (cached tokens x heads); its rate over the samples gives the full step's time, and `value` is
# the step's algorithmic bytes over that time (the same unit as our arm's value).

def cpu_info() -> dict:
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count() or 1, "cpu_model": model}


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=1)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_plan(cfg: mi.MLAConfig, lengths: np.ndarray, i: int) -> tuple:
    """Sample i: (sequence, heads).  Sequences in index order, then the next head block."""
    b = i % cfg.B
    nh = min(ORACLE_HEADS, cfg.H)
    h0 = (nh * (i // cfg.B)) % cfg.H
    heads = [(h0 + k) % cfg.H for k in range(nh)]
    return b, heads


class OracleTimer:
    """Times the fp64 naive oracle on samples of one workload (weights widened once)."""

    def __init__(self, cfg: mi.MLAConfig, lengths: np.ndarray):
        self.cfg, self.lengths = cfg, lengths
        f = mi.bf16_bits_to_f64
        self.Wk, self.Wv = f(mi.weights(cfg, "uk")), f(mi.weights(cfg, "uv"))

    def sample(self, i: int) -> tuple:
        """Returns (seconds, units = cached tokens x heads) of sample i."""
        from oracle import naive as on
        cfg = self.cfg
        b, heads = oracle_sample_plan(cfg, self.lengths, i)
        s = mi.sequence(cfg, b, self.lengths)
        f = mi.bf16_bits_to_f64
        args = (f(s.c_kv), f(s.k_rope), f(s.q_nope), f(s.q_rope), self.Wk, self.Wv, cfg.n_q)
        t = time.perf_counter()
        on.attend_naive(*args, scale=cfg.scale, base=cfg.rope_base, heads=heads)
        return time.perf_counter() - t, int(self.lengths[b]) * len(heads)


def oracle_rate_line(cfg, lengths, secs: list, units: list) -> dict:
    counts = step_counts(cfg, lengths)
    per_unit = sum(secs) / max(sum(units), 1)
    full_s = per_unit * counts["sum_L"] * cfg.H
    return {"value": counts["step_bytes"] / full_s / 1e12, "full_step_s": full_s,
            "sample_s": statistics.mean(secs), "n": len(secs)}


def cpu_baseline(cfg, lengths, target_s: float):
    timer = OracleTimer(cfg, lengths)
    secs, units = [], []
    t0 = time.perf_counter()
    i = 0
    while i < 3 or (time.perf_counter() - t0 < target_s and i < 10 * cfg.B):
        s, u = timer.sample(i)
        secs.append(s)
        units.append(u)
        i += 1
    r = oracle_rate_line(cfg, lengths, secs, units)
    return {"value": round(r["value"], 8), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle", **cpu_info(),
            "sample": f"fp64 naive oracle on {r['n']} samples (one sequence x {min(ORACLE_HEADS, cfg.H)} heads x "
                      f"all queries each, {sum(secs):.1f} s); rate per (cached token x head) scaled to the full "
                      f"step: {r['full_step_s']:.4g} s/step",
            "extrapolated_full_step_s": round(r["full_step_s"], 4)}


def run_reference(args, dist):
    if dist.rank != 0:
        return
    cfg = mi.CONFIGS[args.config]
    lengths = mi.kv_lengths(cfg)
    timer = OracleTimer(cfg, lengths)
    for i in range(args.warmup):
        timer.sample(i)
    secs, units = [], []
    for i in range(args.warmup, args.warmup + args.steps):
        s, u = timer.sample(i)
        secs.append(s)
        units.append(u)
    r = oracle_rate_line(cfg, lengths, secs, units)
    value = round(r["value"], 8)
    sample = (f"each step: the fp64 naive oracle on one sequence x {min(ORACLE_HEADS, cfg.H)} heads x all queries "
              f"(mean {r['sample_s']:.3f} s); rate per (cached token x head) scaled to the full step: "
              f"{r['full_step_s']:.4g} s/step")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(r["sample_s"] * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, mla_inputs)",
        "config": {"workload": workload_name(cfg), "B": cfg.B, "H": cfg.H, "n_q": cfg.n_q,
                   "sum_L": int(lengths.sum()),
                   "step": "one bounded oracle sample of the workload (ms_per_step is its measured time)"},
        "impl": "reference",
        "extrapolated_full_step_s": round(r["full_step_s"], 4),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle", **cpu_info(),
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 200
    dist = Dist(args.gpus)
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        run_ours(args, dist)


if __name__ == "__main__":
    main()
