"""Benchmark: prefill unmasked TFLOP/s (and decode HBM GB/s) of the attention
core on B200, as a fraction of the measured peaks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--no-decode] [--only LEG]

One step = one swa_attn_prefill call (RoPE of the keys, then the fused
tcgen05 attention kernel with RoPE on the Q tile load, causal mask, online
softmax, P.V and the head gate) over one batch of the largest single-GPU
workload, the Step-3.7-Flash full-attention layer (B1 S32768 Hq64 Hkv8,
causal, theta 5e6 on the first 64 dims).  Inputs are resident in HBM and
rotate over 4 copies (1.2 GB each, far more than the 126 MB L2), so no step
reads the previous step's data from L2.

Beside the headline, the same line carries the other three prefill
workloads (the Step sliding layer and the Muse sliding / full layers), each
timed the same way, and the decode, multi-query decode and continued-prefill
legs.

With torchrun (N > 1) every rank runs the same workload on its own GPU (the
work shards by sequence / kv-head with no exchange; weak scaling); time is
the max over ranks of the device-timed region.

--impl reference times the CPU oracle (the plain fp64 definition, OpenMP over
rows) on a bounded row sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from full_gqa_attention_swa_b200 import configs, inputs  # noqa: E402

METRIC = "prefill unmasked TFLOP/s & decode HBM GB/s, as fraction of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
N_ROTATE = 4


# --------------------------------------------------------------- arithmetic

def visible_pairs(S: int, window: int) -> int:
    """Number of (i, j) with j visible to i: i-W < j <= i (W<0: j <= i)."""
    if window < 0 or window >= S:
        return S * (S + 1) // 2
    W = window
    return W * (W + 1) // 2 + (S - W) * W


def chunk_visible_pairs(pos0: int, S: int, window: int) -> int:
    """Visible (i, j) pairs of query rows pos0 .. pos0 + S - 1."""
    return visible_pairs(pos0 + S, window) - visible_pairs(pos0, window)


def chunk_flops(c) -> float:
    return 4.0 * 128 * c.Hq * c.B * chunk_visible_pairs(c.pos0, c.S, c.window)


def prefill_flops(c) -> float:
    """Unmasked FLOPs: QK^T and P.V over visible pairs, 2 * 2 * D each."""
    return 4.0 * 128 * c.Hq * c.B * visible_pairs(c.S, c.window)


def prefill_bytes(c) -> int:
    """Algorithmic HBM bytes: read Q, K, V, gate; write out."""
    q = c.B * c.S * c.Hq * 128 * 2
    kv = 2 * c.B * c.S * c.Hkv * 128 * 2
    gate = c.B * c.S * c.Hq * 4
    return 2 * q + kv + gate


def decode_bytes(c, lens) -> int:
    """Cache bytes read once per kv-head (K and V) plus q, gate and out."""
    W = c.window
    keys = sum(min(int(L), W) if W > 0 else int(L) for L in lens)
    return keys * c.Hkv * 128 * 2 * 2 + c.B * c.Hq * (128 * 2 * 2 + 4)


def decode_mq_bytes(c, lens) -> int:
    """Multi-query decode: the cached keys (the L - T earlier tokens, at most
    W on a ring) read once per kv-head as K and V, plus q, gate and out of the
    T new tokens and their k / v."""
    W = c.window
    ctx = [int(L) - c.T for L in lens]
    keys = sum(min(n, W) if W > 0 else n for n in ctx)
    return keys * c.Hkv * 128 * 2 * 2 + c.B * c.T * (c.Hq * (128 * 2 * 2 + 4) + c.Hkv * 128 * 2 * 2)


# DRAM traffic per launch of the prefill attention kernel from ncu captures
# (dram__bytes_read.sum + dram__bytes_write.sum, one launch per workload; the
# summaries under profiles/).  A figure describes only the kernel source it was
# taken on, so it is reported only while csrc/prefill.cuh and csrc/ptx.cuh still
# hash to the recorded digest, else null.
PREFILL_TRAFFIC = {
    # prefill.cuh and ptx.cuh as captured; any change makes the figures stale
    "source_sha256": "0655f30c06d1c348b18a77fad0b06b7992028d6865f28fc5a29449d239a48043",
    "bytes": {"step37_sliding_B1_S8192_Hq96_Hkv8_W512": 399.4e6,
              "step37_full_B1_S32768_Hq64_Hkv8_causal": 4368.3e6,
              "muse_sliding_B4_S16384_Hq32_Hkv2_W2048": 1116.2e6,
              "muse_full_B4_S16384_Hq32_Hkv2_causal_norope": 1754.3e6},
}
PREFILL_SOURCES = ("prefill.cuh", "ptx.cuh")


def prefill_source_digest():
    import hashlib
    h = hashlib.sha256()
    for name in PREFILL_SOURCES:
        with open(os.path.join(ROOT, "full_gqa_attention_swa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_prefill_traffic(workload: str):
    if workload in PREFILL_TRAFFIC["bytes"] and prefill_source_digest() == PREFILL_TRAFFIC["source_sha256"]:
        return PREFILL_TRAFFIC["bytes"][workload]
    return None


# idle before each extra prefill leg of the default run (seconds)
LEG_IDLE_S = 2.0


# B200 spec sheet (dense, no sparsity) figures, reported beside the measured
# peaks: bf16 tensor 2.25 PFLOP/s; HBM3e 7.7 TB/s (HGX board figure)
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 7700.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: every rank takes part (same collective, same
    order) and every rank gets the maximum."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def combine_ranks(elapsed_ms_per_rank, n_gpus: int, units_per_rank: float):
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    t = max(elapsed_ms_per_rank)
    return n_gpus * units_per_rank / (t / 1e3), t


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.nv = None
        if index < 0:
            return
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no samples
            self.nv = None

    def _sample(self):
        mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        try:
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append(mhz)
        for bit, name in self.REASONS.items():
            if r & bit and bit != 0x1:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self.nv:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- GPU legs

def _layer(c):
    from full_gqa_attention_swa_b200 import api

    return api.LayerParams(c.Hq, c.Hkv, 128, c.window, c.theta, c.rotary_dim)


def bench_prefill(c, steps: int, warmup: int, dev, dist=None, n_rotate: int = N_ROTATE, clocks_on: bool = True):
    from full_gqa_attention_swa_b200 import api

    p = _layer(c)
    sets = [inputs.prefill_inputs(c.B, c.S, c.Hq, c.Hkv, 128, c.seed + 17 * r, device=dev)
            for r in range(n_rotate)]
    out = torch.empty(c.B, c.S, c.Hq, 128, dtype=torch.bfloat16, device=dev)
    ws_bytes = api.prefill_workspace_size(p, c.B, c.S)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        d = sets[i % n_rotate]
        api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"], out=out, workspace=ws, stream=stream)

    for i in range(max(warmup, 0)):
        step(i)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if clocks_on else -1) as clocks:
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for i in range(steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    launches = steps * (2 if ws_bytes > 0 else 1)
    del sets
    torch.cuda.empty_cache()
    return ms, clocks.summary(), launches


def bench_prefill_chunk(c, steps: int, warmup: int, dev):
    """Continued prefill: each step runs swa_attn_prefill_chunk on the same
    chunk against a cache holding positions < pos0 (synthetic N(0,1) keys
    and values); the chunk re-appends itself each step.  Two input sets
    rotate (the full layer's cache of 134 MB alone exceeds L2)."""
    from full_gqa_attention_swa_b200 import api

    p = api.LayerParams(c.Hq, c.Hkv, 128, c.window, c.theta, c.rotary_dim)
    C = c.window if c.window > 0 else c.pos0 + c.S
    sets = []
    for r in range(2):
        d = inputs.prefill_inputs(c.B, c.S, c.Hq, c.Hkv, 128, c.seed + 31 * r, device=dev)
        cache = inputs.decode_inputs(c.B, c.Hq, c.Hkv, 128, C, c.seed + 31 * r + 7, device=dev)
        d["k_cache"], d["v_cache"] = cache["k_cache"], cache["v_cache"]
        sets.append(d)
    out = torch.empty(c.B, c.S, c.Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(api.prefill_chunk_workspace_size(p, c.B, c.S, c.pos0), 1), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        d = sets[i % 2]
        api.attn_prefill_chunk(p, c.pos0, d["q"], d["k"], d["v"], d["gate"], d["k_cache"], d["v_cache"], out=out,
                               workspace=ws, stream=stream)

    for i in range(max(warmup, 3)):
        step(i)
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    ms = ev0.elapsed_time(ev1) / steps
    assert api.device_error() == 0, "a kernel reported a bounded-wait timeout"
    del sets
    torch.cuda.empty_cache()
    return ms


def bench_prefill_e2e(c, steps: int, dev):
    """Same metric through the public API with host buffers: every step copies
    its pinned host inputs in and its output back.  Steps are pipelined as a
    serving loop would run them: two device buffer sets, the next step's
    host->device copy on one stream, attention on the current stream, the
    device->host copy of the result on a third (the link is full duplex)."""
    from full_gqa_attention_swa_b200 import api

    p = _layer(c)
    host = inputs.prefill_inputs(c.B, c.S, c.Hq, c.Hkv, 128, c.seed)
    host = {k: t.pin_memory() for k, t in host.items()}
    out_host = torch.empty(c.B, c.S, c.Hq, 128, dtype=torch.bfloat16).pin_memory()
    bufs = [{k: torch.empty_like(t, device=dev) for k, t in host.items()} for _ in range(2)]
    outs = [torch.empty(c.B, c.S, c.Hq, 128, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = torch.empty(max(api.prefill_workspace_size(p, c.B, c.S), 1), dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]   # attention on buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output of buffer b copied back
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    n = [0]

    def step():
        b = n[0] % 2
        if n[0] >= 2:
            s_in.wait_event(ev_done[b])        # attention of two steps ago no longer reads bufs[b]
        with torch.cuda.stream(s_in):
            for k in host:
                bufs[b][k].copy_(host[k], non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if n[0] >= 2:
            comp.wait_event(ev_out[b])         # outs[b] of two steps ago has been read back
        d = bufs[b]
        api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"], out=outs[b], workspace=ws, stream=comp)
        ev_done[b].record(comp)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            out_host.copy_(outs[b], non_blocking=True)
            ev_out[b].record(s_out)
        n[0] += 1

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(comp)
    s_in.wait_event(ev0)
    for _ in range(steps):
        step()
    comp.wait_event(ev_out[(n[0] - 1) % 2])    # the last result is on the host
    ev1.record(comp)
    torch.cuda.synchronize(dev)
    return ev0.elapsed_time(ev1), h2d, d2h


def time_calls(run, steps: int, warmup: int, stream):
    """Device time per call of `run(i)`, i = 0 .. steps - 1: launched eagerly,
    and replayed from a CUDA graph of the same `steps` calls (how a serving
    loop issues decode steps: no per-call host work between the kernels).
    Returns (ms_graph, ms_eager)."""
    for i in range(max(warmup, 3)):
        run(i)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        run(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    eager = ev0.elapsed_time(ev1) / steps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            run(i)
    g.replay()
    torch.cuda.synchronize()
    ev0.record(stream)
    g.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    graph = ev0.elapsed_time(ev1) / steps
    del g
    return graph, eager


def bench_decode(c, steps: int, warmup: int, dev):
    from full_gqa_attention_swa_b200 import api

    p = _layer(c)
    lens = inputs.uniform_int(c.B, c.len_lo, c.len_hi, c.seed)
    # full layers: caches far larger than L2, one copy; sliding rings (134 MB,
    # about L2-sized): rotate 4 copies
    n_sets = 1 if c.window < 0 else N_ROTATE
    sets = [inputs.decode_inputs(c.B, c.Hq, c.Hkv, 128, c.capacity, c.seed + r, device=dev) for r in range(n_sets)]
    lens_d = lens.to(dev)
    max_len = int(lens.max())
    out = torch.empty(c.B, c.Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(api.decode_workspace_size(p, c.B, max_len), 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        d = sets[i % n_sets]
        api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_d, max_len, out=out, workspace=ws)

    ms, ms_eager = time_calls(step, steps, warmup, stream)
    nbytes = decode_bytes(c, lens.tolist())
    del sets
    torch.cuda.empty_cache()
    return ms, nbytes, ms_eager


def bench_decode_mq(c, steps: int, warmup: int, dev):
    from full_gqa_attention_swa_b200 import api

    p = _layer(c)
    lens = inputs.uniform_int(c.B, c.len_lo, c.len_hi, c.seed)
    n_sets = 1 if c.window < 0 else N_ROTATE
    sets = []
    for r in range(n_sets):
        d = inputs.decode_inputs(c.B, c.Hq, c.Hkv, 128, c.capacity, c.seed + r, device=dev)
        new = inputs.prefill_inputs(c.B, c.T, c.Hq, c.Hkv, 128, c.seed + 100 + r, device=dev)
        sets.append((d, new))
    lens_d = lens.to(dev)
    max_len = int(lens.max())
    out = torch.empty(c.B, c.T, c.Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(api.decode_mq_workspace_size(p, c.B, c.T, max_len), 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        d, new = sets[i % n_sets]
        api.attn_decode_mq(p, new["q"], new["gate"], new["k"], new["v"], d["k_cache"], d["v_cache"], lens_d,
                           max_len, out=out, workspace=ws)

    ms, ms_eager = time_calls(step, steps, warmup, stream)
    nbytes = decode_mq_bytes(c, lens.tolist())
    del sets
    torch.cuda.empty_cache()
    return ms, nbytes, ms_eager


# --------------------------------------------------------------- CPU oracle

def oracle_sample_rate(c, budget_s: float, threads: int = 0):
    """Time the oracle on a growing seeded row sample of the workload until
    about budget_s seconds; returns (TFLOP/s, rows, seconds, threads)."""
    import oracle

    lay = oracle.Layer(c.Hq, c.Hkv, 128, c.window, c.theta, c.rotary_dim)
    d = inputs.prefill_inputs(c.B, c.S, c.Hq, c.Hkv, 128, c.seed)
    qb, kb, vb = (inputs.as_bits(d[k]) for k in ("q", "k", "v"))
    g = d["gate"].numpy()
    rng = np.random.default_rng(c.seed)
    n = 64
    while True:
        rows = np.stack([rng.integers(0, c.B, n), rng.integers(0, c.S, n), rng.integers(0, c.Hq, n)], 1)
        t0 = time.perf_counter()
        oracle.prefill(lay, qb, kb, vb, g, rows=rows, threads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n >= 1 << 20:
            break
        n = int(n * min(8.0, max(2.0, budget_s / max(dt, 1e-3))))
    W = c.window
    pairs = sum(min(int(i) + 1, W) if W > 0 else int(i) + 1 for i in rows[:, 1])
    flops = 4.0 * 128 * pairs
    return flops / dt / 1e12, n, dt, (threads or oracle.num_threads())


def oracle_parity_sample(c, dev, n_rows: int = 512) -> dict:
    """Part of the CPU-baseline leg: the timed workload's first input set once
    more through swa_attn_prefill, and the oracle on a seeded sample of its
    rows; returns the worst and the RMS |gpu - oracle| and how many elements
    exceed the parity tolerance."""
    import oracle
    from full_gqa_attention_swa_b200 import api

    p = _layer(c)
    d = inputs.prefill_inputs(c.B, c.S, c.Hq, c.Hkv, 128, c.seed, device=dev)   # set 0 of the timed loop
    out = api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"])
    torch.cuda.synchronize(dev)
    rng = np.random.default_rng(c.seed + 1)
    rows = np.stack([rng.integers(0, c.B, n_rows), rng.integers(0, c.S, n_rows), rng.integers(0, c.Hq, n_rows)], 1)
    lay = oracle.Layer(c.Hq, c.Hkv, 128, c.window, c.theta, c.rotary_dim)
    ref = oracle.prefill(lay, inputs.as_bits(d["q"].cpu()), inputs.as_bits(d["k"].cpu()), inputs.as_bits(d["v"].cpu()),
                         d["gate"].cpu().numpy(), rows=rows)
    idx = [torch.from_numpy(rows[:, i]).to(dev) for i in range(3)]
    got = out[idx[0], idx[1], idx[2]].float().cpu().double().numpy()
    err = np.abs(got - ref)
    return {"rows": n_rows, "max_abs_err": float(err.max()), "rms_err": float(np.sqrt((err ** 2).mean())),
            "out_of_tolerance": int((err > 1e-2 + 1e-2 * np.abs(ref)).sum()), "tolerance": "1e-2 + 1e-2 |oracle|"}


# --------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default=configs.STEP_FULL.name, choices=sorted(configs.PREFILL))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode_sliding", "decode_full", "chunk_sliding",
                                       "chunk_full", "decode_mq_sliding", "decode_mq_full"], default="all",
                    help="run one leg only (profiling); prints that leg's own JSON line")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rotate", type=int, default=N_ROTATE,
                    help="input sets the prefill steps rotate over (fewer: a smaller device footprint, for profiling)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="with --only decode_*: run that layer with this many sequences (profiling a capped case)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    c = configs.PREFILL[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    flops = prefill_flops(c)
    cfg = {"workload": c.name, "global_batch": c.B * world, "seq_len": c.S, "q_heads": c.Hq, "kv_heads": c.Hkv,
           "head_dim": 128, "window": c.window, "rope_theta": c.theta, "rotary_dim": c.rotary_dim,
           "parallelism": f"replicas{world}" if world > 1 else "single",
           "l2": f"rotating {max(args.rotate, 1)} input sets of {prefill_bytes(c) / 1e6:.0f} MB (> 126 MB L2)"}

    if args.impl == "reference":
        if rank != 0:
            return
        rates = []
        for _ in range(max(args.warmup, 0)):
            oracle_sample_rate(c, 0.5)
        t_all = 0.0
        for _ in range(max(args.steps, 1)):
            r, n, dt, thr = oracle_sample_rate(c, min(2.0, 60.0 / max(args.steps, 1)))
            rates.append(r)
            t_all += dt
        v = float(np.mean(rates))
        sample = f"seeded random (b, i, h) rows of {c.name}, ~{n} rows per step"
        line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * t_all / max(args.steps, 1), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
                "impl": "reference",
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    from full_gqa_attention_swa_b200 import api

    api.load()
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()

    if args.only.startswith("chunk"):
        cc = configs.CHUNK_SLIDING if args.only == "chunk_sliding" else configs.CHUNK_FULL
        c_ms = bench_prefill_chunk(cc, max(args.steps, 1), max(args.warmup, 3), dev)
        c_ms = max_over_ranks(c_ms, dist, dev)
        tf = chunk_flops(cc) * world / (c_ms / 1e3) / 1e12
        if rank == 0:
            print(json.dumps({"metric": "continued prefill unmasked TFLOP/s", "value": tf, "unit": "TFLOP/s",
                              "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
                              "ms_per_step": c_ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                              "config": {"workload": cc.name},
                              "roofline": {"bound": "tensor", "achieved": tf / world, "peak": peaks["bf16_tflops"],
                                           "unit": "TFLOP/s", "frac": tf / world / peaks["bf16_tflops"],
                                           "traffic": None}}), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    if args.only.startswith("decode"):
        mq = args.only.startswith("decode_mq")
        if mq:
            dc = configs.MQ_SLIDING if args.only == "decode_mq_sliding" else configs.MQ_FULL
        else:
            dc = configs.DECODE_SLIDING if args.only == "decode_sliding" else configs.DECODE_FULL
        if args.decode_batch > 0:
            import dataclasses

            dc = dataclasses.replace(dc, B=args.decode_batch, name=f"{dc.name}_capped_B{args.decode_batch}")
        if dist is not None:
            dist.barrier()
        run = bench_decode_mq if mq else bench_decode
        d_ms, nbytes, _ = run(dc, max(args.steps, 1), max(args.warmup, 3), dev)
        d_ms = max_over_ranks(d_ms, dist, dev)
        gbs = nbytes * world / (d_ms / 1e3) / 1e9
        if rank == 0:
            print(json.dumps({"metric": "decode HBM GB/s", "value": gbs, "unit": "GB/s", "n_gpus": world,
                              "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": d_ms,
                              "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                              "config": {"workload": dc.name},
                              "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                           "frac": gbs / world / peaks["hbm_gbs"], "traffic": None}}), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    ms, clocks, launches = bench_prefill(c, args.steps, max(args.warmup, 3), dev, dist, n_rotate=max(args.rotate, 1))
    ms = max_over_ranks(ms, dist, dev)
    value, _ = combine_ranks([ms], world, flops * args.steps / 1e12)   # TFLOP/s over all ranks
    per_step_ms = ms / args.steps
    achieved = flops / (per_step_ms / 1e3) / 1e12
    assert api.device_error() == 0, "a kernel reported a bounded-wait timeout"

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": per_step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic N(0,1) bf16 q/k/v, N(0,1) fp32 gate logits (seeded)", "config": cfg,
            "clocks": clocks, "gpu_launches": launches}
    line["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": achieved / peaks["bf16_tflops"], "traffic": measured_prefill_traffic(c.name),
                        "frac_of_spec": achieved / SPEC_PEAKS["bf16_tflops"],
                        "peak_source": f"{peak_src} bf16 burst",
                        # the timed loop runs for seconds at the power cap, like the
                        # sustained GEMM figure: that fraction too, for reference
                        "peak_sustained": peaks["bf16_tflops_sustained"],
                        "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
                        "kernel": "swa_attn_prefill (key-RoPE pre-pass + attention kernel), CUDA events"}
    if not args.no_e2e:
        # every rank runs its own end-to-end loop at the same time (they share
        # the host's links); the slowest rank's time counts
        e2e_steps = max(3, min(args.steps, 30))
        if dist is not None:
            dist.barrier()
        e_ms, h2d, d2h = bench_prefill_e2e(c, e2e_steps, dev)
        e_ms = max_over_ranks(e_ms, dist, dev)
        line["e2e"] = {"value": flops * e2e_steps * world / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if rank == 0:
        # the extra legs and the CPU baseline describe one GPU: single-process runs only
        if world == 1 and args.only == "all":
            # the other prefill workloads, each timed like the headline
            # (rotating input sets, CUDA events around the steps, clocks
            # sampled).  Each starts after LEG_IDLE_S of idle: right after
            # the headline's kilowatt steps the power controller still holds
            # the SM clock down, and a short leg would be timed in that tail.
            legs = {}
            for pc in (configs.STEP_SLIDING, configs.STEP_FULL, configs.MUSE_SLIDING, configs.MUSE_FULL):
                if pc.name == c.name:
                    p_ms, p_steps, p_clk = ms, args.steps, clocks
                else:
                    p_steps = max(5, min(200, int(200.0 / max(prefill_flops(pc) / 1e12, 1e-3))))
                    time.sleep(LEG_IDLE_S)
                    p_ms, p_clk, _ = bench_prefill(pc, p_steps, 3, dev, n_rotate=max(args.rotate, 1))
                tf = prefill_flops(pc) / (p_ms / p_steps / 1e3) / 1e12
                legs[pc.name] = {"ms": p_ms / p_steps, "steps": p_steps, "TFLOP/s": tf,
                                 "frac_bf16": tf / peaks["bf16_tflops"], "frac_of_spec": tf / SPEC_PEAKS["bf16_tflops"],
                                 "peak_source": f"{peak_src} bf16 burst", "unmasked_flop": prefill_flops(pc),
                                 "traffic": measured_prefill_traffic(pc.name), "clocks": p_clk,
                                 "timing": "swa_attn_prefill (key pre-pass + attention), CUDA events"
                                           + ("" if pc.name == c.name else f", after {LEG_IDLE_S:g} s idle")}
            line["prefill"] = legs
            assert api.device_error() == 0, "a kernel reported a bounded-wait timeout"
        if world == 1 and not args.no_decode and args.only == "all":
            # the short legs first, the two 34 GB full-layer decode legs last
            chunks = {}
            for cc in (configs.CHUNK_SLIDING, configs.CHUNK_FULL):
                time.sleep(LEG_IDLE_S)
                c_ms = bench_prefill_chunk(cc, 20 if cc.window > 0 else 5, 3, dev)
                tf = chunk_flops(cc) / (c_ms / 1e3) / 1e12
                chunks[cc.name] = {"ms": c_ms, "TFLOP/s": tf, "frac_bf16": tf / peaks["bf16_tflops"],
                                   "frac_of_spec": tf / SPEC_PEAKS["bf16_tflops"],
                                   "peak_source": f"{peak_src} bf16 burst",
                                   "timing": f"CUDA events, after {LEG_IDLE_S:g} s idle"}
            extra, mqs = {}, {}
            for kind, dc in (("decode", configs.DECODE_SLIDING), ("mq", configs.MQ_SLIDING),
                             ("decode", configs.DECODE_FULL), ("mq", configs.MQ_FULL)):
                steps = 200 if dc.window > 0 else 10
                d_ms, nbytes, e_ms = (bench_decode if kind == "decode" else bench_decode_mq)(dc, steps, 3, dev)
                gbs = nbytes / (d_ms / 1e3) / 1e9
                (extra if kind == "decode" else mqs)[dc.name] = {
                    "ms": d_ms, "ms_eager": e_ms, "timing": "CUDA graph replay of the steps (ms_eager: launched one by one)",
                    "bytes": nbytes, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                    "frac_of_spec": gbs / SPEC_PEAKS["hbm_gbs"],
                    "peak_source": f"{peak_src} hbm copy"}
            line["decode"] = extra
            line["decode_mq"] = mqs
            line["prefill_chunk"] = chunks
        if world == 1 and args.cpu_budget > 0:
            r, n, dt, thr = oracle_sample_rate(c, args.cpu_budget)
            line["cpu_baseline"] = {"value": r, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                    "sample": f"{n} seeded random (b, i, h) rows of {c.name}, {dt:.1f} s",
                                    "parity_sample": oracle_parity_sample(c, dev)}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
