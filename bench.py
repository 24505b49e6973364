#!/usr/bin/env python
"""Benchmark of the Ulysses SP hot path on B200 (one JSON line on rank 0).

One step = the whole path on one batch of seeded synthetic input already in
HBM:  seq_to_head(q, k, v) -> attention forward -> head_to_seq(O);
seq_to_head(dO) -> attention backward -> head_to_seq(dQ, dK, dV).
Outputs are stored fp32 (the precision the parity tests gate).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --profile-case      # one small fwd + bwd for ncu captures

`value` is the algorithmic fwd+bwd attention FLOP rate of the whole step
(12 * d * H_q * pairs per step, pairs = sum over samples of L(L+1)/2, i.e.
only key/query pairs the causal, sample-segmented mask allows), over all
ranks.  Under torchrun each GPU runs its own copy of the workload (weak
scaling, no data-path collective); time is the max over ranks.
`--impl reference` times the CPU fp64 oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "causal attn TFLOP/s fwd & fwd+bwd (% bf16 peak); re-layout GB/s (% HBM)"
DEFAULT_WORKLOAD = "roundtrip_p4_n128k"


# DRAM traffic per launch of a kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum, --print-units base) of the
# named workload.  It applies only while the kernel's sources hash to the
# value recorded with it; otherwise traffic is null.
KERNEL_SOURCES = {
    # kernel -> (file, first line of its source region or None for the whole file, ...)
    "attn_bwd_dkdv_kernel": (("ulysses_head_attention_b200/csrc/attn_bwd.cu", "namespace dkdv {", "}  // namespace dkdv"),
                             ("ulysses_head_attention_b200/csrc/sm100.cuh", None, None),
                             ("ulysses_head_attention_b200/csrc/common.cuh", None, None)),
    "attn_bwd_dq_kernel": (("ulysses_head_attention_b200/csrc/attn_bwd.cu", "namespace dq {", "}  // namespace dq"),
                           ("ulysses_head_attention_b200/csrc/sm100.cuh", None, None),
                           ("ulysses_head_attention_b200/csrc/common.cuh", None, None)),
    "attn_fwd_kernel": (("ulysses_head_attention_b200/csrc/attn_fwd.cu", "namespace fwd {", "}  // namespace fwd"),
                        ("ulysses_head_attention_b200/csrc/sm100.cuh", None, None),
                        ("ulysses_head_attention_b200/csrc/common.cuh", None, None)),
}
# kernel -> {"workload", "bytes_per_launch", "sources_sha256"}
TRAFFIC = {
    "attn_bwd_dkdv_kernel": {"workload": "roundtrip_p4_n128k", "bytes_per_launch": 10050001152,
                            "sources_sha256": "25ba9ffc0dea0c17d52ac7cfe2889817052ba88dd6947055c6bf0849e6766407"},
    "attn_bwd_dq_kernel": {"workload": "roundtrip_p4_n128k", "bytes_per_launch": 7764684288,
                          "sources_sha256": "f92c9d5fccec072838f206836a167345d7f35ac885823a480f515ec27b22d589"},
    "attn_fwd_kernel": {"workload": "roundtrip_p4_n128k", "bytes_per_launch": 5586175744,
                       "sources_sha256": "c55d43ca904be9c95352be16bee5dd11ca9c663aed6b9ddc1ede2dce789570bc"},
}


def sources_sha256(kernel: str) -> str:
    """Hash of the kernel's own source region and the headers it uses."""
    import hashlib
    h = hashlib.sha256()
    for rel, begin, end in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        if begin is not None:
            text = text[text.index(begin):text.index(end)]
        h.update(text.encode())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    rec = TRAFFIC.get(kernel)
    if rec is None or rec["workload"] != workload or rec["sources_sha256"] != sources_sha256(kernel):
        return None
    return rec["bytes_per_launch"]


# ----------------------------------------------------------------------------- multi-rank plumbing
def max_over_ranks(val: float, world: int, device=None) -> float:
    """Max of `val` over all ranks of the default process group (identity at world 1).
    NCCL groups need `device` (the rank's GPU); gloo groups take the CPU default."""
    if world == 1:
        return float(val)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(val)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job rate: every rank runs its own copy of the step (weak scaling),
    and the step time is the slowest rank's."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def reports(rank: int) -> bool:
    """Only rank 0 prints the JSON line."""
    return rank == 0


def pairs_of(lengths):
    return sum(L * (L + 1) // 2 for row in lengths for L in row)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 50 ms) of SM clock and clock-event reasons,
    kept with their host time stamps; summary(t0, t1) reports the samples
    read inside one timed window."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.sw_power_cap,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.active")
    # NVML clock-event reason bits, for the names of whatever else is active
    BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.1)   # let the last in-window line arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons, masks = [], None, set(), set()
        names = ("sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
        for t, ln in list(self.lines):
            if not (t0 <= t <= t1 + 0.06):
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(nm)
            try:
                mask = int(parts[7], 16)
            except ValueError:
                continue
            masks.add(mask)
            for bit, nm in self.BITS.items():
                if mask & bit:
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "sm_mhz_min": min(sm) if sm else None, "sm_mhz_max": max(sm) if sm else None,
                "reasons": sorted(reasons), "active_masks": sorted(hex(m) for m in masks), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_sample(w, x, rows: int, heads: int):
    """fwd + bwd of the CPU oracle on the last `rows` query rows of `heads`
    query heads (their full visible key ranges).  Returns (flops, seconds)."""
    import oracle
    q = synthetic.bf16_bits_to_f64(x["q"][0])
    k = synthetic.bf16_bits_to_f64(x["k"][0])
    v = synthetic.bf16_bits_to_f64(x["v"][0])
    do = synthetic.bf16_bits_to_f64(x["do"][0]) if "do" in x else None
    ss = oracle.segment_starts(x["position_ids"])[0]
    rows = min(rows, w.n)
    lo = w.n - rows
    visible = int(sum(i - ss[i] + 1 for i in range(lo, w.n)))
    scale = oracle.default_scale(w.d)
    t0 = time.perf_counter()
    for h in range(heads):
        g = h // w.group
        oracle.attention_fwd_head(q[:, h], k[:, g], v[:, g], ss, scale, row_lo=lo)
        if do is not None:
            oracle.attention_bwd_head(q[:, h], k[:, g], v[:, g], do[:, h], ss, scale, row_lo=lo)
    dt = time.perf_counter() - t0
    per = (12 if do is not None else 4) * w.d
    return per * visible * heads, dt


def sample_rows_for(w) -> int:
    """Query rows of the oracle's bounded sample: the last rows of the
    sequence, about 512 x 32768 row-key pairs per head whatever n is."""
    return max(64, min(512, (512 * 32768) // w.n))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if not reports(rank):   # the oracle runs on rank 0 only; other ranks exit without work
        return 0
    x = synthetic.make_inputs(w)
    rows, heads = sample_rows_for(w), 2
    for _ in range(args.warmup):
        oracle_sample(w, x, rows, heads)
    flops, secs = 0, 0.0
    for _ in range(args.steps):
        f, s = oracle_sample(w, x, rows, heads)
        flops += f
        secs += s
    value = flops / secs / 1e12
    cores = len(os.sched_getaffinity(0))
    sample = f"oracle fwd+bwd of the last {rows} query rows of {heads} query heads per step"
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "P": w.P, "b": w.b, "n": w.n, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d},
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return 0


# ----------------------------------------------------------------------------- GPU arm
# Kernel launches of one step: s2h q, k, v (3); forward: segments, V's
# largest magnitude, its fp16 copy, attention (4); h2s O (1); s2h dO (1);
# backward: segments, largest magnitudes, fp16 copies, row statistics, dK/dV,
# dQ (6); h2s dQ, dK, dV (3).
LAUNCHES_FWD = 4
LAUNCHES_FWD_BWD = 3 + LAUNCHES_FWD + 1 + 1 + 6 + 3
# tcgen05 dense bf16 rate per SM and clock (M = 128, N = 256, K = 16 in 128 cycles)
TENSOR_FLOP_PER_CLK_SM = 8192
NUM_SMS = 148


class Layer:
    """Device buffers and the step of one workload: seq-sharded inputs in
    HBM, the re-layouts, the attention calls, fp32 outputs."""

    def __init__(self, w, x, dev, uly, pin=True):
        import torch
        self.w, self.uly, self.dev = w, uly, dev
        P, b, n, hq, hkv, d = w.P, w.b, w.n, w.h_q, w.h_kv, w.d
        m = n // P
        self.pairs = pairs_of(x["lengths"])
        self.fwd_flops = 4 * d * hq * self.pairs
        self.bwd_flops = 8 * d * hq * self.pairs if w.backward else 0
        bf, f32 = torch.bfloat16, torch.float32

        def host(bits):   # pinned when the end-to-end measurement copies from it every step
            t = torch.from_numpy(bits.reshape(P, b, m, bits.shape[2], d).view(np.int16)).view(bf)
            return t.pin_memory() if pin else t

        keys = ("q", "k", "v", "do") if w.backward else ("q", "k", "v")
        self.host = {k: host(x[k]) for k in keys}
        self.host_pos = torch.from_numpy(x["position_ids"])
        if pin:
            self.host_pos = self.host_pos.pin_memory()
        self.seq = {k: self.host[k].to(dev) for k in keys}
        self.pos = self.host_pos.to(dev)
        hkv_r = hkv // P if hkv >= P else 1   # kv heads per rank (one replicated head when H_kv < P)
        self.head = {"q": torch.empty((P, b, n, hq // P, d), dtype=bf, device=dev),
                     "k": torch.empty((P, b, n, hkv_r, d), dtype=bf, device=dev),
                     "v": torch.empty((P, b, n, hkv_r, d), dtype=bf, device=dev)}
        if w.backward:
            self.head["do"] = torch.empty((P, b, n, hq // P, d), dtype=bf, device=dev)
        self.o_head = torch.empty((P, b, n, hq // P, d), dtype=f32, device=dev)
        self.lse = torch.empty((P, b, hq // P, n), dtype=f32, device=dev)
        self.o_seq = torch.empty((P, b, m, hq, d), dtype=f32, device=dev)
        self.shape = uly.make_shape(b, n, hq, hkv, d, P)
        self.ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(self.shape), dev)
        nbytes = lambda t: t.numel() * t.element_size()   # noqa: E731
        # every re-layout reads its source once and writes its destination once
        self.relayout_bytes = sum(nbytes(self.seq[k]) + nbytes(self.head[k]) for k in keys)
        self.relayout_bytes += nbytes(self.o_head) + nbytes(self.o_seq)
        self.l2_note = f"inputs larger than L2 (q {nbytes(self.seq['q']) >> 20} MiB per step)"
        if w.backward:
            self.g_head = {"q": torch.empty_like(self.o_head),
                           "k": torch.empty((P, b, n, hkv_r, d), dtype=f32, device=dev),
                           "v": torch.empty((P, b, n, hkv_r, d), dtype=f32, device=dev)}
            self.g_seq = {"q": torch.empty((P, b, m, hq, d), dtype=f32, device=dev),
                          "k": torch.empty((P, b, m, hkv, d), dtype=f32, device=dev),
                          "v": torch.empty((P, b, m, hkv, d), dtype=f32, device=dev)}
            self.ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(self.shape, uly.ULY_F32), dev)
            self.relayout_bytes += sum(nbytes(self.g_head[k]) + nbytes(self.g_seq[k]) for k in self.g_seq)
        # forward-only workloads run s2h(q, k, v), the forward (rank by rank when
        # asked) and h2s(O)
        self.launches = LAUNCHES_FWD_BWD if w.backward else 3 + LAUNCHES_FWD * (P if w.rank_by_rank else 1) + 1

    def step(self, ev=None, kev=None):
        """One pass of the path.  ev: 6 events around its stages; kev: 5 events
        around the backward's kernels."""
        uly, h, s = self.uly, self.head, self.seq
        mark = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        mark(0)
        uly.ulysses_seq_to_head(s["q"], h["q"])
        for k in ("k", "v"):   # plain re-layout, or one copied kv head per rank when H_kv < P
            uly.ulysses_kv_seq_to_head(s[k], h[k])
        mark(1)
        if self.w.rank_by_rank:   # each virtual rank's head slice in turn
            for r in range(self.w.P):
                uly.ulysses_attn_fwd(h["q"], h["k"], h["v"], self.pos, self.o_head, self.lse, self.ws_f, rank=r)
        else:
            uly.ulysses_attn_fwd(h["q"], h["k"], h["v"], self.pos, self.o_head, self.lse, self.ws_f)
        mark(2)
        uly.ulysses_head_to_seq(self.o_head, self.o_seq)
        if not self.w.backward:
            mark(3), mark(4), mark(5)
            return
        uly.ulysses_seq_to_head(s["do"], h["do"])
        mark(3)
        g = self.g_head
        if kev is not None:   # the same call, with events around its kernels
            uly.ulysses_attn_bwd_timed(h["q"], h["k"], h["v"], self.o_head, self.lse, h["do"], self.pos,
                                       g["q"], g["k"], g["v"], self.ws_b, kev)
        else:
            uly.ulysses_attn_bwd(h["q"], h["k"], h["v"], self.o_head, self.lse, h["do"], self.pos,
                                 g["q"], g["k"], g["v"], self.ws_b)
        mark(4)
        uly.ulysses_head_to_seq(g["q"], self.g_seq["q"])
        for k in ("k", "v"):   # the copies' gradients are summed when H_kv < P
            uly.ulysses_kv_head_to_seq(g[k], self.g_seq[k])
        mark(5)

    def check_status(self, where: str):
        for ws in ((self.ws_f, self.ws_b) if self.w.backward else (self.ws_f,)):
            if self.uly.ulysses_workspace_status(ws) != 0:
                raise RuntimeError(f"a kernel reported a pipeline timeout {where}")


def time_layer(layer, steps: int, warmup: int, clocks, barrier=lambda: None):
    """Warm-up, then `steps` steps bracketed by a barrier and a synchronize.
    Returns the device time of the region, per-stage and per-kernel means and
    the clock record of the window."""
    import torch
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    layer.check_status("during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        layer.step(evs[i], kevs[i] if layer.w.backward else None)
    end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    layer.check_status("in the timed region")
    names = ("s2h_qkv", "attn_fwd", "h2s_o_s2h_do", "attn_bwd", "h2s_grads")
    st = {k: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, k in enumerate(names)}
    km = {}
    if layer.w.backward:
        km = {"bwd_prep (segments, magnitudes, fp16 copies, statistics)":
              statistics.mean(e[0].elapsed_time(e[2]) for e in kevs),
              "attn_bwd_dkdv_kernel": statistics.mean(e[2].elapsed_time(e[3]) for e in kevs),
              "attn_bwd_dq_kernel": statistics.mean(e[3].elapsed_time(e[4]) for e in kevs)}
    return {"ms_total": start.elapsed_time(end), "stage_ms": st, "kernel_ms": km,
            "clocks": clocks.summary(t0, t1), "seconds": t1 - t0}


def time_graph(layer, steps: int) -> float:
    """The same step captured once as a CUDA graph and replayed `steps` times
    (ms per step): what the step costs when its launches are submitted as
    one.  Nothing in the step synchronises or allocates, so it captures as
    it runs."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.step()
    graph.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    layer.check_status("under graph replay")
    del graph
    return start.elapsed_time(end) / steps


def clock_peak_tflops(sm_mhz):
    """The tensor pipe's dense bf16 rate at the sampled SM clock."""
    return None if not sm_mhz else TENSOR_FLOP_PER_CLK_SM * NUM_SMS * sm_mhz * 1e6 / 1e12


def layer_figures(layer, t, peaks):
    """Absolute figures and fractions of one timed workload."""
    st = t["stage_ms"]
    fwd_tf = layer.fwd_flops / (st["attn_fwd"] * 1e-3) / 1e12
    # the burst peak for short timed regions, the sustained one for long ones
    basis = "bf16_tflops_sustained" if t["seconds"] >= 2.0 else "bf16_tflops"
    peak = peaks[basis]
    cpk = clock_peak_tflops(t["clocks"].get("sm_mhz"))
    relayout_ms = st["s2h_qkv"] + st["h2s_o_s2h_do"] + st["h2s_grads"]
    out = {"pairs": layer.pairs, "ms_per_step": t["ms_total"] / max(1, t["steps"]), "steps": t["steps"],
           "stage_ms": st, "peak_basis": f"{basis} ({peaks['source']})",
           "attn_fwd_tflops": fwd_tf, "attn_fwd_frac": fwd_tf / peak,
           "attn_fwd_frac_of_clock_peak": fwd_tf / cpk if cpk else None,
           "relayout_gbs": layer.relayout_bytes / (relayout_ms * 1e-3) / 1e9,
           "relayout_bytes": layer.relayout_bytes, "clocks": t["clocks"]}
    out["relayout_frac"] = out["relayout_gbs"] / peaks["hbm_gbs"]
    if layer.w.backward:
        bwd_tf = layer.bwd_flops / (st["attn_bwd"] * 1e-3) / 1e12
        fb_tf = (layer.fwd_flops + layer.bwd_flops) / ((st["attn_fwd"] + st["attn_bwd"]) * 1e-3) / 1e12
        out.update({"attn_bwd_tflops": bwd_tf, "attn_bwd_frac": bwd_tf / peak,
                    "attn_fwd_bwd_tflops": fb_tf, "attn_fwd_bwd_frac": fb_tf / peak,
                    "attn_fwd_bwd_frac_of_clock_peak": fb_tf / cpk if cpk else None,
                    "bwd_kernel_ms": t["kernel_ms"]})
    return out


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    import ulysses_head_attention_b200 as uly

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)   # before the process group, so NCCL binds this rank's GPU
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)

    x = synthetic.make_inputs(w)
    layer = Layer(w, x, dev, uly)
    warm = max(args.warmup, 3)
    t = time_layer(layer, args.steps, warm, clocks, barrier)
    t["steps"] = args.steps
    ms_step = max_over_ranks(t["ms_total"], world, dev) / args.steps
    fig = layer_figures(layer, t, peaks)
    value = whole_job_tflops(world, layer.fwd_flops + layer.bwd_flops, ms_step)
    clk = t["clocks"]

    # ---- the dominant kernel's roofline: its algorithmic flops per launch (the
    # method's products it completes; recomputed S and dP are not counted) over
    # its event-timed duration
    if w.backward:
        d, hq, pairs = w.d, w.h_q, layer.pairs
        k_ms = {"attn_fwd_kernel": t["stage_ms"]["attn_fwd"],
                "attn_bwd_dkdv_kernel": t["kernel_ms"]["attn_bwd_dkdv_kernel"],
                "attn_bwd_dq_kernel": t["kernel_ms"]["attn_bwd_dq_kernel"]}
        # forward: S and PV; dK/dV kernel: dP, dV, dK; dQ kernel: dQ
        k_flops = {"attn_fwd_kernel": 4 * d * hq * pairs, "attn_bwd_dkdv_kernel": 6 * d * hq * pairs,
                   "attn_bwd_dq_kernel": 2 * d * hq * pairs}
        dom = max(k_ms, key=lambda kname: k_ms[kname])
        dom_tf = k_flops[dom] / (k_ms[dom] * 1e-3) / 1e12
        basis = "bf16_tflops_sustained" if t["seconds"] >= 2.0 else "bf16_tflops"
        cpk = clock_peak_tflops(clk.get("sm_mhz"))
        roofline = {"bound": "tensor", "kernel": dom, "achieved": dom_tf, "peak": peaks[basis], "unit": "TFLOP/s",
                    "frac": dom_tf / peaks[basis], "peak_kind": f"{basis} ({peaks['source']})",
                    "frac_of_clock_peak": dom_tf / cpk if cpk else None,
                    "flops_per_launch": k_flops[dom], "ms_per_launch": k_ms[dom],
                    "kernel_tflops": {kn: k_flops[kn] / (k_ms[kn] * 1e-3) / 1e12 for kn in k_ms},
                    "traffic": recorded_traffic(dom, w.name),
                    "kernel_traffic": {kn: recorded_traffic(kn, w.name) for kn in k_ms}}
    else:
        roofline = None

    # ---- end to end: pinned host inputs in, all outputs back to pinned host,
    # copies on their own streams so they overlap the attention kernels
    e2e = measure_e2e(layer, args.steps, barrier, world, dev) if w.backward else None

    # ---- the other workloads, each timed the same way in this run
    extras = {}
    if not args.no_extras:
        extras["configs"] = measure_configs(args, w, dev, uly, peaks, clocks)
        extras.update(measure_ring(layer, dev))
        extras["sp_loss_aggregate"] = measure_loss(layer, x, dev)
    clocks.stop()

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "P": w.P, "b": w.b, "n": w.n, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d,
                   "samples": sum(len(r) for r in x["lengths"]), "pairs": layer.pairs, "outputs": "fp32",
                   "l2": layer.l2_note, "parallelism": f"{world} independent replica(s), one per GPU"},
        "detail": {**fig, "fwd_flops": layer.fwd_flops, "bwd_flops": layer.bwd_flops,
                   "bwd_flops_with_recompute_convention": 10 * w.d * w.h_q * layer.pairs,
                   "peaks": peaks, **extras},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": layer.launches * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, secs = 0, 0.0
        rows, heads = sample_rows_for(w), 2
        for _ in range(4):
            f, s = oracle_sample(w, x, rows, heads)
            flops += f
            secs += s
        cpu_tf = flops / secs / 1e12
        out["cpu_baseline"] = {"value": cpu_tf, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
                               "kind": "oracle",
                               "sample": f"4 x oracle fwd+bwd of the last {rows} query rows of {heads} heads",
                               # the whole step's algorithmic work at the sample's rate (not run)
                               "extrapolated_step_s": (layer.fwd_flops + layer.bwd_flops) / (cpu_tf * 1e12)}
    if reports(rank):
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_e2e(layer, steps, barrier, world, dev):
    """The same metric through the C ABI's host-buffer call
    (ulysses_layer_step_host): every step copies its inputs in from pinned
    host memory and its outputs (O, dQ, dK, dV) back, inside the timed
    region.  The library runs the copies on two side streams, ordered by
    events against the kernels, so that dO arrives during the forward, O
    leaves during the backward, and one step's gradients leave while the
    next step's inputs arrive."""
    import torch
    uly, w = layer.uly, layer.w
    P, b, m, d = w.P, w.b, w.n // w.P, w.d
    f32 = torch.float32
    step = uly.LayerStepHost(b, w.n, w.h_q, w.h_kv, d, P, dev)
    h_out = [torch.empty((P, b, m, h, d), dtype=f32).pin_memory() for h in (w.h_q, w.h_q, w.h_kv, w.h_kv)]
    ins = [layer.host[k] for k in ("q", "k", "v", "do")]
    h2d = sum(t.numel() * t.element_size() for t in ins) + layer.host_pos.numel() * 8
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    main = torch.cuda.current_stream()

    def run(n_steps):
        for _ in range(n_steps):
            step.step(*ins, layer.host_pos, *h_out)
        main.wait_event(step.done_event())

    run(1)
    torch.cuda.synchronize()
    if step.status() != 0:
        raise RuntimeError("a kernel reported a pipeline timeout in the end-to-end warm-up")
    barrier()
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(main)
    run(steps)
    e2.record(main)
    torch.cuda.synchronize()
    barrier()
    if step.status() != 0:
        raise RuntimeError("a kernel reported a pipeline timeout in the end-to-end region")
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), world, dev) / steps
    del step
    torch.cuda.empty_cache()
    return {"value": whole_job_tflops(world, layer.fwd_flops + layer.bwd_flops, e2e_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "api": "ulysses_layer_step_host (C ABI, pinned host buffers in and out)",
            "copies": "H2D and D2H on two side streams ordered by events, overlapping attention"}


# the other workloads timed in the same run: (name, steps, warm-up)
OTHER_CONFIGS = (("tiny_p2_n256", 20, 3), ("llama8b_p4_n32k", 5, 3), ("packed_sft_p8_n64k", 5, 3),
                 ("long_p8_n512k", 2, 1))
# also timed as a replayed CUDA graph: the launch-bound workload, and one with
# the backward (whose step must capture as well)
GRAPH_CONFIGS = ("tiny_p2_n256", "llama8b_p4_n32k")


def measure_configs(args, w_main, dev, uly, peaks, clocks):
    import torch
    res = {}
    for name, steps, warm in OTHER_CONFIGS:
        if name == w_main.name:
            continue
        wk = synthetic.WORKLOADS[name]
        lay = Layer(wk, synthetic.make_inputs(wk), dev, uly, pin=False)
        t = time_layer(lay, steps, warm, clocks)
        t["steps"] = steps
        res[name] = layer_figures(lay, t, peaks)
        if args.graphs and name in GRAPH_CONFIGS:
            g_ms = time_graph(lay, steps)
            res[name]["graph"] = {"ms_per_step": g_ms, "launches_per_step": lay.launches,
                                  "note": "the step captured once as a CUDA graph, replayed"}
        del lay
        torch.cuda.empty_cache()
    return res


def measure_ring(layer, dev):
    """Ring attention as the ring driver computes it (ring.LibraryOps: block
    forward, LSE merge, block backward, accumulate) over R = 4 sequence
    blocks of every virtual Ulysses rank's head slice, the ranks one after
    another on this GPU: the ring's computation without its exchange (the
    composition of Ulysses over heads with a ring over the sequence)."""
    import torch
    from ulysses_head_attention_b200.ring import LibraryOps
    w, h = layer.w, layer.head
    R = 4
    P, b, n, hq_r, d = h["q"].shape
    hkv_r = h["k"].shape[3]
    if not w.backward or b != 1 or n % (R * 128):
        return {}   # blocks are row ranges of whole 128-row tiles, contiguous only for b = 1
    m, f32 = n // R, torch.float32
    ops = LibraryOps()

    def blocks(t):   # [p][r]: rows [r m, (r + 1) m) of rank p, block layout (1, b, m, heads, d)
        return [[t[p:p + 1, :, r * m:(r + 1) * m] for r in range(R)] for p in range(P)]

    Q, K, V, DO = blocks(h["q"]), blocks(h["k"]), blocks(h["v"]), blocks(h["do"])
    o_parts = torch.empty((R, 1, b, m, hq_r, d), dtype=f32, device=dev)
    l_parts = torch.empty((R, 1, b, hq_r, m), dtype=f32, device=dev)
    o_blk = torch.empty((P, R, 1, b, m, hq_r, d), dtype=f32, device=dev)   # merged O, LSE per (rank, block)
    l_blk = torch.empty((P, R, 1, b, hq_r, m), dtype=f32, device=dev)
    dq = torch.empty((1, b, m, hq_r, d), dtype=f32, device=dev)
    share_q = torch.empty_like(dq)
    share_k = torch.empty((1, b, m, hkv_r, d), dtype=f32, device=dev)
    share_v = torch.empty_like(share_k)
    acc_k = torch.empty((R, 1, b, m, hkv_r, d), dtype=f32, device=dev)   # key blocks' dK, dV accumulators
    acc_v = torch.empty_like(acc_k)
    calls = {"fwd_block": 0, "merge": 0, "bwd_block": 0, "accumulate": 0}

    def ring_fwd():
        for p in range(P):
            for r in range(R):
                for s in range(r + 1):   # key blocks at or before the query block
                    ops.fwd_block(Q[p][r], K[p][s], V[p][s], layer.pos, r * m, s * m, o_parts[s], l_parts[s])
                ops.merge(o_parts[:r + 1], l_parts[:r + 1], o_blk[p, r], l_blk[p, r], hkv_r)
                calls["fwd_block"] += r + 1
                calls["merge"] += 1

    def ring_bwd():
        for p in range(P):
            for r in range(R):
                for s in range(r, -1, -1):
                    if s == r:   # the diagonal block starts dQ and key block s's accumulators
                        ops.bwd_block(Q[p][r], K[p][s], V[p][s], o_blk[p, r], l_blk[p, r], DO[p][r], layer.pos,
                                      r * m, s * m, dq, acc_k[s], acc_v[s])
                    else:
                        ops.bwd_block(Q[p][r], K[p][s], V[p][s], o_blk[p, r], l_blk[p, r], DO[p][r], layer.pos,
                                      r * m, s * m, share_q, share_k, share_v)
                        ops.accumulate(dq, share_q)
                        ops.accumulate(acc_k[s], share_k)
                        ops.accumulate(acc_v[s], share_v)
                        calls["accumulate"] += 3
                    calls["bwd_block"] += 1

    ring_fwd()
    ring_bwd()
    torch.cuda.synchronize()
    calls = dict.fromkeys(calls, 0)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    ring_fwd()
    ev[1].record()
    ring_bwd()
    ev[2].record()
    torch.cuda.synchronize()
    ops.check()
    fwd_ms, bwd_ms = ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])
    del o_parts, l_parts, o_blk, l_blk, dq, share_q, share_k, share_v, acc_k, acc_v, ops
    torch.cuda.empty_cache()
    return {"ring_attention": {
        "blocks": R, "ulysses_ranks": P, "fwd_ms": fwd_ms, "fwd_tflops": layer.fwd_flops / (fwd_ms * 1e-3) / 1e12,
        "bwd_ms": bwd_ms, "bwd_tflops": layer.bwd_flops / (bwd_ms * 1e-3) / 1e12, "calls": calls,
        "note": "every virtual Ulysses rank's head slice cut into R sequence blocks; forward = block forwards of "
                "each query block against the key blocks at or before it + one LSE merge per query block; "
                "backward = block backwards from the merged O and LSE, dQ and the key blocks' dK, dV summed "
                "with the accumulate call; ranks run one after another, no exchange"}}


def measure_loss(layer, x, dev):
    """Weighted SP loss aggregation (the custom training loop's per-rank loss
    weighting), timed on its own: it needs a model's per-rank losses, which
    this path does not produce, so it is not part of the step."""
    import torch
    w, uly = layer.w, layer.uly
    P, b, m = w.P, w.b, w.n // w.P
    lab = synthetic.sft_shift_labels(w.wid, x["lengths"])
    lab_sh = torch.from_numpy(np.ascontiguousarray(lab.reshape(b, P, m).transpose(1, 0, 2))).to(dev)
    l_in = torch.from_numpy(synthetic.rank_losses(w.wid, P)).to(dev)
    l_out, l_good, l_dl = (torch.empty(1, device=dev), torch.empty(P, dtype=torch.int64, device=dev),
                           torch.empty(P, device=dev))
    for _ in range(5):
        uly.ulysses_sp_loss_aggregate(l_in, lab_sh, l_out, l_good, l_dl)
    torch.cuda.synchronize()
    s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 50
    s3.record()
    for _ in range(reps):
        uly.ulysses_sp_loss_aggregate(l_in, lab_sh, l_out, l_good, l_dl)
    e3.record()
    torch.cuda.synchronize()
    loss_us = s3.elapsed_time(e3) * 1e3 / reps
    loss_bytes = lab_sh.numel() * 8 + 3 * P * 8 + 4
    return {"us_per_call": loss_us, "bytes_per_call": loss_bytes,
            "gbs": loss_bytes / (loss_us * 1e-6) / 1e9, "launches_per_call": 2,
            "labels": "packed SFT: per sample a U[0.1, 0.6) prompt fraction and the last position are -100"}


# ----------------------------------------------------------------------------- profiling case
def run_profile_case():
    """Small launches of the step's kernels for ncu captures: one seq_to_head
    re-layout of a Llama-8B-shaped q (P = 4, n = 32768, 32 heads, d = 128:
    256 MiB in, 256 MiB out, each above L2's size), then one forward and one
    backward of virtual rank 0 at P = 4, b = 1, n = 16384, H_q = 32,
    H_kv = 8, d = 128 (its 8 query heads), one causal sample,
    standard-normal bf16 inputs drawn on the device (seed 0).  The device
    holds about 2 GB.  Times nothing."""
    import torch
    import ulysses_head_attention_b200 as uly
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev).manual_seed(0)
    P, b, hq, hkv, d = 4, 1, 32, 8, 128
    x_seq = torch.randn((P, b, 32768 // P, hq, d), device=dev, generator=g).to(torch.bfloat16)
    x_head = torch.empty((P, b, 32768, hq // P, d), dtype=torch.bfloat16, device=dev)
    uly.ulysses_seq_to_head(x_seq, x_head)
    del x_seq, x_head
    n = 16384

    def mk(h):
        return torch.randn((P, b, n, h // P, d), device=dev, generator=g).to(torch.bfloat16)

    q, k, v, do = mk(hq), mk(hkv), mk(hkv), mk(hq)
    pos = torch.arange(n, device=dev).view(1, n)
    o = torch.empty((P, b, n, hq // P, d), dtype=torch.float32, device=dev)
    lse = torch.empty((P, b, hq // P, n), dtype=torch.float32, device=dev)
    shape = uly.make_shape(b, n, hq, hkv, d, P)
    wf = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    wb = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev)
    dq = torch.empty_like(o)
    dk = torch.empty((P, b, n, hkv // P, d), device=dev)
    dv = torch.empty((P, b, n, hkv // P, d), device=dev)
    uly.ulysses_attn_fwd(q, k, v, pos, o, lse, wf, rank=0)
    uly.ulysses_attn_bwd(q, k, v, o, lse, do, pos, dq, dk, dv, wb, rank=0)
    torch.cuda.synchronize()
    if uly.ulysses_workspace_status(wf) != 0 or uly.ulysses_workspace_status(wb) != 0:
        raise RuntimeError("a kernel reported a pipeline timeout")
    print("profile case done")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graphs", dest="graphs", action="store_false",
                    help="skip timing the launch-bound workloads as replayed CUDA graphs")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the separately timed ring-attention and loss-aggregation measurements")
    ap.add_argument("--profile-case", action="store_true",
                    help="run one small forward + backward for an ncu capture, then exit (no timing, no JSON)")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case()
    w = synthetic.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
