#!/usr/bin/env python
"""Benchmark of the HGA per-segment attention step on B200.

Workload: one Qwen3-8B-shaped attention layer in bf16 -- 32 query / 8 KV
heads, d = 128, history 14,336 tokens (112 blocks of 128), active segment
2,048 tokens (16 query blocks), top-K = 16 -- with seeded synthetic inputs.
One step = every kernel of the hot path over that layer: block summaries,
top-K selection, attention forward, backward preprocess, dK/dV, dQ.

Metric: attention fwd+bwd tokens/s per layer (segment tokens / step time),
summed over the GPUs (each GPU runs its own independent layer: replicas).
Timing: CUDA events on the launching stream around every kernel; L2 is
flushed (256 MiB write) between steps, outside the timed events.

Extra keys: roofline of the dominant kernel, per-kernel breakdown, e2e
(the same step through the public API with host buffers: pinned H2D of the
segment's inputs, history blocks fetched from a pinned host tier by
hga_fetch_blocks, D2H of every result: O, LSE, dQ, dK, dV), the 131K-token
prefill's summaries, selection and forward timed the same way (where the
HBM-bound kernels move enough bytes for their roofline fraction to mean
something), cpu_baseline (the fp64 oracle on a bounded sample, on this
host's cores), and SM clocks sampled during the timed region.

--impl reference times the fp64 CPU oracle (the reference arm) on the same
workload: each step is a bounded sample (selection for every head, forward
and backward for one KV head), scaled to the metric's unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "HGA attn fwd+bwd tokens/s per layer on 1 B200; % of bf16 tensor peak / HBM BW"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS = ("summaries", "select", "fwd", "bwd_pre", "bwd_dkdv", "bwd_dq")
KERNEL_SOURCES = {"fwd": "hga_attn_fwd_tc.cu", "bwd_dq": "hga_attn_bwd_tc.cu", "bwd_dkdv": "hga_attn_bwd_tc.cu",
                  "summaries": "hga_select.cu", "select": "hga_select.cu", "bwd_pre": "hga_select.cu"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_config(w: synth.Workload, l2_note: str):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.d, "block": w.blk,
            "q_block": w.qb, "segment_tokens": w.S, "history_blocks": w.nblk, "topk": w.topk, "l2": l2_note}


# ---------------------------------------------------------------- ranks

def max_over_ranks(x: float, world: int, device) -> float:
    """Largest x over the ranks of the default process group (every rank
    calls it with its own x; identity for a single process)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own replica of the step."""
    return world * tokens_per_step / (ms_per_step / 1e3)


# ---------------------------------------------------------------- work model

def work_model(w: synth.Workload, keff_sum_per_head: float):
    """Algorithmic work of one step.  Attention counts only the (query, key)
    pairs the method computes: per query head, history pairs = sum over query
    rows of K_eff*block, segment pairs = S(S+1)/2.  Forward 4d FLOP per pair;
    backward 4d per history pair (dP, dQ) and 8d per segment pair (dP, dQ, dK,
    dV); of those, the dQ kernel does dP and dQ for every pair, the dK/dV
    kernel dK and dV for segment pairs."""
    d = w.d
    hist_pairs = keff_sum_per_head * w.qb * w.blk  # per head: sum_i K_eff(i) * q_block rows * block keys
    seg_pairs = w.S * (w.S + 1) / 2
    H = w.Hq * w.B
    flops = {
        "fwd": 4 * d * (hist_pairs + seg_pairs) * H,
        "bwd_dq": 4 * d * (hist_pairs + seg_pairs) * H,
        "bwd_dkdv": 4 * d * seg_pairs * H,
    }
    es = 2 if w.dtype == "bf16" else 4
    bytes_ = {
        "summaries": w.B * w.nblk * w.blk * w.Hkv * d * es + w.B * w.Hkv * w.nblk * d * 4,
        "select": w.B * w.S * w.Hq * d * es + w.B * w.Hkv * w.nblk * d * 4 + w.B * w.Hkv * w.nqb * w.topk * 4,
        "bwd_pre": 2 * w.B * w.S * w.Hq * d * es + w.B * w.Hq * w.S * 4,
    }
    return flops, bytes_


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML unavailable: report no clocks
            self._nvml = None
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nvml:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- helpers

def to_dev(t: synth.Tensor, device):
    if t.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.store)).to(device)


def to_pinned(t: synth.Tensor):
    if t.dtype == "bf16":
        x = torch.from_numpy(np.ascontiguousarray(t.store).view(np.int16)).view(torch.bfloat16)
    else:
        x = torch.from_numpy(np.ascontiguousarray(t.store))
    return x.pin_memory()


def source_sha(fname: str) -> str:
    """Hash of a kernel's source file and the headers every kernel includes."""
    h = hashlib.sha256()
    for name in (fname, "hga_ptx.cuh", "hga_kernels.h"):
        with open(os.path.join(ROOT, "segmented_fine_tuning_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, or None when
    the kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- device leg

# Device workloads of `--workload`: the headline layer step, and the two
# parity workloads (dense-equivalence, 131K prefill forward) timed the same way.
DEVICE_WORKLOADS = {"layer": synth.QWEN3_8B_LAYER, "dense": synth.DENSE_EQUIV, "prefill": synth.PREFILL_131K,
                    "layer64": synth.QWEN3_8B_LAYER64, "layer32": synth.QWEN3_8B_LAYER32}


def run_device(args, rank, world, device, w=None, steps=None):
    import segmented_fine_tuning_b200 as hga
    from segmented_fine_tuning_b200.step import AttentionStep

    w = DEVICE_WORKLOADS[args.workload] if w is None else w
    steps = args.steps if steps is None else steps
    D = hga.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk, w.dtype, w.qblk)
    x = synth.draw(w)
    dev = {n: to_dev(getattr(x, n), device) for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    st = AttentionStep(D, device)
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def step(evs=None, s=stream, combined=False):
        """combined: the backward through hga_attn_bwd (preprocess, then dQ and
        dK/dV on two streams); otherwise one entry point per kernel, so that
        events can sit between them."""
        def mark(k):
            if evs is not None:
                evs[k].record(s)
        mark(0)
        hga.hga_block_summaries(D, dev["k_hist"], 0, D.n_hist_blocks, st.summ, s)
        mark(1)
        hga.hga_select_topk(D, dev["q"], st.summ, st.idx, None, s)
        mark(2)
        hga.hga_attn_fwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], D.n_hist_blocks,
                         st.idx, st.o, st.lse, s)
        mark(3)
        if combined:
            if not w.fwd_only:
                hga.hga_attn_bwd(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"],
                                 D.n_hist_blocks, st.idx, st.o, st.lse, dev["d_o"], st.dq, st.dk, st.dv, st.ws, s)
            return
        if not w.fwd_only:
            hga.hga_attn_bwd_preprocess(D, st.o, dev["d_o"], st.ws, s)
        mark(4)
        if not w.fwd_only:
            hga.hga_attn_bwd_dkdv(D, dev["q"], dev["k_seg"], dev["v_seg"], st.lse, dev["d_o"], st.ws, st.dk, st.dv,
                                  s)
        mark(5)
        if not w.fwd_only:
            hga.hga_attn_bwd_dq(D, dev["q"], dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"],
                                D.n_hist_blocks, st.idx, st.lse, dev["d_o"], st.ws, st.dq, s)
        mark(6)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    hga.hga_device_status(stream)
    keff_sum = float((st.idx >= 0).sum().item()) / (w.B * w.Hkv)  # sum over query blocks, per KV head

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        for k in range(steps):
            flush.zero_()
            step(evs[k])
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    hga.hga_device_status(stream)

    per_kernel = {name: [] for name in KERNELS}
    step_ms = []
    for e in evs:
        step_ms.append(e[0].elapsed_time(e[6]))
        for j, name in enumerate(KERNELS):
            per_kernel[name].append(e[j].elapsed_time(e[j + 1]))
    eager_ms = max_over_ranks(float(sum(step_ms)), world, device) / steps

    # The same step captured once as a CUDA graph and replayed: the kernels
    # and their arguments are identical, but no host work (argument checks,
    # tensor-map encoding, launch calls) sits between them on the timeline.
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    cap.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap, capture_error_mode="relaxed"):
        step(s=cap, combined=True)
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        flush.zero_()
        graph.replay()
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as gclk:
        for e0, e1 in gev:
            flush.zero_()
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    hga.hga_device_status(stream)
    del graph
    total_ms = max_over_ranks(float(sum(e0.elapsed_time(e1) for e0, e1 in gev)), world, device)
    ms_per_step = total_ms / steps
    value = job_throughput(world, w.S, ms_per_step)

    peaks, peak_src = load_peaks()
    flops, bytes_ = work_model(w, keff_sum)
    kern = {}
    for name in KERNELS:
        ms = float(np.mean(per_kernel[name]))
        entry = {"ms": round(ms, 4)}
        if name in flops:
            tf = flops[name] / (ms / 1e3) / 1e12
            entry.update({"tflops": round(tf, 1), "frac_bf16_peak": round(tf / peaks["bf16_tflops"], 3)})
        if name in bytes_:
            gbs = bytes_[name] / (ms / 1e3) / 1e9
            entry.update({"gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)})
        kern[name] = entry
    if w.fwd_only:
        for name in ("bwd_pre", "bwd_dkdv", "bwd_dq"):
            kern.pop(name)
    dom = max([n for n in ("fwd", "bwd_dq", "bwd_dkdv") if n in kern], key=lambda n: kern[n]["ms"])
    dom_ms = kern[dom]["ms"]
    achieved = flops[dom] / (dom_ms / 1e3) / 1e12
    traffic = committed_traffic(dom)
    roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": traffic,
                "peak_source": f"{peak_src} dense bf16 (burst)",
                "algorithmic_flop_per_launch": flops[dom]}
    attn = [n for n in ("fwd", "bwd_dq", "bwd_dkdv") if n in kern]
    fwd_bwd_flops = sum(flops[n] for n in attn)
    attn_ms = sum(kern[n]["ms"] for n in attn)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1); block-structured keys)",
        "config": workload_config(w, "flushed between steps (256 MiB write, outside the timed events)"),
        "roofline": roofline,
        ("attention_fwd" if w.fwd_only else "attention_fwd_bwd"): {"tflops": round(fwd_bwd_flops / (attn_ms / 1e3) / 1e12, 1),
                              "frac_bf16_peak": round(fwd_bwd_flops / (attn_ms / 1e3) / 1e12 /
                                                      peaks["bf16_tflops"], 3),
                              "algorithmic_gflop": round(fwd_bwd_flops / 1e9, 2)},
        "kernels": kern,
        "launch": "the step (summaries, selection, forward, hga_attn_bwd: preprocess, then dQ and dK/dV on two "
                  "streams) replayed as one CUDA graph; per-kernel times from the same kernels launched eagerly one "
                  "entry point at a time with an event between them (small kernels' spans include their launch "
                  "latency)",
        "eager": {"ms_per_step": round(eager_ms, 4), "tokens_per_s": round(job_throughput(world, w.S, eager_ms), 1),
                  "clocks": clk.summary()},
        "gpu_launches": (3 if w.fwd_only else 6) * steps,
        "clocks": gclk.summary(),
    }
    return out, (w, x, D, dev, st)


def run_e2e(args, ctx, device):
    """The same step through the public API with host buffers: every step
    copies the segment's Q, K, V, dO from pinned host memory, fetches its
    selected history blocks from a pinned host tier (hga_fetch_blocks), runs
    selection, forward and backward, and copies every result (O, LSE, dQ,
    dK, dV) back to pinned host memory.  Steps are pipelined two deep, as a
    training loop with a prefetching data loader runs them: step k+1's
    inputs travel host -> device, its selection runs and its history blocks
    are fetched, and step k-1's results travel device -> host, while step k
    computes (separate copy and selection streams, double-buffered device
    sets).
    The timed region spans the first input copy to the last result copy."""
    import segmented_fine_tuning_b200 as hga
    w, x, D, dev, st0 = ctx
    stream = torch.cuda.current_stream(device)
    h2d, d2h, fetch_stream, sel_stream = (torch.cuda.Stream(device) for _ in range(4))
    host = {n: to_pinned(getattr(x, n)) for n in ("q", "k_seg", "v_seg", "d_o")}
    tier_k, tier_v = to_pinned(x.k_hist), to_pinned(x.v_hist)
    # the history's summaries are resident on the device (computed once, when
    # the blocks entered the history)
    hga.hga_block_summaries(D, dev["k_hist"], 0, D.n_hist_blocks, st0.summ, stream)
    from segmented_fine_tuning_b200.step import AttentionStep
    sets = []
    for _ in range(2):
        st = AttentionStep(D, device)
        r = {"st": st, "seg": {n: torch.empty_like(dev[n]) for n in host},
             "pool_k": torch.empty_like(dev["k_hist"]), "pool_v": torch.empty_like(dev["v_hist"]),
             "idx_pool": torch.empty_like(st.idx),
             "scratch": torch.empty(tuple(st.idx.shape), dtype=torch.int32).pin_memory(),
             "results": {"o": st.o, "lse": st.lse, "dq": st.dq, "dk": st.dk, "dv": st.dv}}
        r["out"] = {n: torch.empty(tuple(t.shape), dtype=t.dtype).pin_memory() for n, t in r["results"].items()}
        r["ev"] = {e: torch.cuda.Event() for e in ("q", "h2d", "comp", "d2h", "fetch")}
        r["ev"]["fetch"].record(fetch_stream)  # materialise the handle the C call records into
        sets.append(r)
    blk_bytes = w.blk * w.Hkv * w.d * 2 * 2  # K and V of one block
    fetched = []

    def inputs_in(k):
        r = sets[k % 2]
        h2d.wait_event(r["ev"]["comp"])  # step k-2 has consumed this set's inputs
        with torch.cuda.stream(h2d):
            # Q first: the selection and the history fetch it drives need only Q, so they start while
            # K, V and dO are still on the link
            r["seg"]["q"].copy_(host["q"], non_blocking=True)
            r["ev"]["q"].record(h2d)
            for n in ("k_seg", "v_seg", "d_o"):
                r["seg"][n].copy_(host[n], non_blocking=True)
        r["ev"]["h2d"].record(h2d)

    def select_and_fetch(k):
        # selection needs only this step's queries and the resident summaries, so it (and the history
        # fetch it drives) runs as soon as Q lands, while the previous step computes
        r = sets[k % 2]
        st, seg = r["st"], r["seg"]
        sel_stream.wait_event(r["ev"]["q"])
        sel_stream.wait_event(r["ev"]["comp"])  # step k-2 has finished with this set's idx and pool
        hga.hga_select_topk(D, seg["q"], st0.summ, st.idx, None, sel_stream)
        nu = hga.hga_fetch_blocks(D, tier_k, tier_v, D.n_hist_blocks, st.idx, r["scratch"], r["pool_k"],
                                  r["pool_v"], D.n_hist_blocks, r["idx_pool"], sel_stream, fetch_stream,
                                  r["ev"]["fetch"])
        fetched.append(nu)

    def compute_and_out(k):
        r = sets[k % 2]
        st, seg = r["st"], r["seg"]
        stream.wait_event(r["ev"]["h2d"])
        stream.wait_event(r["ev"]["d2h"])  # step k-2's results have left this set's outputs
        stream.wait_event(r["ev"]["fetch"])
        hga.hga_attn_fwd(D, seg["q"], seg["k_seg"], seg["v_seg"], r["pool_k"], r["pool_v"], D.n_hist_blocks,
                         r["idx_pool"], st.o, st.lse, stream)
        hga.hga_attn_bwd(D, seg["q"], seg["k_seg"], seg["v_seg"], r["pool_k"], r["pool_v"], D.n_hist_blocks,
                         r["idx_pool"], st.o, st.lse, seg["d_o"], st.dq, st.dk, st.dv, st.ws, stream)
        r["ev"]["comp"].record(stream)
        d2h.wait_event(r["ev"]["comp"])
        with torch.cuda.stream(d2h):
            for n, t in r["results"].items():
                r["out"][n].copy_(t, non_blocking=True)
        r["ev"]["d2h"].record(d2h)

    def run(n):
        inputs_in(0)
        select_and_fetch(0)
        for k in range(n):
            if k + 1 < n:
                inputs_in(k + 1)
            compute_and_out(k)
            if k + 1 < n:
                select_and_fetch(k + 1)  # the host waits here for step k+1's indices, step k already queued
        for s_ in (h2d, d2h, fetch_stream, sel_stream):
            stream.wait_stream(s_)

    run(max(2, args.warmup))
    torch.cuda.synchronize(device)
    fetched.clear()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = args.steps
    e0.record(stream)
    for s_ in (h2d, d2h, fetch_stream, sel_stream):
        s_.wait_event(e0)
    run(n)
    e1.record(stream)
    torch.cuda.synchronize(device)
    hga.hga_device_status(stream)
    ms = e0.elapsed_time(e1) / n
    r0 = sets[0]
    h2d_bytes = sum(t.numel() * t.element_size() for t in host.values()) + np.mean(fetched) * blk_bytes \
        + r0["idx_pool"].numel() * 4
    d2h_bytes = r0["scratch"].numel() * 4 + sum(t.numel() * t.element_size() for t in r0["out"].values())
    return {"value": round(w.S / (ms / 1e3), 1), "unit": UNIT, "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
            "fetched_blocks_per_step": float(np.mean(fetched)),
            "path": "pinned host tier + hga_fetch_blocks; O, LSE, dQ, dK, dV copied back to pinned host memory; "
                    "steps pipelined two deep (inputs, selection and history fetch of k+1 and results of k-1 in "
                    "flight during k)"}


# ---------------------------------------------------------------- segmented pass

def h2d_probe(device, nbytes=1 << 30, reps=5):
    """Pinned host -> device copy bandwidth (GB/s), the roofline of the fetch."""
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream(device)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        dst.copy_(src, non_blocking=True)
        e1.record(st)
        torch.cuda.synchronize(device)
        best = max(best, nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    return best


SEGMENTED_MODES = {
    # history served from the pinned host tier: finished segments are not
    # inserted into the device pool, so every step copies its new blocks over
    # the host link; selection and fetch of layer l+1 overlap layer l
    "host_tier": dict(keep_new_blocks=False, prefetch=True),
    # the same without the one-layer lookahead (the host waits for each
    # layer's indices before its copies start)
    "host_tier_no_prefetch": dict(keep_new_blocks=False, prefetch=False),
    # finished segments also enter each layer's device block cache: no host
    # transfer in the pass (the compute-only reference)
    "resident": dict(keep_new_blocks=True, prefetch=True),
}


def run_segmented(args, device):
    """The full segmented pass: 36 Qwen3-8B-shaped layers over a 16,384-token
    sequence as 8 segments of 2,048 (history in a pinned host tier, selected
    blocks fetched per (layer, segment) unless already resident in the
    layer's device block cache, summaries appended on the device).
    Inputs: the 8 segments of layer 0 drawn with the workload's recipe and
    reused for every layer (the kernels' speed does not depend on values;
    selection, and so fetch volume, is representative).  One step = one pass.
    Every mode of --segmented-modes is timed; the first is the line's value."""
    import segmented_fine_tuning_b200 as hga
    from segmented_fine_tuning_b200.segmented import SegmentedPass
    w = synth.QWEN3_8B_LAYER
    L, NS = synth.SEGMENTED_LAYERS, synth.SEGMENTED_SEGMENTS
    seg = hga.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, 0, w.topk, "bf16")
    xs = [synth.draw_segment(w, 0, s) for s in range(NS)]
    dev = [tuple(to_dev(t, device) for t in (x.q, x.k_seg, x.v_seg, x.d_o)) for x in xs]
    stream = torch.cuda.current_stream(device)
    blk_bytes = w.blk * w.Hkv * w.d * 2 * 2
    probe = h2d_probe(device)
    modes = [m for m in args.segmented_modes.split(",") if m]
    results = {}
    for mode in modes:
        sp = SegmentedPass(seg, L, NS, device, pool_slots=args.pool_slots, **SEGMENTED_MODES[mode])

        def one_pass():
            sp.new_sequence()  # each pass is a new sequence: nothing resident carries over
            for s in range(NS):
                sp.run_segment(s, [dev[s]] * L)

        for _ in range(args.warmup):
            one_pass()
        torch.cuda.synchronize(device)
        hga.hga_device_status(stream)
        sp.fetched_blocks.clear()
        sp.selected_blocks.clear()
        sp.device_remaps = 0
        times = []
        with ClockSampler(device.index if device.index is not None else 0) as clk:
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                one_pass()
                e1.record(stream)
                torch.cuda.synchronize(device)
                times.append(e0.elapsed_time(e1))
        hga.hga_device_status(stream)
        ms = float(np.mean(times))
        fetched = float(np.mean(sp.fetched_blocks))
        h2d_bytes = float(np.sum(sp.fetched_blocks)) * blk_bytes / args.steps
        remaps = sp.device_remaps // args.steps
        results[mode] = {"ms_per_pass": round(ms, 3), "tokens_per_s": round(NS * w.S * L / (ms / 1e3), 1),
                         "blocks_copied_per_layer_step": round(fetched, 1), "h2d_bytes_per_pass": int(h2d_bytes),
                         "fetch_time_at_probe_ms": round(h2d_bytes / (probe * 1e9) * 1e3, 2),
                         "steps_remapped_on_device_per_pass": remaps,
                         "device_block_cache_slots_per_layer": sp.pool_slots,
                         "gpu_launches_per_pass": int(L * NS * 6 + remaps), "clocks": clk.summary(),
                         **SEGMENTED_MODES[mode]}
        del sp
        torch.cuda.empty_cache()
    head = results[modes[0]]
    out = {"metric": "HGA full segmented pass tokens/s per layer (fwd+bwd, history fetched from a pinned host tier)",
           "value": head["tokens_per_s"], "unit": UNIT, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": head["ms_per_pass"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic (layer 0's 8 segments reused for all layers)",
           "config": {"workload": "segmented pass: 36 Qwen3-8B-shaped layers x 8 segments of 2,048 tokens, "
                                  "history +16 blocks of 128 per segment, K16, pinned host tier",
                      "layers": L, "segments": NS, "segment_tokens": w.S, "topk": w.topk, "mode": modes[0]},
           "h2d_probe_gbs": round(probe, 1), "modes": results,
           "gpu_launches": head["gpu_launches_per_pass"] * args.steps, "clocks": head["clocks"]}
    if "resident" in results and modes[0] != "resident":
        compute = results["resident"]["ms_per_pass"]
        bound = max(compute, head["fetch_time_at_probe_ms"])
        out["overlap"] = {"compute_only_ms": compute, "h2d_at_probe_ms": head["fetch_time_at_probe_ms"],
                          "pass_over_bound": round(head["ms_per_pass"] / bound, 3)}
    return out


def run_decode(args, device):
    """Decode at 131K context: 992 history blocks with resident summaries, a
    4,096-token segment buffer, one new token at its last position, K = 32.
    One step = decode selection + decode attention (split over key chunks,
    then the merge), L2 flushed between steps.  Each kernel's bytes are its
    algorithmic HBM traffic: the summaries for the selection; the selected
    history blocks, the segment prefix and the new queries for attention."""
    import segmented_fine_tuning_b200 as hga
    w = synth.DECODE_131K
    nq, t0 = 1, w.S - 1
    D = hga.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk, w.dtype, w.qblk)
    x = synth.draw_decode(w, nq, t0)
    dev = {n: to_dev(getattr(x, n), device) for n in ("k_seg", "v_seg", "k_hist", "v_hist")}
    qn = to_dev(x.extra["q_new"], device)
    summ = torch.empty((w.B, w.nblk, w.Hkv, w.d), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    hga.hga_block_summaries(D, dev["k_hist"], 0, w.nblk, summ, stream)
    idx = torch.empty((w.B, w.Hkv, w.topk), dtype=torch.int32, device=device)
    o = torch.empty_like(qn)
    lse = torch.empty((w.B, w.Hq, nq), dtype=torch.float32, device=device)
    ws = torch.empty((hga.hga_decode_workspace_size(D, nq),), dtype=torch.uint8, device=device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        hga.hga_decode_select(D, qn, summ, idx, None, ws, stream)
        if evs:
            evs[1].record(stream)
        hga.hga_decode_attn(D, t0, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk, idx, o,
                            lse, ws, stream)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    hga.hga_device_status(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        for k in range(args.steps):
            flush.zero_()
            step(evs[k])
        torch.cuda.synchronize(device)
    hga.hga_device_status(stream)
    t_sel = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_att = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms = t_sel + t_att
    # whole step as one CUDA graph (three launches replayed without host launch cost)
    graph = {}
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                hga.hga_decode_select(D, qn, summ, idx, None, ws, side)
                hga.hga_decode_attn(D, t0, qn, dev["k_seg"], dev["v_seg"], dev["k_hist"], dev["v_hist"], w.nblk,
                                    idx, o, lse, ws, side)
        stream.wait_stream(side)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize(device)
        gt = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize(device)
            gt.append(e0.elapsed_time(e1))
        hga.hga_device_status(stream)
        ms_graph = float(np.mean(gt))
        graph = {"ms_per_step": round(ms_graph, 4), "tokens_per_s": round(nq / (ms_graph / 1e3), 1)}
    except Exception as e:  # report, do not hide: the eager numbers above stand
        graph = {"error": str(e)[:300]}
    keff = min(w.topk, w.nblk)
    kv_bytes = (keff * w.blk + t0 + nq) * w.Hkv * w.d * 2 * 2 + qn.numel() * 2
    sel_bytes = w.nblk * w.Hkv * w.d * 4 + qn.numel() * 2
    peaks, peak_src = load_peaks()
    att_gbs = kv_bytes / (t_att / 1e3) / 1e9
    return {"metric": "HGA decode tokens/s per layer (131K context, one new token per step)",
            "value": round(nq / (ms / 1e3), 1), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1); block-structured keys)",
            "config": {"workload": w.name, "history_blocks": w.nblk, "segment_buffer": w.S, "t0": t0, "n_q": nq,
                       "topk": w.topk, "l2": "flushed between steps (256 MiB write, outside the timed events)"},
            "kernels": {"decode_select": {"ms": round(t_sel, 4), "bytes": sel_bytes,
                                          "gbs": round(sel_bytes / (t_sel / 1e3) / 1e9, 1)},
                        "decode_attn": {"ms": round(t_att, 4), "bytes": kv_bytes, "gbs": round(att_gbs, 1),
                                        "frac_hbm": round(att_gbs / peaks["hbm_gbs"], 3)}},
            "roofline": {"kernel": "decode_attn (partial + merge)", "bound": "hbm", "achieved": round(att_gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(att_gbs / peaks["hbm_gbs"], 4),
                         "traffic": None, "peak_source": f"{peak_src} HBM copy bandwidth"},
            "cuda_graph": graph,
            "gpu_launches": 4 * args.steps, "clocks": clk.summary()}


def run_tier(args, device):
    """The history-tier paths on the Qwen3-8B-shaped layer: fetching the
    selected blocks (every one of the 112 history blocks is selected by some
    query block) from a pinned host tier by the copy engines
    (hga_fetch_blocks) and by the SMs over mapped memory
    (hga_gather_blocks_mapped), the device idx remap, and a finished segment's
    append in one pass (hga_append_segment) against the three separate calls
    it replaces.  Each timed on the stream with CUDA events (mean of --steps,
    L2 flushed between steps); bytes are the algorithmic bytes moved."""
    import segmented_fine_tuning_b200 as hga
    w = synth.QWEN3_8B_LAYER
    D = hga.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk, w.dtype, w.qblk)
    x = synth.draw(w)
    stream = torch.cuda.current_stream(device)
    copy_stream = torch.cuda.Stream(device)
    q, ks, vs, kh = (to_dev(t, device) for t in (x.q, x.k_seg, x.v_seg, x.k_hist))
    tier_k, tier_v = to_pinned(x.k_hist), to_pinned(x.v_hist)
    summ = torch.empty((1, w.nblk, w.Hkv, w.d), dtype=torch.float32, device=device)
    idx = torch.empty((1, w.Hkv, w.nqb, w.topk), dtype=torch.int32, device=device)
    hga.hga_block_summaries(D, kh, 0, w.nblk, summ, stream)
    hga.hga_select_topk(D, q, summ, idx, None, stream)
    torch.cuda.synchronize(device)
    n_sel = len(set(idx.cpu().numpy().ravel().tolist()) - {-1})
    pool_k = torch.empty((1, w.nblk * w.blk, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    pool_v = torch.empty_like(pool_k)
    idx_pool = torch.empty_like(idx)
    scratch = torch.empty(tuple(idx.shape), dtype=torch.int32).pin_memory()
    done = torch.cuda.Event()
    done.record(copy_stream)
    slot_of = torch.arange(w.nblk, dtype=torch.int32, device=device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    blk_bytes = w.blk * w.Hkv * w.d * 2
    # append: a segment entering a history of capacity nblk + nqb blocks
    cap = w.nblk + w.nqb
    Da = hga.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, cap, w.topk, "bf16")
    summ_a = torch.zeros((1, cap, w.Hkv, w.d), dtype=torch.float32, device=device)
    cache = hga.BlockCache(cap, w.nblk + w.nqb)
    pk = torch.empty((1, cache.pool_slots * w.blk, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    pv = torch.empty_like(pk)
    tk = torch.empty((1, cap * w.blk, w.Hkv, w.d), dtype=torch.bfloat16).pin_memory()
    tv = torch.empty_like(tk).pin_memory()

    def fetch():
        hga.hga_fetch_blocks(D, tier_k, tier_v, w.nblk, idx, scratch, pool_k, pool_v, w.nblk, idx_pool, stream,
                             copy_stream, done)
        stream.wait_event(done)

    def gather():
        hga.hga_gather_blocks_mapped(D, tier_k, tier_v, w.nblk, idx, pool_k, pool_v, w.nblk, idx_pool, stream)

    def remap():
        hga.hga_remap_idx(D, idx, slot_of, idx_pool, stream)

    def append_fused():
        cache.reset()
        hga.hga_append_segment(Da, ks, vs, w.nblk, summ_a, pk, pv, cache, None, None, 0, stream)

    def append_separate():
        cache.reset()
        hga.hga_segment_summaries(Da, ks, w.nblk, summ_a, stream)
        hga.hga_cache_segment(hga.Dims(1, w.Hq, w.Hkv, w.d, w.blk, w.S, 0, w.topk, "bf16"), ks, vs, pk, pv, cache,
                              w.nblk, stream)

    def append_with_offload():
        cache.reset()
        hga.hga_append_segment(Da, ks, vs, w.nblk, summ_a, pk, pv, cache, tk, tv, cap, stream, copy_stream)
        stream.wait_stream(copy_stream)

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize(device)
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
            ts.append(e0.elapsed_time(e1))
        hga.hga_device_status(stream)
        return float(np.mean(ts))

    probe = h2d_probe(device)
    peaks, peak_src = load_peaks()
    fetch_bytes = n_sel * blk_bytes * 2
    seg_bytes = w.S * w.Hkv * w.d * 2
    res = {}
    for name, fn, nbytes, ref in (
            ("fetch_copy_engines", fetch, fetch_bytes, "h2d"), ("gather_mapped_sms", gather, fetch_bytes, "h2d"),
            ("remap_idx", remap, idx.numel() * 8, "hbm"),
            ("append_fused", append_fused, 4 * seg_bytes + w.nqb * w.Hkv * w.d * 4, "hbm"),
            ("append_separate", append_separate, 5 * seg_bytes + w.nqb * w.Hkv * w.d * 4, "hbm"),
            ("append_fused_with_tier_offload", append_with_offload, 2 * seg_bytes, "d2h")):
        ms = timed(fn)
        gbs = nbytes / (ms / 1e3) / 1e9
        e = {"ms": round(ms, 4), "bytes": int(nbytes), "gbs": round(gbs, 1)}
        if ref == "h2d":
            e["frac_of_h2d_probe"] = round(gbs / probe, 3)
        elif ref == "hbm":
            e["frac_hbm"] = round(gbs / peaks["hbm_gbs"], 3)
        res[name] = e
    return {"metric": "HGA history-tier paths on the Qwen3-8B-shaped layer (fetch, gather, remap, segment append)",
            "value": res["fetch_copy_engines"]["gbs"], "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded)",
            "config": {"workload": w.name, "selected_blocks": n_sel, "l2": "flushed between steps"},
            "h2d_probe_gbs": round(probe, 1), "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
            "paths": res}


# ---------------------------------------------------------------- oracle legs

def oracle_sample(w: synth.Workload, x, kv_heads):
    """One bounded sample of the workload on the fp64 oracle: selection for
    every head, then forward and backward for the given KV heads."""
    import oracle
    od = oracle.Dims(w.B, w.Hq, w.Hkv, w.d, w.blk, w.S, w.nblk, w.topk)
    q, kh = x["q"], x["k_hist"]
    idx, _ = oracle.select(od, q, kh)
    args = (q, x["k_seg"], x["v_seg"], kh, x["v_hist"], idx)
    oracle.attn_fwd(od, *args, kv_heads=kv_heads)
    oracle.attn_bwd(od, *args, x["d_o"], kv_heads=kv_heads)


def cpu_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


def run_cpu_baseline(w, x_inputs, budget_s=12.0):
    x = {n: getattr(x_inputs, n).f64 for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    t0 = time.perf_counter()
    done = 0
    while done < w.Hkv and (time.perf_counter() - t0) < budget_s:
        oracle_sample(w, x, range(done, done + 1))
        done += 1
    el = time.perf_counter() - t0
    out = {"value": round(w.S * (done / w.Hkv) / el, 2), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
           "sample": f"fp64 oracle: selection for all heads + fwd and bwd for {done} of {w.Hkv} KV heads "
                     f"({done * w.G} of {w.Hq} query heads) in {el:.1f} s, scaled to the full layer"}
    # the same oracle on one host core: selection for all heads + fwd and bwd of one KV head
    import oracle
    n0 = oracle.max_threads()
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle_sample(w, x, range(0, 1))
        el1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(n0)
    out["one_core"] = {"value": round(w.S * (1 / w.Hkv) / el1, 2), "unit": UNIT, "cores": 1,
                       "sample": f"fp64 oracle on 1 thread: selection for all heads + fwd and bwd for 1 of "
                                 f"{w.Hkv} KV heads in {el1:.1f} s, scaled to the full layer"}
    return out


def run_reference(args, rank, world=1):
    if rank != 0:
        return None
    w = synth.QWEN3_8B_LAYER
    xi = synth.draw(w)
    x = {n: getattr(xi, n).f64 for n in ("q", "k_seg", "v_seg", "k_hist", "v_hist", "d_o")}
    for _ in range(args.warmup):
        oracle_sample(w, x, range(0, 1))
    times = []
    for k in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample(w, x, range(k % w.Hkv, k % w.Hkv + 1))
        times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    value = w.S * (1 / w.Hkv) / (ms / 1e3)
    sample = (f"each step: fp64 oracle selection for all heads + fwd and bwd for 1 of {w.Hkv} KV heads "
              f"(4 query heads), scaled to the full layer (x{w.Hkv})")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
            "config": workload_config(w, "n/a (CPU)"),
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("hga", "reference"), default="hga")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--segmented-modes", default="host_tier,resident,host_tier_no_prefetch",
                    help="comma list of " + ", ".join(SEGMENTED_MODES) + " for --workload segmented")
    ap.add_argument("--pool-slots", type=int, default=None,
                    help="device pool (cache) slots per layer for --workload segmented (default: the largest history)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the 131K-token prefill and dense-equivalence sub-measurements of the default (layer) run")
    ap.add_argument("--workload", choices=("layer", "segmented", "dense", "prefill", "decode", "tier", "layer64",
                                           "layer32"),
                    default="layer",
                    help="layer: one Qwen3-8B-shaped layer step (the headline); layer64: the same layer with "
                         "64-token history blocks under 128-row query blocks; layer32: with 32-token history "
                         "blocks and K 64; segmented: the full 36-layer, "
                         "8-segment pass with the pinned host tier; dense / prefill: the dense-equivalence step and "
                         "the 131K prefill forward, device-timed only; decode: one new token at 131K context; "
                         "tier: the history-tier fetch, gather, remap and segment-append paths")
    args = ap.parse_args()
    if args.workload in ("dense", "prefill", "decode", "tier", "layer64", "layer32"):
        args.no_e2e = args.no_cpu_baseline = True
    if args.warmup < 3 and args.impl == "hga":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    try:
        if args.workload in ("segmented", "decode", "tier"):
            out = {"segmented": run_segmented, "decode": run_decode, "tier": run_tier}[args.workload](args, device)
            if rank == 0:
                print(json.dumps(out), flush=True)
            return
        out, ctx = run_device(args, rank, world, device)
        if not args.no_e2e:
            e2e = run_e2e(args, ctx, device)
            if world > 1:
                e2e["ms_per_step"] = round(max_over_ranks(e2e["ms_per_step"], world, device), 4)
                e2e["value"] = round(job_throughput(world, ctx[0].S, e2e["ms_per_step"]), 1)
            out["e2e"] = e2e
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = run_cpu_baseline(ctx[0], ctx[1])
        if args.workload == "layer" and not args.no_prefill:
            del ctx
            torch.cuda.empty_cache()
            pf, _ = run_device(args, rank, world, device, w=synth.PREFILL_131K, steps=min(args.steps, 20))
            out["prefill_131k"] = {k: pf[k] for k in ("value", "unit", "ms_per_step", "steps", "config", "kernels",
                                                      "attention_fwd", "launch", "eager", "gpu_launches", "clocks")}
            out["prefill_131k"]["metric"] = "HGA attn fwd tokens/s per layer (131K-token prefill, forward only)"
            de, _ = run_device(args, rank, world, device, w=synth.DENSE_EQUIV, steps=min(args.steps, 20))
            out["dense_equivalence"] = {k: de[k] for k in ("value", "unit", "ms_per_step", "steps", "config",
                                                           "kernels", "attention_fwd_bwd", "launch", "eager",
                                                           "gpu_launches")}
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
