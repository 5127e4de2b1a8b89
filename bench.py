#!/usr/bin/env python
"""Benchmark of the paged MLA decode hot path on B200.

One *step* is one pass of the whole hot path over one batch: the length-balanced
schedule (get_mla_metadata), the split-KV decode kernel and the merge kernel,
replayed as one CUDA graph (the kernels form a programmatic launch chain).

By default every one of the five decode workloads is timed back to back in one
process (tiny, uniform, varlen, causal2, skew; shapes and length recipes in
mla_workloads).  The headline line is the largest single-GPU workload, causal2
(batch 128, two causal query tokens x 128 heads, lengths U[1024, 8192], 724 MB
of KV), which is tensor-bound: ``value`` is its whole-job TFLOP/s per step
(flops of all ranks' steps / max-over-ranks device time of the K timed steps).
``per_config`` carries every workload's figures: us per step, per decode call
and for the decode kernel alone, TFLOP/s, KV-read GB/s, the roofline bound and
fraction, and the ncu DRAM traffic.  Workloads whose KV is larger than the
126 MB L2 run back to back; the tiny one is timed with an L2 flush before every
replay.

``roofline`` reports the split-KV decode kernel, replayed alone min(K, 300)
times right after the timed steps with CUDA events around each replay, against
the measured HBM or bf16 peak; ``us_per_call`` is the decode call.  ``e2e``
times the headline step through the public Python API from pinned host buffers
(inputs copied in, o and lse copied out every step).  ``cpu_baseline`` times
the fp64 oracle on the host cores on a bounded sample of the headline workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...     # the oracle as the reference arm
    python bench.py --profile --config NAME  # plain launches, for ncu
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_workloads as W  # noqa: E402

METRIC = "MLA decode TFLOPS & KV-read GB/s vs B200 roofline; µs per decode call"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def work_counts(inp: dict) -> dict:
    """Algorithmic bytes and flops of one decode call.

    Bytes: every cached row a query row can see, read once (576 bf16 per token
    per KV head), plus q read, o written (bf16) and lse written (fp32).  Split
    partials, page-tail padding and L2 re-reads are not algorithmic.
    Flops: 2 * (576 + 512) per (query row, visible token) pair.
    """
    lens = inp["cache_seqlens"].astype(np.int64)
    s_q, h_q, h_kv, b = inp["s_q"], inp["h_q"], inp["h_kv"], inp["batch"]
    kv_bytes = int(lens.sum()) * h_kv * W.D_QK * 2
    if inp["causal"]:
        vis = sum(int(np.clip(lens - (s_q - 1 - i), 0, None).sum()) for i in range(s_q))
    else:
        vis = int(lens.sum()) * s_q
    flops = 2 * (W.D_QK + W.D_V) * h_q * vis
    io_bytes = b * s_q * h_q * (W.D_QK * 2 + W.D_V * 2 + 4)
    return dict(kv_bytes=kv_bytes, bytes=kv_bytes + io_bytes, flops=flops, tokens=int(lens.sum()))


def roofline_time(wc, peaks, sustained=False):
    t_hbm = wc["bytes"] / (peaks["hbm_gbs"] * 1e9)
    tf = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    t_tc = wc["flops"] / (tf * 1e12)
    return (t_hbm, "hbm") if t_hbm >= t_tc else (t_tc, "tensor")


def workload_desc(w: W.Workload) -> str:
    return (f"{w.name} decode: batch={w.batch} s_q={w.s_q} h_q={w.h_q} h_kv={w.h_kv} d=576 dv=512 "
            f"page=64 causal={w.causal} lengths={w.seqlen_kind}{list(w.seqlen_args)} bf16 N(0,1)")


# ----------------------------------------------------------------------------- traffic
KERNEL_SOURCES = ["decode.cu", "ptx.cuh", "pagedmla_internal.cuh"]


def kernel_sources_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_mla_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(config: str):
    """DRAM bytes per decode-kernel launch from the committed ncu summary of this
    workload, or None when there is none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", f"decode_{config}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            parts = line.strip().split(":")
            if len(parts) == 2 and parts[0] in ("traffic_bytes_per_launch", "kernel_sources_sha256_16"):
                vals[parts[0]] = parts[1].strip()
    if vals.get("kernel_sources_sha256_16") != kernel_sources_hash():
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- ranks
def rank_inputs(w: W.Workload, rank: int) -> dict:
    """Each rank decodes its own batch of the same workload (weak scaling): the
    seed is offset by the rank, shapes and length distribution are shared."""
    return W.make_inputs(w, seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, kv_bytes_per_rank: int, per_step_s: float) -> float:
    """Whole-job KV-read bandwidth: every rank's KV bytes over the slowest rank's step time."""
    return world * kv_bytes_per_rank / per_step_s / 1e9


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.ok = [], 0, False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            log("clock sampling unavailable:", e)
            self.max_mhz = None
        self._stop = threading.Event()

    def sample(self):
        """One reading now (also taken at the start and the end of the timed region,
        so that a short timed loop still records more than one sample)."""
        if not self.ok:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self.sample()

    def summary(self):
        if not self.ok:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- our arm
L2_BYTES = 126 * 1024 * 1024
# The headline workload: the largest single-GPU configuration (batch 128, two
# causal query tokens, 128 heads, lengths U[1024, 8192]), the compute-bound one.
HEADLINE = "causal2"


def timed_replays(graph, n, stream, flush_buf=None, read_flush=False):
    """Replays `graph` n times on `stream`; returns the per-replay times (ms) from
    CUDA events recorded on that stream.  With `flush_buf` (larger than L2) the
    buffer is overwritten before every replay, outside the bracketing events, so
    each replay starts with a cold L2; without it the replays run back to back
    (used when the inputs are larger than L2).  `read_flush` reads the buffer
    instead of writing it: L2 then starts cold and clean, with no dirty lines
    whose write-back the timed kernels would pay for."""
    import torch
    with torch.cuda.stream(stream):
        if flush_buf is None:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
            ev[0].record(stream)
            for k in range(n):
                graph.replay()
                ev[k + 1].record(stream)
            torch.cuda.synchronize()
            return [ev[k].elapsed_time(ev[k + 1]) for k in range(n)]
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        sink = torch.empty((1,), dtype=flush_buf.dtype, device=flush_buf.device)
        for k in range(n):
            if read_flush:
                torch.sum(flush_buf, dim=0, keepdim=True, out=sink)
            else:
                flush_buf.add_(1)
            ev0[k].record(stream)
            graph.replay()
            ev1[k].record(stream)
        torch.cuda.synchronize()
        return [ev0[k].elapsed_time(ev1[k]) for k in range(n)]


def bench_ours(args, rank, world, local_rank, name, headline):
    """Times one workload: K whole steps (schedule + counter clear + decode kernel +
    merge kernel, one CUDA graph per step), then the decode kernel alone and the
    decode call alone, each replayed min(K, 300) times with events around every
    replay.  For the headline workload also the end-to-end run from host buffers."""
    import torch
    import paged_mla_attention_b200 as pm
    sys.path.insert(0, os.path.join(ROOT, "tests"))

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[name]
    inp = rank_inputs(w, rank)   # weak scaling: each rank its own batch
    wc = work_counts(inp)
    peaks, peaks_src = load_peaks()

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    host = dict(q=up(inp["q"]).pin_memory(), kvcache=up(inp["kvcache"]).pin_memory(),
                block_table=torch.from_numpy(inp["block_table"]).pin_memory(),
                cache_seqlens=torch.from_numpy(inp["cache_seqlens"]).pin_memory())
    d = {k: v.to(dev) for k, v in host.items()}
    R = inp["s_q"] * inp["h_q"] // inp["h_kv"]
    o = torch.empty((inp["batch"], inp["s_q"], inp["h_q"], W.D_V), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((inp["batch"], inp["h_q"], inp["s_q"]), dtype=torch.float32, device=dev)
    ws = torch.empty((pm.workspace_bytes(inp["batch"], inp["s_q"], inp["h_q"], inp["h_kv"]),),
                     dtype=torch.uint8, device=dev)

    meta_holder = {}

    def step_meta():
        meta_holder["m"], meta_holder["s"] = pm.get_mla_metadata(d["cache_seqlens"], R, inp["h_kv"])

    def step_decode(stage="all"):
        pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], W.D_V,
                                  meta_holder["m"], meta_holder["s"], inp["causal"], inp["softmax_scale"],
                                  out=(o, lse), workspace=ws, stage=stage)

    if args.profile:
        # minimal plain-launch run for ncu: W warm-up steps then K steps, no graphs
        for _ in range(args.warmup + args.steps):
            step_meta()
            step_decode()
        torch.cuda.synchronize(dev)
        err = pm.device_error()
        if err:
            raise RuntimeError(f"device error {err}")
        return None, inp, wc

    # inputs that fit in L2 (the tiny parity workload) are timed with an L2 flush
    # before every replay; the others are larger than L2 and run back to back
    flush_buf = (torch.zeros((2 * L2_BYTES // 4,), dtype=torch.int32, device=dev)
                 if wc["kv_bytes"] < 2 * L2_BYTES else None)

    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            step_meta()
            step_decode()
    torch.cuda.current_stream(dev).wait_stream(stream)
    torch.cuda.synchronize(dev)
    err = pm.device_error()
    if err:
        raise RuntimeError(f"device error {err} during warm-up")
    # a schedule with lighter parts (weight < 128) runs them as a second decode launch
    decode_launches_extra = int(bool((meta_holder["m"][:, 5] < 128).any().item()))

    # CUDA graphs: the whole step (schedule, counter clear, decode kernel, merge
    # kernel: a programmatic launch chain, so each kernel's launch overlaps the
    # one before); the decode call alone (schedule excluded); and the decode
    # kernel alone, for the roofline
    g_meta, g_all, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_meta, stream=stream):
        step_meta()
    with torch.cuda.graph(g_all, stream=stream):
        step_decode("all")
    with torch.cuda.graph(g_dec, stream=stream):
        step_decode("decode")
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step_meta()
        step_decode("all")
    with torch.cuda.stream(stream):
        for _ in range(3):
            g_meta.replay()  # fills the schedule that g_all and g_dec read
            g_step.replay()
            g_all.replay()
            g_dec.replay()
    torch.cuda.synchronize(dev)

    K = args.steps
    KA = min(K, 300)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        if flush_buf is None:
            with torch.cuda.stream(stream):
                ev_start = torch.cuda.Event(enable_timing=True)
                ev_end = torch.cuda.Event(enable_timing=True)
                ev_start.record(stream)
                for k in range(K):
                    g_step.replay()
                ev_end.record(stream)
            torch.cuda.synchronize(dev)
            elapsed_ms = ev_start.elapsed_time(ev_end)
        else:
            elapsed_ms = float(np.sum(timed_replays(g_step, K, stream, flush_buf)))
        clk.sample()
        # the decode kernel alone, then the decode call alone: KA more replays each
        # right after the timed steps (same stream, same inputs), each bracketed by
        # events; KA is capped so that these runs add little heat after long step loops
        dec_ms = float(np.mean(timed_replays(g_dec, KA, stream, flush_buf)))   # clear + decode kernel
        call_ms = float(np.mean(timed_replays(g_all, KA, stream, flush_buf)))  # clear + decode + merge
    if world > 1:
        dist.barrier()
    err = pm.device_error()
    if err:
        raise RuntimeError(f"device error {err} in the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    t_roof, bound = roofline_time(wc, peaks)
    per_step_s = elapsed_ms / 1e3 / K
    if bound == "tensor":
        value, unit = world * wc["flops"] / per_step_s / 1e12, "TFLOP/s"
    else:
        value, unit = whole_job_gbs(world, wc["kv_bytes"], per_step_s), "GB/s"

    e2e = None
    if headline:
        # end-to-end through the public API from pinned host buffers
        e2e_steps = max(3, min(K, args.e2e_steps))
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

        def e2e_step():
            dd = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
            m, s = pm.get_mla_metadata(dd["cache_seqlens"], R, inp["h_kv"])
            oo, ll = pm.flash_mla_with_kvcache(dd["q"], dd["kvcache"], dd["block_table"],
                                               dd["cache_seqlens"], W.D_V, m, s, inp["causal"],
                                               inp["softmax_scale"])
            o_h.copy_(oo, non_blocking=True)
            lse_h.copy_(ll, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e_s = e2e_ms / 1e3 / e2e_steps
        e2e_v = (world * wc["flops"] / e2e_s / 1e12) if unit == "TFLOP/s" else (world * wc["kv_bytes"] / e2e_s / 1e9)
        e2e = {"value": round(e2e_v, 3), "unit": unit, "steps": e2e_steps, "ms_per_step": round(e2e_s * 1e3, 4),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # correctness spot-check of this very run against the oracle (rank 0, two sequences)
    spot = None
    if rank == 0 and not args.no_spot_check:
        import oracle
        from gpu_helpers import compare, subset
        seqs = [0, inp["batch"] - 1]
        sub = subset(inp, seqs, list(range(0, inp["h_q"], 8)))
        ro, rl = oracle.decode_inputs(sub)
        og = o.float().cpu().numpy()[seqs][:, :, ::8].astype(np.float64)
        lg = lse.cpu().numpy()[seqs][:, ::8].astype(np.float64)
        spot = compare(og, lg, ro, rl, what="bench spot check")

    dec_s = dec_ms / 1e3
    if bound == "hbm":
        achieved = wc["bytes"] / dec_s / 1e9
        peak, runit = peaks["hbm_gbs"], "GB/s"
    else:
        achieved = wc["flops"] / dec_s / 1e12
        peak, runit = peaks["bf16_tflops"], "TFLOP/s"
    l2 = ("inputs fit in L2: L2 flushed (256 MB write) before every timed replay" if flush_buf is not None
          else f"inputs ({wc['kv_bytes'] / 1e6:.0f} MB KV) larger than the 126 MB L2; no flush")
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(elapsed_ms / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "global_batch": inp["batch"] * world,
                   "kv_tokens_per_gpu": wc["tokens"], "parallelism": f"replicas x{world} (batch-sharded, no exchange)",
                   "l2": l2,
                   "step": "schedule + counter clear + split-KV decode + merge, one CUDA graph per step"},
        "us_decode_kernel": round(dec_ms * 1e3, 3),
        "us_per_call": round(call_ms * 1e3, 3),
        "tflops": round(wc["flops"] / dec_s / 1e12, 2),
        "tflops_per_call": round(wc["flops"] / (call_ms / 1e3) / 1e12, 2),
        "kv_read_gbs_per_call": round(wc["kv_bytes"] / (call_ms / 1e3) / 1e9, 1),
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": runit,
                     "frac": round(achieved / peak, 4), "traffic": (args.traffic if args.traffic is not None
                                                               else measured_traffic(name)),
                     "traffic_unit": "bytes per decode call's decode launches (ncu dram read + write)",
                     "kernel": ("split-KV decode kernels: the 4-CTA launch and the 2-CTA launch on the SMs it "
                                "leaves free, timed alone together; the merge kernel follows them"
                                if decode_launches_extra else
                                "split-KV decode kernel (timed alone; the merge kernel follows it)"),
                     "peak_source": f"{peaks_src} (MEASURED_PEAKS.json)" if peaks_src == "measured" else "fallback",
                     "algorithmic_bytes": wc["bytes"], "algorithmic_flops": wc["flops"],
                     "roofline_us": round(t_roof * 1e6, 2),
                     "frac_of_roofline_time": round(t_roof / dec_s, 4)},
        # schedule, counter clear, decode (two launches when parts run on the SMs
        # the 4-CTA clusters leave free: metadata weight < 128), merge per timed step
        "gpu_launches": (4 + decode_launches_extra) * K,
        "clocks": clk.summary(),
    }
    if e2e is not None:
        result["e2e"] = e2e
    if spot is not None:
        result["parity_spot_check"] = {k: float(f"{v:.4g}") for k, v in spot.items()}
    return result, inp, wc


def config_summary(res: dict) -> dict:
    """The per-workload figures carried in the headline line's per_config object."""
    r = res["roofline"]
    return {"workload": res["config"]["workload"], "us_per_step": round(res["ms_per_step"] * 1e3, 3),
            "us_per_call": res["us_per_call"], "us_decode_kernel": res["us_decode_kernel"],
            "tflops": res["tflops"], "kv_read_gbs": round(res["kv_read_gbs_per_call"], 1),
            "bound": r["bound"], "achieved": r["achieved"], "peak": r["peak"], "unit": r["unit"],
            "frac": r["frac"], "roofline_us": r["roofline_us"], "traffic": r["traffic"],
            "l2": res["config"]["l2"], "clocks": res["clocks"]}


def cpu_baseline(inp, wc, budget_s, unit="GB/s"):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload,
    in the headline's unit (KV GB/s, or TFLOP/s for a tensor-bound workload)."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from gpu_helpers import subset
    order = list(range(inp["batch"]))
    done_tokens, t_total, seqs_done = 0, 0.0, 0
    for b in order:
        sub = subset(inp, [b])
        t = time.perf_counter()
        oracle.decode_inputs(sub)
        t_total += time.perf_counter() - t
        done_tokens += int(inp["cache_seqlens"][b])
        seqs_done += 1
        if t_total >= budget_s:
            break
    frac = done_tokens / max(wc["tokens"], 1)
    value = frac * (wc["flops"] / 1e12 if unit == "TFLOP/s" else wc["kv_bytes"] / 1e9) / t_total
    return {"value": round(value, 8), "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{seqs_done} of {inp['batch']} sequences (all heads, all tokens), "
                      f"{frac:.3f} of the workload's KV-token work, fp64, {t_total:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def bench_reference(args):
    """The fp64 oracle on the host cores, timed on a bounded sample per step."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from gpu_helpers import subset
    w = W.WORKLOADS[args.config or HEADLINE]
    inp = W.make_inputs(w)
    wc = work_counts(inp)
    peaks, _ = load_peaks()
    unit = "TFLOP/s" if roofline_time(wc, peaks)[1] == "tensor" else "GB/s"
    # size each step so that warm-up + timed steps take about `budget` seconds
    probe = subset(inp, [0], [0, 1])
    t = time.perf_counter()
    oracle.decode_inputs(probe)
    per_head = max((time.perf_counter() - t) / 2, 1e-5)
    budget = args.reference_budget
    heads = int(np.clip(budget / (args.steps + args.warmup) / per_head, 1, inp["h_q"]))
    def one(k):
        b = k % inp["batch"]
        hs = [(k * heads + j) % inp["h_q"] for j in range(heads)]
        sub = subset(inp, [b], sorted(set(hs)))
        t0 = time.perf_counter()
        oracle.decode_inputs(sub)
        return time.perf_counter() - t0, int(inp["cache_seqlens"][b]) * len(set(hs))
    for k in range(args.warmup):
        one(k)
    tt, work = 0.0, 0
    for k in range(args.steps):
        dt, wk = one(args.warmup + k)
        tt += dt
        work += wk
    frac = work / (wc["tokens"] * inp["h_q"])
    value = frac * (wc["flops"] / 1e12 if unit == "TFLOP/s" else wc["kv_bytes"] / 1e9) / tt
    sample = (f"each step: 1 sequence x {heads} of {inp['h_q']} heads (all tokens); "
              f"{frac:.4f} of one workload's row-token work in total, fp64")
    return {
        "metric": METRIC, "value": round(value, 8), "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_desc(w), "global_batch": inp["batch"]},
        "cpu_baseline": {"value": round(value, 8), "unit": unit, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 8), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def bench_append(args):
    """The cache append (mla_append_kvcache), timed with CUDA events per launch on
    two shapes: one decode step (64 sequences x 1 new token) and a 1024-token
    prefill into 64 sequences.  HBM-bound: 2 x 1152 bytes per (token, KV head)."""
    import torch
    import paged_mla_attention_b200 as pm
    peaks, _ = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rng = np.random.default_rng(7)
    out = []
    for name, batch, s_new, L0 in (("decode step", 64, 1, 4096), ("prefill 1024", 64, 1024, 0)):
        pages_per = (L0 + s_new + 63) // 64
        pool = batch * pages_per
        bt = torch.from_numpy(rng.permutation(pool).astype(np.int32).reshape(batch, pages_per)).to(dev)
        kv = torch.empty((pool, 64, 1, W.D_QK), dtype=torch.bfloat16, device=dev)
        new = torch.randn((batch, s_new, 1, W.D_QK), device=dev).to(torch.bfloat16)
        lens = torch.full((batch,), L0, dtype=torch.int32, device=dev)
        stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                pm.append_kvcache(new, bt, lens, kv)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()            # one launch per replay, no host overhead inside
        with torch.cuda.graph(g, stream=stream):
            pm.append_kvcache(new, bt, lens, kv)
        g.replay()
        torch.cuda.synchronize(dev)
        K = max(args.steps, 10)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        ev[0].record()
        for k in range(K):
            g.replay()
            ev[k + 1].record()
        torch.cuda.synchronize(dev)
        if pm.device_error():
            raise RuntimeError("device error in the append bench")
        us = float(np.mean([ev[k].elapsed_time(ev[k + 1]) for k in range(K)])) * 1e3
        nbytes = 2 * batch * s_new * W.D_QK * 2
        gbs = nbytes / (us * 1e-6) / 1e9
        out.append({"shape": f"{name}: batch {batch} x {s_new} tokens, h_kv 1", "us_per_call": round(us, 3),
                    "bytes": nbytes, "achieved_gbs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4)})
    return {"metric": "KV-cache append GB/s (read new rows + write cache rows)", "append": out,
            "n_gpus": 1, "steps": max(args.steps, 10)}


def bench_proj(args):
    """The absorbed projections (mla_absorb_query before the decode, mla_project_output
    after it), timed with CUDA events at three token counts with 128 heads, two ways:
    one call alone per graph replay, and a chain of 8 calls in one graph, one per
    "layer", each with its own weights and activations (8 x 16.8 MB of weights, more
    than L2), as a model runs them; the kernels are programmatic dependents of the
    kernel before them, so in the chain each call's launch, setup and weight prefetch
    overlap the previous call's tail.  L2 is flushed (by reading a buffer twice its
    size, which leaves no dirty lines) before every replay.
    Algorithmic bytes: activations in and out plus each head's 128 x 512 bf16 weight
    matrix once (the kernels re-read it per 128-token tile, mostly from L2); FLOPs
    2 x 128 x 512 per (token, head)."""
    import torch
    import paged_mla_attention_b200 as pm
    peaks, _ = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H, LAYERS = 128, 8
    flush_buf = torch.zeros((2 * L2_BYTES // 4,), dtype=torch.int32, device=dev)
    out = []
    for T in (64, 128, 1024):
        def rnd(*shape, scale=1.0):
            return [(torch.randn(shape, device=dev) * scale).to(torch.bfloat16) for _ in range(LAYERS)]
        qn, qr, ol = rnd(T, H, 128), rnd(T, H, 64), rnd(T, H, 512)
        w_uk, w_uv = rnd(H, 128, 512, scale=1 / 11.3), rnd(H, 128, 512, scale=1 / 22.6)
        q = [torch.empty((T, H, 576), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        o = [torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        wbytes = H * 128 * 512 * 2
        for name, fn, nbytes in (
                ("absorb_query", lambda l: pm.absorb_query(qn[l], qr[l], w_uk[l], out=q[l]),
                 T * H * (192 + 576) * 2 + wbytes),
                ("project_output", lambda l: pm.project_output(ol[l], w_uv[l], out=o[l]),
                 T * H * (512 + 128) * 2 + wbytes)):
            stream = torch.cuda.Stream(dev)
            with torch.cuda.stream(stream):
                for _ in range(max(args.warmup, 3)):
                    for l in range(LAYERS):
                        fn(l)
            torch.cuda.synchronize(dev)
            g1, gl = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1, stream=stream):
                fn(0)
            with torch.cuda.graph(gl, stream=stream):
                for l in range(LAYERS):
                    fn(l)
            g1.replay()
            gl.replay()
            torch.cuda.synchronize(dev)
            K = max(args.steps, 10)
            us1 = float(np.mean(timed_replays(g1, K, stream, flush_buf, read_flush=True))) * 1e3
            usl = float(np.mean(timed_replays(gl, K, stream, flush_buf, read_flush=True))) * 1e3 / LAYERS
            if pm.device_error():
                raise RuntimeError("device error in the projection bench")
            for mode, us in (("chain of 8 layers (per call)", usl), ("one call alone", us1)):
                gbs = nbytes / (us * 1e-6) / 1e9
                tfs = 2.0 * T * H * 128 * 512 / (us * 1e-6) / 1e12
                out.append({"kernel": name, "tokens": T, "heads": H, "timing": mode, "us_per_call": round(us, 3),
                            "bytes": nbytes, "achieved_gbs": round(gbs, 1),
                            "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4),
                            "tflops": round(tfs, 2), "frac_of_bf16_peak": round(tfs / peaks["bf16_tflops"], 4)})
    return {"metric": "absorbed projection kernels (us per call; HBM and tensor fractions)", "proj": out,
            "n_gpus": 1, "steps": max(args.steps, 10), "l2": "flushed before every replay (read of 252 MB)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=None, choices=list(W.WORKLOADS),
                    help="bench this workload only (default: all five, headline " + HEADLINE + ")")
    ap.add_argument("--out", default=None)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--reference-budget", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-spot-check", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="plain launches only (warm-up + steps), for ncu; prints one short line")
    ap.add_argument("--append", action="store_true",
                    help="time the cache append kernel instead (one JSON line)")
    ap.add_argument("--proj", action="store_true",
                    help="time the absorbed projection kernels instead (one JSON line)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per decode call from an ncu capture of the same kernels")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(bench_reference(args)), flush=True)
        return
    if args.proj:
        if rank == 0:
            print(json.dumps(bench_proj(args)), flush=True)
        return
    if args.append:
        if rank == 0:
            print(json.dumps(bench_append(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.profile:
            bench_ours(args, rank, world, local_rank, args.config or HEADLINE, False)
            if rank == 0:
                print(json.dumps({"profile_run": args.config or HEADLINE, "steps": args.steps,
                                  "warmup": args.warmup}))
            return
        # every workload back to back in one process (or the one --config names);
        # the headline line is the largest workload, with the others in per_config
        headline = args.config or HEADLINE
        configs = [args.config] if args.config else list(W.WORKLOADS)
        per_config, main = {}, None
        for name in configs:
            res, inp, wc = bench_ours(args, rank, world, local_rank, name, name == headline)
            per_config[name] = config_summary(res)
            if name == headline:
                main = (res, inp, wc)
            if rank == 0:
                log(json.dumps(res))
        res, inp, wc = main
        res["per_config"] = per_config
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(inp, wc, args.cpu_budget, res["unit"])
        if rank == 0:
            if args.out:
                with open(args.out, "w") as f:
                    f.write(json.dumps(res) + "\n")
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
