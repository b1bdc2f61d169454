#!/usr/bin/env python
"""Attention backward throughput on B200: one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic input:
attn_fwd (O and LSE) followed by attn_bwd (dQ, dK, dV). The metric is the
backward's counted FLOPs (2.5x the forward's two matmuls, 4*B*H*n*m*d, halved
when causal) over the backward's device time, in TFLOP/s, summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the float64 CPU oracle, timed

With N > 1 the script runs under torch.distributed.run, one rank per GPU. The
(batch, head) problems are independent, so there is no collective on the data
path in either of the two ways of spreading work over ranks:
  --split replicas (default)  every rank runs the whole workload on its own
                              seeded data ("weak" scaling);
  --split heads               the ranks share one workload: rank r takes a
                              contiguous slice of its B*H problems, the same
                              inputs the 1-GPU run sees ("strong" scaling).
The timed region is bracketed by barriers and reduced as a max over ranks;
`value` is all ranks' counted FLOPs over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

DEFAULT_WORKLOAD = "causal_b2h32_n4096_d128"
METRIC = "attn backward TFLOP/s (bf16, causal) and % of B200 dense-BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "bwd_tc_causal_b2h32_n4096_d128.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "scaled_dot_product_saving_b200", "csrc", f)
                  for f in ("bwd_tc.cuh", "sm100.cuh")]


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    p.add_argument("--e2e-steps", type=int, default=16)
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--path", choices=["auto", "simt", "tensor"], default="auto",
                   help="kernel path the library may use (attn_set_path)")
    p.add_argument("--proj", action="store_true",
                   help="time attn_proj_bwd (projection and input gradients) instead")
    p.add_argument("--dq-path", choices=["auto", "reduce", "separate"], default="auto",
                   help="how the bf16 tensor-core backward computes dQ (attn_set_dq_path)")
    p.add_argument("--split", choices=["replicas", "heads"], default="replicas",
                   help="replicas: every rank runs the whole workload; heads: the ranks "
                        "share the workload's (batch, head) problems")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    if a.steps < 1:
        p.error("--steps must be >= 1")
    return a


# ---------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the backward kernel from the committed ncu
    summary, or None when it is missing, for another workload, or taken on a
    kernel source that has changed since."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            fields = dict(line.split(":", 1) for line in f if ":" in line)
    except OSError:
        return None
    fields = {k.strip(): v.strip() for k, v in fields.items()}
    if fields.get("workload") != workload or fields.get("source_sha256") != kernel_source_hash():
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count() or 1


def metric_for(w: synth.Workload) -> str:
    """The headline metric, with its precision and mask tags for the workload."""
    tags = ["bf16" if w.dtype == "bf16" else "fp32", "causal" if w.causal else "non-causal"]
    if w.key_len() is not None:
        tags.append("key padding mask")
    return METRIC.replace("(bf16, causal)", "(" + ", ".join(tags) + ")")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nvml = None

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                mask = get(self.handle)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- multi-rank
def init_distributed(backend=None):
    """Join the process group described by RANK / WORLD_SIZE / LOCAL_RANK
    (torch.distributed.run sets them); NCCL on GPUs, gloo otherwise."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def max_over_ranks(values, world, device):
    """Element-wise max of a list of floats over all ranks."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate(per_rank_flops, local_ms, world, device):
    """Whole-job throughput: all ranks' FLOPs over the slowest rank's time."""
    (slowest_ms,) = max_over_ranks([local_ms], world, device)
    return world * per_rank_flops / (slowest_ms * 1e-3) / 1e12, slowest_ms


def sum_over_ranks(value, world, device):
    if world == 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_slice(problems, rank, world):
    """Rank `rank`'s contiguous share [lo, hi) of `problems` (batch, head)
    problems numbered b*H + h; the shares of all ranks tile [0, problems)."""
    return problems * rank // world, problems * (rank + 1) // world


def slice_runs(B, H, lo, hi):
    """Problems [lo, hi) as runs the library takes in one call each, as
    (b0, nb, h0, nh): whole batch elements b0..b0+nb-1 (h0 = 0, nh = H), or
    heads h0..h0+nh-1 of the single batch element b0 (nb = 1)."""
    runs, p = [], lo
    while p < hi:
        b, h = divmod(p, H)
        if h == 0 and hi - p >= H:
            nb = (hi - p) // H
            runs.append((b, nb, 0, H))
            p += nb * H
        else:
            nh = min(H - h, hi - p)
            runs.append((b, 1, h, nh))
            p += nh
    return runs


def run_flops(w, run):
    """Counted backward FLOPs of one run of problems."""
    b0, nb, _, nh = run
    return sum(nh * w.head_bwd_flops(b) for b in range(b0, b0 + nb))


def make_parts(w, split, rank, world):
    """The CPU inputs this rank works on, as a list of parts: (sub-workload,
    (q, k, v, do), key lengths or None, counted backward FLOPs). A part is one
    attn_fwd + attn_bwd call."""
    if split == "replicas":
        return [(w, synth.make_inputs(w, seed=w.seed + 1000 * rank), w.key_len(), w.bwd_flops())]
    q, k, v, do = synth.make_inputs(w)               # the 1-GPU run's inputs
    kl = w.key_len()
    parts = []
    for run in slice_runs(w.B, w.H, *rank_slice(w.B * w.H, rank, world)):
        b0, nb, h0, nh = run
        sub = dataclasses.replace(w, name=f"{w.name}[b{b0}:{b0 + nb},h{h0}:{h0 + nh}]", B=nb, H=nh,
                                  lengths=None if kl is None else tuple(kl[b0:b0 + nb]), pad_min=0)
        ts = tuple(t[b0:b0 + nb, h0:h0 + nh].contiguous() for t in (q, k, v, do))
        parts.append((sub, ts, None if kl is None else kl[b0:b0 + nb], run_flops(w, run)))
    return parts


# ---------------------------------------------------------------- our arm
def run_ours(args, w, rank, world, local):
    import scaled_dot_product_saving_b200 as lib

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib.attn_set_path({"auto": lib.ATTN_PATH_AUTO, "simt": lib.ATTN_PATH_SIMT,
                       "tensor": lib.ATTN_PATH_TENSOR}[args.path])
    lib.attn_set_dq_path({"auto": lib.ATTN_DQ_AUTO, "reduce": lib.ATTN_DQ_REDUCE,
                          "separate": lib.ATTN_DQ_SEPARATE}[args.dq_path])

    # Device buffers of every part (one attn_fwd + attn_bwd call each).
    class Part:
        def __init__(self, sub, cpu, kl_list, flops):
            self.w, self.flops = sub, flops
            self.q, self.k, self.v, self.do = (t.to(dev) for t in cpu)
            self.kl = None if kl_list is None else torch.tensor(kl_list, dtype=torch.int32,
                                                                device=dev)
            self.o = torch.empty((sub.B, sub.H, sub.n, sub.dv), dtype=self.q.dtype, device=dev)
            self.lse = torch.empty((sub.B, sub.H, sub.n), dtype=torch.float32, device=dev)
            self.dq, self.dk, self.dv = (torch.empty_like(t) for t in (self.q, self.k, self.v))
            self.ws = torch.empty(lib.attn_bwd_workspace_size(sub.B, sub.H, sub.n, sub.m, sub.d,
                                                              sub.dv, self.q.dtype),
                                  dtype=torch.uint8, device=dev)

        def tensors(self):
            return (self.q, self.k, self.v, self.o, self.do, self.dq, self.dk, self.dv, self.ws)

        def fwd(self, stream=None):
            lib.attn_fwd(self.q, self.k, self.v, causal=self.w.causal, scale=self.w.scale,
                         out=self.o, lse=self.lse, key_len=self.kl, stream=stream)

        def bwd(self, stream=None):
            lib.attn_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, causal=self.w.causal,
                         scale=self.w.scale, workspace=self.ws, dq=self.dq, dk=self.dk,
                         dv=self.dv, key_len=self.kl, stream=stream)

    parts = [Part(*p) for p in make_parts(w, args.split, rank, world)]
    local_flops = sum(p.flops for p in parts)
    working_set = sum(t.numel() * t.element_size() for p in parts for t in p.tensors())
    flush = None
    if working_set < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step(evs=None):
        if flush is not None:
            flush.zero_()
        if evs:
            evs[0].record()
        for p in parts:
            p.fwd()
        if evs:
            evs[1].record()
        for p in parts:
            p.bwd()
        if evs:
            evs[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if lib.attn_get_device_error() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world, local)
    torch.cuda.synchronize()
    sampler.start()
    t_start.record()
    for s in range(args.steps):
        step(evs[s])
    t_end.record()
    torch.cuda.synchronize()
    barrier(world, local)
    sampler.stop()
    if lib.attn_get_device_error() != 0:
        raise RuntimeError("device-side timeout in the timed region")
    # The per-kernel breakdown comes from a second, traced run of the same
    # steps: the library's trace events sit between its kernels, where they
    # would keep the backward from starting its setup under the preprocess
    # kernel's tail, so the timed run above is untraced.
    lib.attn_trace_begin(min(65536, 8 * len(parts) * args.steps))
    for s in range(args.steps):
        step()
    torch.cuda.synchronize()
    trace = lib.attn_trace_end()
    if lib.attn_get_device_error() != 0:
        raise RuntimeError("device-side timeout in the traced run")

    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    bwd_sum, fwd_sum = sum(bwd_ms), sum(fwd_ms)
    slow_total, slow_bwd, slow_fwd = max_over_ranks([total_ms, bwd_sum, fwd_sum], world, dev)
    job_flops = sum_over_ranks(local_flops, world, dev)            # backward FLOPs of one step
    job_fwd_flops = job_flops * w.fwd_flops() / w.bwd_flops()
    value = args.steps * job_flops / (slow_bwd * 1e-3) / 1e12

    by_kernel = {}
    for name, ms in trace:
        by_kernel.setdefault(name, []).append(ms)
    peaks, peaks_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_note = f"bf16_tflops ({peaks_src}, burst)"
    # FLOPs each backward kernel performs, as a share of the counted backward
    # FLOPs (five contractions): the fused kernel all five; the separate dK/dV
    # pass four (S, dP, dV, dK) and the dQ pass three (S and dP again, dQ).
    share = {"bwd_tensor": 1.0, "bwd_simt": 1.0, "bwd_f32x": 1.0, "bwd_kv": 0.8, "bwd_dq": 0.6}
    if "bwd_f32x" in by_kernel:
        # fp32 by bf16 pieces: six bf16 MMAs per fp32 product, so the peak is
        # a sixth of the bf16 one. The one launch runs both passes (the dQ
        # pass recomputes S and dP, which the count does not credit).
        main = "bwd_f32x"
        peak, peak_note = peak / 6.0, f"bf16_tflops / 6 ({peaks_src}, burst)"
    elif "bwd_kv" in by_kernel:
        main = max(("bwd_kv", "bwd_dq"), key=lambda k2: sum(by_kernel[k2]))
    else:
        main = "bwd_tensor" if "bwd_tensor" in by_kernel else "bwd_simt"

    def kernel_tflops(name):
        # the kernel's own FLOPs per step over its device time per step
        ms = statistics.mean(by_kernel[name]) * len(by_kernel[name]) / args.steps
        return share[name] * local_flops / (ms * 1e-3) / 1e12
    achieved = kernel_tflops(main)
    per_kernel = {k2: {"tflops": round(kernel_tflops(k2), 3), "frac": round(kernel_tflops(k2) / peak, 4)}
                  for k2 in by_kernel if k2 in share}

    # End to end through the public API with host buffers. Every step copies
    # its Q, K, V, dO in from pinned host memory, runs attn_fwd + attn_bwd and
    # copies dQ, dK, dV back; steps are pipelined over two device buffer sets
    # and three streams, so step i+1's upload and step i-1's download overlap
    # step i's kernels, as a training loop feeding the library would.
    e2e = None
    if args.e2e_steps > 0:
        sets = [parts, [Part(p.w, (p.q.cpu(), p.k.cpu(), p.v.cpu(), p.do.cpu()),
                             None if p.kl is None else p.kl.tolist(), p.flops) for p in parts]]
        pin_in = [[[t.to("cpu").pin_memory() for t in (p.q, p.k, p.v, p.do)
                    + (() if p.kl is None else (p.kl,))] for p in parts] for _ in range(2)]
        pin_out = [[[torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                     for t in (p.dq, p.dk, p.dv)] for p in parts] for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for pp in pin_in[0] for t in pp)
        d2h = sum(t.numel() * t.element_size() for pp in pin_out[0] for t in pp)
        s_in, s_run, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_run = [torch.cuda.Event() for _ in range(2)]
        ev_free = [torch.cuda.Event() for _ in range(2)]
        for e in ev_free:
            e.record(torch.cuda.current_stream())

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev_free[b])
            with torch.cuda.stream(s_in):
                for p, srcs in zip(sets[b], pin_in[b]):
                    dsts = (p.q, p.k, p.v, p.do) + (() if p.kl is None else (p.kl,))
                    for src, dst in zip(srcs, dsts):
                        dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
            s_run.wait_event(ev_in[b])
            for p in sets[b]:
                p.fwd(stream=s_run)
            for p in sets[b]:
                p.bwd(stream=s_run)
            ev_run[b].record(s_run)
            s_out.wait_event(ev_run[b])
            with torch.cuda.stream(s_out):
                for p, dsts in zip(sets[b], pin_out[b]):
                    for src, dst in zip((p.dq, p.dk, p.dv), dsts):
                        dst.copy_(src, non_blocking=True)
                ev_free[b].record(s_out)

        for i in range(2):                       # untimed: one round of both buffer sets
            e2e_step(i)
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        eb.record(s_out)
        torch.cuda.synchronize()
        if lib.attn_get_device_error() != 0:
            raise RuntimeError("device-side timeout in the end-to-end leg")
        (slow_e2e,) = max_over_ranks([ea.elapsed_time(eb)], world, dev)
        e2e = {"value": round(args.e2e_steps * job_flops / (slow_e2e * 1e-3) / 1e12, 3),
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(slow_e2e / args.e2e_steps, 4),
               "pipelined": "2 buffer sets, upload/compute/download streams"}

    kl_list = w.key_len()
    if world == 1:
        parallelism = "single GPU"
    elif args.split == "heads":
        parallelism = f"(batch, head) problems split over {world} ranks"
    else:
        parallelism = f"replicas: the whole workload on each of {world} ranks"
    result = {
        "metric": metric_for(w),
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(slow_total / args.steps, 4),
        "higher_is_better": True,
        "scaling": "strong" if args.split == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "H": w.H, "n": w.n, "m": w.m, "d": w.d, "dv": w.dv,
            "causal": w.causal, "scale": w.scale, "path": args.path, "dq_path": args.dq_path,
            **({} if kl_list is None else {"key_len": kl_list}),
            "parallelism": parallelism,
            "l2": ("flushed between steps (256 MiB write)" if flush is not None else
                   f"inputs larger than L2 ({working_set / 2**20:.0f} MiB per step)"),
        },
        "fwd_ms": round(slow_fwd / args.steps, 4),
        "bwd_ms": round(slow_bwd / args.steps, 4),
        "fwd_tflops": round(args.steps * job_fwd_flops / (slow_fwd * 1e-3) / 1e12, 3),
        "frac_of_datasheet_bf16": round(value / world / DATASHEET_BF16_TFLOPS, 4),
        "kernel_ms": {k2: round(statistics.mean(v2), 4) for k2, v2 in by_kernel.items()},
        "roofline": {
            "bound": "tensor", "kernel": main, "achieved": round(achieved, 3),
            "peak": round(peak, 3), "peak_source": peak_note,
            "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "traffic": (profiled_traffic(w.name)
                        if len(parts) == 1 and parts[0].w is w and main == "bwd_tensor" else None),
            "kernels": per_kernel,
        },
        "e2e": e2e,
        "gpu_launches": len(trace),
        "clocks": sampler.summary(),
    }
    return result


# ---------------------------------------------------------------- oracle timing
PROJ_SHAPE = dict(B=2, n=4096, d_model=4096, H=32, d=128, dv=128)


def run_proj(args, rank, world, local):
    """attn_proj_bwd at the headline attention shape with d_model = H*d:
    dX = [dQ|dK|dV] [Wq|Wk|Wv]^T and dWq, dWk, dWv = X^T dQ, ... over all
    B*n tokens. Inputs are synthetic bf16 normals, resident in HBM."""
    import scaled_dot_product_saving_b200 as lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c = PROJ_SHAPE
    B, n, d_model, H, d, dv = c["B"], c["n"], c["d_model"], c["H"], c["d"], c["dv"]
    g = torch.Generator().manual_seed(7 + 1000 * rank)

    def r(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).to(dev)
    X = r(B, n, d_model)
    Wq, Wk, Wv = (r(d_model, H * w_, std=d_model ** -0.5) for w_ in (d, d, dv))
    dQ, dK, dV = r(B, H, n, d), r(B, H, n, d), r(B, H, n, dv)
    outs = [torch.empty_like(t) for t in (X, Wq, Wk, Wv)]
    ws = torch.empty(lib.attn_proj_bwd_workspace_size(B, n, d_model, H, d, dv, 1),
                     dtype=torch.uint8, device=dev)
    tokens, wtot = B * n, 2 * H * d + H * dv
    flops = 2.0 * tokens * d_model * wtot * 2      # dX and the three dW, same count each

    def step():
        lib.attn_proj_bwd(X, Wq, Wk, Wv, dQ, dK, dV, workspace=ws, dx=outs[0], dwq=outs[1],
                          dwk=outs[2], dwv=outs[3])
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(world, local)
    torch.cuda.synchronize()
    sampler.start()
    lib.attn_trace_begin(min(65536, 16 * args.steps))
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier(world, local)
    sampler.stop()
    trace = lib.attn_trace_end()
    if lib.attn_get_device_error() != 0:
        raise RuntimeError("device-side timeout in the timed region")
    (slow_ms,) = max_over_ranks([t0.elapsed_time(t1)], world, dev)
    gemm_ms = sum(ms for name, ms in trace if name == "gemm") / args.steps
    gather_ms = sum(ms for name, ms in trace if name == "proj_gather") / args.steps
    peaks, peaks_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (gemm_ms * 1e-3) / 1e12

    # The output projection of Problem 10 at the same shape: dWo = O_cat^T G,
    # dO = G Wo^T sliced into heads.
    O = r(B, H, n, dv)
    Wo = r(H * dv, d_model, std=(H * dv) ** -0.5)
    Gy = r(B, n, d_model)
    o_outs = [torch.empty_like(O), torch.empty_like(Wo)]
    o_ws = torch.empty(lib.attn_outproj_bwd_workspace_size(B, n, d_model, H, dv, 1),
                       dtype=torch.uint8, device=dev)
    o_flops = 2.0 * tokens * d_model * (H * dv) * 2

    def o_step():
        lib.attn_outproj_bwd(O, Wo, Gy, workspace=o_ws, do=o_outs[0], dwo=o_outs[1])
    for _ in range(args.warmup):
        o_step()
    torch.cuda.synchronize()
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lib.attn_trace_begin(min(65536, 8 * args.steps))
    t2.record()
    for _ in range(args.steps):
        o_step()
    t3.record()
    torch.cuda.synchronize()
    o_trace = lib.attn_trace_end()
    if lib.attn_get_device_error() != 0:
        raise RuntimeError("device-side timeout in the output-projection timing")
    (o_ms,) = max_over_ranks([t2.elapsed_time(t3)], world, dev)
    o_gemm_ms = sum(ms for name, ms in o_trace if name == "gemm") / args.steps
    outproj = {
        "value": round(world * args.steps * o_flops / (o_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
        "ms_per_step": round(o_ms / args.steps, 4),
        "kernel_ms": {"gemm": round(o_gemm_ms, 4),
                      "proj_gather": round(sum(ms for nm, ms in o_trace if nm == "proj_gather")
                                           / args.steps, 4)},
        "roofline": {"bound": "tensor", "achieved": round(o_flops / (o_gemm_ms * 1e-3) / 1e12, 3),
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": round(o_flops / (o_gemm_ms * 1e-3) / 1e12 / peak, 4)},
    }
    if rank != 0:
        return None
    return {
        "metric": "attention projection-gradient TFLOP/s (bf16)",
        "value": world * args.steps * flops / (slow_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(slow_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "proj_b2n4096_dmodel4096_h32_d128", **c,
                   "parallelism": "replicas" if world > 1 else "none"},
        "kernel_ms": {"gemm": round(gemm_ms, 4), "proj_gather": round(gather_ms, 4)},
        "roofline": {"bound": "tensor", "kernel": "gemm (4 launches a step)",
                     "achieved": round(achieved, 3), "peak": peak,
                     "peak_source": f"bf16_tflops ({peaks_src}, burst)", "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None},
        "gpu_launches": sum(1 for _ in trace),
        "clocks": sampler.summary(),
        "outproj": outproj,
    }


def oracle_sample(w, seconds, max_heads=None):
    """Time the oracle backward on whole heads of the workload until `seconds`
    have passed. Returns (TFLOP/s in the metric's counting, heads, elapsed)."""
    import oracle.ref as ref
    q, k, v, do = synth.make_inputs(w)
    kl = w.key_len()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    done, flops, t0 = 0, 0.0, time.perf_counter()
    while True:
        b, h = heads[done % len(heads)]
        Q, K, V, dO = (t[b, h].to(torch.float64).numpy() for t in (q, k, v, do))
        ref.head_backward(Q, K, V, dO, causal=w.causal, scale=w.scale,
                          key_len=None if kl is None else kl[b])
        done += 1
        flops += w.head_bwd_flops(b)
        elapsed = time.perf_counter() - t0
        if elapsed >= seconds or (max_heads and done >= max_heads):
            break
    return flops / elapsed / 1e12, done, elapsed


def run_reference(args, w, rank, world):
    if rank != 0:
        return None
    import oracle.ref as ref
    q, k, v, do = synth.make_inputs(w)
    kl = w.key_len()
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]

    def one(i):
        b, h = heads[i % len(heads)]
        Q, K, V, dO = (t[b, h].to(torch.float64).numpy() for t in (q, k, v, do))
        ref.head_backward(Q, K, V, dO, causal=w.causal, scale=w.scale,
                          key_len=None if kl is None else kl[b])
        return w.head_bwd_flops(b)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    flops = sum(one(i) for i in range(args.steps))
    elapsed = time.perf_counter() - t0
    value = flops / elapsed / 1e12
    cores = blas_threads()
    sample = (f"one (batch, head) problem of {w.name} per step "
              f"(n={w.n}, m={w.m}, d={w.d}), float64 oracle backward")
    return {
        "impl": "reference",
        "metric": metric_for(w), "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * elapsed / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "m": w.m, "d": w.d,
                   "dv": w.dv, "causal": w.causal, "scale": w.scale},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    w = synth.workload(args.workload)
    rank, world, local = init_distributed()
    try:
        if args.proj:
            out = run_proj(args, rank, world, local)
        elif args.impl == "reference":
            out = run_reference(args, w, rank, world)
        else:
            out = run_ours(args, w, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                tf, nheads, secs = oracle_sample(w, args.cpu_seconds)
                out["cpu_baseline"] = {
                    "value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                    "sample": f"{nheads} (batch, head) problems of {w.name} through the float64 "
                              f"oracle backward in {secs:.1f} s"}
            elif rank == 0:
                out["cpu_baseline"] = None
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
