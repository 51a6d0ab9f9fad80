#!/usr/bin/env python
"""Throughput of one Split-KV anchor-attention training step on B200.

A step is one pass of the whole path over one batch of synthetic input:
  host plan (mask metadata + LPT) -> plan upload -> chunk partial forward ->
  merge (in-block term + exact LSE combine) -> backward Delta -> chunk partial
  backward (dK, dV local per chunk, dQ partials) -> dQ reduce + in-block backward.

Default workload (N=1): 32 query / 8 KV heads, head_dim 128, a 65536-token
packed context (sample lengths uniform in [2048, 16384]), 512 anchors x 16 =
8192 draft queries, KV chunk 512, bf16 inputs drawn N(0,1), fp32 outputs.

Metric: masked-pair TFLOP/s = (4 + 10) * d * (allowed (query, key, head)
pairs) per step / step time; allowed pairs are counted exactly (context pairs
from the plan plus the in-block pairs).  Timing: CUDA events on the launch
stream, W untimed warm-up steps, barrier + synchronize around K timed steps,
max over ranks.  Every step's inputs and outputs (~4 GB with the workspaces)
exceed the 126 MB L2, so no flush is needed between steps.

With --gpus N > 1 (torchrun, one process per GPU) every rank runs an
independent replica of the workload (the path has no exchange step on one
GPU: replicas only), and the value is the sum of their work over the max time.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "masked-pair attn TFLOP/s fwd/bwd, % of BF16 tensor peak; LPT imbalance %"

# DRAM bytes per launch at the default (64k context / 8k queries) workload and
# schedule (backward LPT by tile cost), from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum, mean of 5 launches), keyed by
# kernel, with the sha256 of the sources the kernel was built from when it was
# taken; a changed source voids the figure.
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch at the 64k / 8k fwd+bwd
    # workload (ncu --clock-control none, one pass), with a hash of the kernel's sources at
    # the capture: a kernel whose sources changed since reports traffic null
    "fwd_partial": {"bytes": 926116864 + 1154541568, "src": "f9c145e1db5443a1"},
    "bwd_dkdv": {"bytes": 1148916992 + 486914048, "src": "981b70cc1d42b122"},
    "bwd_dq": {"bytes": 1159078656 + 1141427968, "src": "981b70cc1d42b122"},
    "merge": {"bytes": 1430378752 + 126864896, "src": "650d9add59a164a1"},
    "bwd_reduce": {"bytes": 1365891072 + 188002560, "src": "650d9add59a164a1"},
    "bwd_delta": {"bytes": 201351424 + 736768, "src": "650d9add59a164a1"},
}
# the workload and schedule the figures were taken on (bench.py's defaults)
NCU_TRAFFIC_CONFIG = {"workload": "bwd", "anchors": None, "schedule": "lpt", "lpt_cost": "tiles",
                      "fwd_lpt_cost": "pairs", "q_slice": 2, "partial_bf16": False, "claims": "run-time"}
_KERNEL_SOURCES = {
    "fwd_partial": ("fwd_partial_sm100.cu", "sm100.cuh", "splitkv_internal.h"),
    "bwd_dkdv": ("bwd_partial_sm100.cu", "sm100.cuh", "splitkv_internal.h"),
    "bwd_dq": ("bwd_partial_sm100.cu", "sm100.cuh", "splitkv_internal.h"),
}


def _src_hash(kernel: str) -> str:
    m = hashlib.sha256()
    for name in _KERNEL_SOURCES.get(kernel, ("merge.cu", "common.cuh", "splitkv_internal.h")):
        with open(os.path.join(ROOT, "context_block_sparse_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    return m.hexdigest()[:16]


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clock, power and clock-event reasons sampled while the timed region runs.

    NVML (read-only queries) polled every 2 ms from a thread, so that a timed region
    of a few tens of milliseconds still gets samples; nvidia-smi at 100 ms when NVML
    cannot be opened."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.rows = []          # (time, sm_mhz, max_mhz, {reason names})
        self.proc = None
        self.t = None
        self.stop_flag = False
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
        except Exception:
            return self._start_smi()
        self.source = "nvml"

        def poll():
            while not self.stop_flag:
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    break
                self.rows.append((time.time(), float(sm), float(mx),
                                  {n for n, b in zip(self.NAMES, bits) if rs & b}))
                time.sleep(0.002)

        self.t = threading.Thread(target=poll, daemon=True)
        self.t.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        def read():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 7:
                    self.rows.append((time.time(), num(parts[0]), num(parts[1]),
                                      {n for n, v in zip(self.NAMES, parts[3:]) if v.lower() == "active"}))

        self.t = threading.Thread(target=read, daemon=True)
        self.t.start()

    def stop(self):
        self.stop_flag = True
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=1.0)

    def summary(self, t0: float, t1: float):
        rows = [r for r in self.rows if t0 <= r[0] <= t1] or [r for r in self.rows if t0 - 0.15 <= r[0] <= t1 + 0.15]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [r[1] for r in rows if r[1] is not None]
        mx = [r[2] for r in rows if r[2] is not None]
        reasons = sorted(set().union(*[r[3] for r in rows]))
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": self.source}


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: every rank of an N-GPU run reports the max (all-reduce MAX)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    x = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return float(x.item())


def whole_job_tflops(world: int, steps: int, flops_per_step: float, max_ms: float) -> float:
    """Work of all ranks (each runs one replica) over the slowest rank's time, in TFLOP/s."""
    return world * steps * flops_per_step / (max_ms * 1e-3) / 1e12


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def _kernel_work(st, w, E, rec_bytes=4.0):
    """Algorithmic FLOPs or bytes of one launch of each kernel; rec_bytes: bytes of one
    O_c / dQ-partial element (4, or 2 with bf16 partial records)."""
    d, Hq, Hkv, bs, Nq = w.head_dim, w.num_q_heads, w.num_kv_heads, w.block_size, w.num_queries
    ctx = st["context_pairs"]
    rec_rows = E * bs * Hq
    return {
        "fwd_partial": ("tensor", 4.0 * d * ctx),
        # the backward partial step is two kernels that each recompute S and dP:
        # dK/dV kernel S, dP, dV, dK = 8d per allowed pair; dQ kernel S, dP, dQ = 6d
        "bwd_dkdv": ("tensor", 8.0 * d * ctx),
        "bwd_dq": ("tensor", 6.0 * d * ctx),
        # partial records (O_c, m, l) read; o, lse written; q, kb, vb read once
        "merge": ("hbm", rec_rows * (rec_bytes * d + 8) + Nq * Hq * (4.0 * d + 4) + Nq * Hq * d * 2.0
                  + 2.0 * Nq * Hkv * d * 2),
        # o (fp32) and dout read, Delta written
        "bwd_delta": ("hbm", Nq * Hq * d * (4.0 + 2.0) + Nq * Hq * 4.0),
        # dq partials read; q, dout, kb, vb, lse, Delta read; dq, dkb, dvb written
        "bwd_reduce": ("hbm", rec_rows * d * rec_bytes + Nq * Hq * (d * 4.0 + 8) + Nq * Hq * d * 4.0
                       + 2.0 * Nq * Hkv * d * 2 + 2.0 * Nq * Hkv * d * 4),
    }


def _bwd_is_two_launches(w) -> bool:
    return (w.head_dim == 128 and (w.num_q_heads // w.num_kv_heads * w.block_size) % 8 == 0
            and os.environ.get("SPLITKV_BWD_KERNEL") != "mma")


def bench_config(args, w, W, Wb, world):
    """The workload and launch options of a bench line (both arms report the same)."""
    return {"workload": w.config.description, "context_len": w.context_len, "num_queries": w.num_queries,
            "num_anchors": int(w.anchors.size), "block_size": w.block_size, "heads": [w.num_q_heads, w.num_kv_heads],
            "head_dim": w.head_dim, "kv_chunk": w.kv_chunk, "fwd_workers": W, "bwd_workers": Wb,
            "seed": args.seed if args.seed is not None else 1000 + w.config.index,
            "q_slice": args.q_slice, "partial_records": "bf16" if args.partial_bf16 else "f32",
            "lpt_cost": args.lpt_cost, "fwd_lpt_cost": args.fwd_lpt_cost,
            "schedule": args.schedule, "item_claims": "run-time" if args.dynamic_claim else "static",
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "no flush: each step touches ~4 GB (> 126 MB L2)"}


def _workers(args):
    """Forward and backward CTA counts: the options, else the SM count of the GPU (None without one)."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else None
    return args.workers or sms, args.bwd_workers or sms


def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist

    import context_block_sparse_b200 as skv
    from synth import make_workload

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    w = make_workload(args.workload, num_anchors=args.anchors, seed=args.seed, with_grad=True)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    W = args.workers or sms
    Wb = args.bwd_workers or sms
    stream = torch.cuda.current_stream(dev)

    def up(name):
        return torch.from_numpy(w.bits[name].view(np.int16)).view(torch.bfloat16).to(dev)

    t = {n: up(n) for n in ("q", "k", "v", "kb", "vb", "dout")}
    d, Hq, Nq = w.head_dim, w.num_q_heads, w.num_queries
    plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, Hq, w.num_kv_heads, d, w.kv_chunk, W,
                            num_bwd_workers=Wb, q_slice=args.q_slice, partial_bf16=args.partial_bf16,
                            tile_cost=args.lpt_cost == "tiles", fwd_tile_cost=args.fwd_lpt_cost == "tiles",
                            dynamic_claim=args.dynamic_claim, contiguous_schedule=args.schedule == "contiguous")
    plan.upload(stream)
    st = plan.stats()
    if args.dump_plan and rank == 0:
        plan.dump(args.dump_plan)
    ws_f = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_BWD), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    o = torch.empty((Nq, Hq, d), **f32)
    lse = torch.empty((Nq, Hq), **f32)
    g = {"dq": torch.empty(t["q"].shape, **f32), "dk": torch.empty(t["k"].shape, **f32),
         "dv": torch.empty(t["v"].shape, **f32), "dkb": torch.empty(t["kb"].shape, **f32),
         "dvb": torch.empty(t["vb"].shape, **f32)}
    kernels = ["fwd_partial", "merge", "bwd_delta", "bwd_dkdv", "bwd_dq", "bwd_reduce"]
    plan_us = []

    def step(ev=None):
        skv.splitkv_plan_update(plan, w.sample_lens, w.anchors)
        plan_us.append(plan.stats()["plan_us"])
        plan.upload(stream)
        if ev is not None:
            ev[0].record(stream)
        skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws_f, stream)
        if ev is not None:
            ev[1].record(stream)
        skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], w.scale, ws_f, o, lse, stream)
        if ev is not None:
            ev[2].record(stream)
        skv.splitkv_bwd_delta(plan, o, t["dout"], ws_b, stream)
        if ev is not None:
            ev[3].record(stream)
        skv.splitkv_bwd_dkdv(plan, t["q"], t["k"], t["v"], lse, t["dout"], g["dk"], g["dv"], w.scale, ws_b, stream)
        if ev is not None:
            ev[4].record(stream)
        skv.splitkv_bwd_dq(plan, t["q"], t["k"], t["v"], lse, t["dout"], w.scale, ws_b, stream)
        if ev is not None:
            ev[5].record(stream)
        skv.splitkv_bwd_reduce(plan, t["q"], t["kb"], t["vb"], lse, t["dout"], g["dq"], g["dkb"], g["dvb"],
                               w.scale, ws_b, stream)
        if ev is not None:
            ev[6].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    sampler = None
    if rank == 0 and not args.no_clocks:
        props = torch.cuda.get_device_properties(dev)
        sampler = ClockSampler("GPU-" + str(props.uuid))
        sampler.start()
        time.sleep(0.3)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(kernels) + 1)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    plan_us.clear()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(start.elapsed_time(end), dev)
    per_kernel = {k: float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)]))
                  for j, k in enumerate(kernels)}
    clocks = sampler.summary(wall0, wall1) if sampler else {"sm_mhz": None, "sm_max_mhz": None,
                                                              "reasons": ["unsampled"]}
    if sampler:
        sampler.stop()

    # measured per-CTA busy time of the last step (untimed read)
    cta_f = skv.splitkv_read_cta_times(plan, skv.WS_FWD, stream)
    cta_b = skv.splitkv_read_cta_times(plan, skv.WS_BWD, stream)
    cta_q = skv.splitkv_read_cta_times(plan, skv.TIMES_DQ, stream) if _bwd_is_two_launches(w) else None

    def imb(x):
        x = np.asarray(x, dtype=np.float64)
        return float(x.max() / x.mean() - 1.0) if x.size and x.mean() > 0 else 0.0

    if args.dump_cta_times and rank == 0:
        with open(args.dump_cta_times, "w") as f:
            json.dump({"workload": args.workload, "anchors": int(w.anchors.size), "q_slice": args.q_slice,
                       "lpt_cost": args.lpt_cost, "fwd_lpt_cost": args.fwd_lpt_cost,
                       "dynamic_claim": bool(args.dynamic_claim), "partial_bf16": bool(args.partial_bf16),
                       "schedule": args.schedule,
                       "fwd_workers": W, "bwd_workers": Wb,
                       "fwd_ns": [int(x) for x in cta_f], "bwd_ns": [int(x) for x in cta_b],
                       "dq_ns": None if cta_q is None else [int(x) for x in cta_q]}, f)

    pairs = st["context_pairs"] + st["block_pairs"]
    flops_fwd = 4.0 * d * pairs
    flops_bwd = 10.0 * d * pairs
    flops_step = flops_fwd + flops_bwd
    value = whole_job_tflops(world, args.steps, flops_step, ms)
    peaks = _peaks()
    work = _kernel_work(st, w, st["num_entries"], 2.0 if args.partial_bf16 else 4.0)
    dom = max(kernels, key=lambda k: per_kernel[k])
    bound, amount = work[dom]
    dom_s = per_kernel[dom] * 1e-3
    tr = NCU_TRAFFIC.get(dom)
    same_config = all(getattr(args, k) == v for k, v in NCU_TRAFFIC_CONFIG.items())
    traffic = tr["bytes"] if tr and same_config and tr.get("src") == _src_hash(dom) else None
    if bound == "tensor":
        achieved = amount / dom_s / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 (burst)", "launch_ms": per_kernel[dom]}
    else:
        achieved = amount / dom_s / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{peaks['source']} copy", "launch_ms": per_kernel[dom]}
    kern = {}
    for k in kernels:
        b_, a_ = work[k]
        s_ = max(per_kernel[k] * 1e-3, 1e-9)
        rate = a_ / s_ / 1e12 if b_ == "tensor" else a_ / s_ / 1e9
        kern[k] = {"ms": per_kernel[k], ("tflops" if b_ == "tensor" else "gbs"): rate,
                   "frac": rate / (peaks["bf16_tflops"] if b_ == "tensor" else peaks["hbm_gbs"])}
    fwd_ms = per_kernel["fwd_partial"] + per_kernel["merge"]
    bwd_ms = sum(per_kernel[k] for k in ("bwd_delta", "bwd_dkdv", "bwd_dq", "bwd_reduce"))

    result = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(args, w, W, Wb, world),
        "fwd_tflops": flops_fwd / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": flops_bwd / (bwd_ms * 1e-3) / 1e12,
        "pct_of_bf16_peak": 100.0 * value / world / peaks["bf16_tflops"],
        "lpt_imbalance_pct": {"fwd_plan": 100 * st["fwd_imbalance"], "bwd_plan": 100 * st["bwd_imbalance"],
                              "contiguous_plan": 100 * st["contig_imbalance"], "fwd_measured": 100 * imb(cta_f),
                              "bwd_measured": 100 * imb(cta_b),
                              "dq_measured": None if cta_q is None else 100 * imb(cta_q)},
        "plan_us": float(np.median(plan_us)) if plan_us else None,
        "kernels": kern,
        "roofline": roof,
        # the dQ kernel is a separate launch on the tcgen05 path (head_dim 128, G * bs a
        # multiple of 8); on the mma.sync path the dK/dV launch also writes dQ and the
        # dQ call launches nothing
        "gpu_launches": (len(kernels) - (0 if _bwd_is_two_launches(w) else 1)) * args.steps,
        "clocks": clocks,
    }

    if rank == 0:
        result["device_lpt"] = device_lpt_report(skv, w)
    if rank == 0 and world == 1 and args.emulate_ranks > 1:
        lpt = rank_emulation_report(skv, w, args, args.emulate_ranks, dev, stream, t, W, Wb, peaks)
        con = rank_emulation_report(skv, w, args, args.emulate_ranks, dev, stream, t, W, Wb, peaks,
                                    contiguous=True)
        step = lambda r: max(f + b for f, b in zip(r["fwd_ms"], r["bwd_ms"]))   # noqa: E731
        result["split_kv_ranks"] = {"lpt_ownership": lpt, "contiguous_ownership": con,
                                    "step_ms_contiguous_over_lpt": step(con) / step(lpt)}
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, w, plan, dev, stream, flops_step, world=world, out_bf16=True)
        e32 = run_e2e(args, w, plan, dev, stream, flops_step, world=world, out_bf16=False)
        result["e2e"]["f32_outputs"] = {k: e32[k] for k in ("value", "ms_per_step", "d2h_bytes_per_step")}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        def gpu_rows(rows):
            idx = torch.as_tensor(rows, device=dev)
            return {n: x.index_select(0, idx).double().cpu().numpy()
                    for n, x in (("o", o), ("lse", lse), ("dq", g["dq"]), ("dkb", g["dkb"]), ("dvb", g["dvb"]))}

        def gpu_keys(keys):
            idx = torch.as_tensor(keys, device=dev)
            return {n: g[n].index_select(0, idx).double().cpu().numpy() for n in ("dk", "dv")}

        result["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds, gpu_rows=gpu_rows,
                                              gpu_keys=gpu_keys)
    if world > 1:
        dist.destroy_process_group()
    return result if rank == 0 else None


def device_lpt_report(skv, w, workers=(8, 16, 32, 64)):
    """The planner in the pages' device regime (news page, "Balance actual attention
    work": W devices, equal chunk counts, against leaving chunks unbalanced), on the
    host, untimed: for each W, plan latency and max/mean load imbalance of plain LPT,
    equal-count LPT and the contiguous assignment, over whole (chunk, KV head) items;
    `makespan_ratio` = (1 + contiguous) / (1 + equal-count LPT), the step-time ratio the
    imbalance alone implies."""
    out = {}
    for W in workers:
        row = {}
        for mode, eq in (("lpt", False), ("equal_count", True)):
            plan = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.kv_chunk, W, num_bwd_workers=W, q_slice=0, equal_count=eq)
            st = plan.stats()
            row[f"{mode}_imbalance_pct"] = 100 * st["fwd_imbalance"]
            row[f"{mode}_plan_us"] = st["plan_us"]
            row["contiguous_imbalance_pct"] = 100 * st["contig_imbalance"]
            plan.destroy()
        row["makespan_ratio"] = (1 + row["contiguous_imbalance_pct"] / 100) / (1 + row["equal_count_imbalance_pct"] / 100)
        out[str(W)] = row
    return out


def run_split_kv(args, world, rank, local):
    """Split-KV over the torchrun ranks (one GPU each): the whole workload split by chunk
    ownership, a step = SplitKVContextParallel forward + backward (query-side broadcasts,
    local kernels, all-to-all of result rows, combine, dq sum); every rank's K, V hold the
    whole context (only its chunks are read).  Timed like the main arm: CUDA events on the
    launch stream between barriers, max over ranks; `value` = the whole problem's FLOPs per
    second (total work fixed as N grows: strong scaling)."""
    import datetime

    import torch
    import torch.distributed as dist

    from context_block_sparse_b200.context_parallel import SplitKVContextParallel
    from synth import make_workload

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if "MASTER_ADDR" not in os.environ:      # run without torchrun: a one-rank group
        import socket
        s = socket.socket()
        s.bind(("127.0.0.1", 0))
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(s.getsockname()[1]), RANK="0", WORLD_SIZE="1")
        s.close()
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    try:
        w = make_workload(args.workload, num_anchors=args.anchors, seed=args.seed, with_grad=True)
        W, Wb = _workers(args)
        W = W or torch.cuda.get_device_properties(dev).multi_processor_count
        Wb = Wb or W
        cp = SplitKVContextParallel(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.kv_chunk, num_workers=W, num_bwd_workers=Wb, q_slice=args.q_slice,
                                    tile_cost=args.lpt_cost == "tiles", dynamic_claim=args.dynamic_claim,
                                    partial_bf16=args.partial_bf16, contiguous_ranks=args.schedule == "contiguous",
                                    exchange=args.exchange)
        up = lambda n: torch.from_numpy(w.bits[n].view(np.int16)).view(torch.bfloat16).to(dev)   # noqa: E731
        t = {n: up(n) for n in ("q", "k", "v", "kb", "vb", "dout")}
        rows = cp.rows
        q, kb, vb, dout = (t[n][rows].contiguous() for n in ("q", "kb", "vb", "dout"))
        stream = torch.cuda.current_stream(dev)

        def step():
            o, lse = cp.forward(q, t["k"], t["v"], kb, vb, w.scale)
            cp.backward(t["k"], t["v"], o, lse, dout, w.scale)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        ms = max_over_ranks(a.elapsed_time(b), dev)
        full = skv_plan_stats_of(w, W)
        flops_step = 14.0 * w.head_dim * (full["context_pairs"] + full["block_pairs"])
        res = {"metric": METRIC, "value": flops_step * args.steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
               "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic", "impl": "split-kv",
               "config": {**bench_config(args, w, W, Wb, world), "parallelism": f"split-kv over {world} ranks",
                          "chunk_ownership": "contiguous" if args.schedule == "contiguous" else "lpt",
                          "exchange": args.exchange}}
        return res if rank == 0 else None
    finally:
        dist.destroy_process_group()


def skv_plan_stats_of(w, W):
    """Pair counts of the whole (unsplit) problem, from a host-only plan."""
    import context_block_sparse_b200 as skv
    p = skv.splitkv_plan(w.sample_lens, w.anchors, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                         w.kv_chunk, W)
    st = p.stats()
    p.destroy()
    return st


def rank_emulation_report(skv, w, args, R, dev, stream, t, W, Wb, peaks, reps=5, contiguous=False):
    """Split-KV over R ranks with one GPU standing in for each rank in turn (after the timed
    region, untimed by the bench line): per rank, the device time of its forward
    (splitkv_attn_fwd + splitkv_merge) and backward (splitkv_attn_bwd) on its rank plan, the
    median of `reps`; the measured rank imbalance (max / mean - 1 of forward + backward)
    against the planned one (the ranks' summed chunk costs, news page "Balance actual
    attention work"); and the combine / sum kernels of the exchange against the HBM peak.
    The collectives themselves are not timed (one GPU).  contiguous: chunks owned in order
    (the pages' unbalanced device baseline) instead of by LPT."""
    import torch
    f32 = dict(dtype=torch.float32, device=dev)
    d, Hq, Hkv, Nq, N = w.head_dim, w.num_q_heads, w.num_kv_heads, w.num_queries, w.context_len
    kw = dict(num_bwd_workers=Wb, q_slice=args.q_slice, partial_bf16=args.partial_bf16,
              tile_cost=args.lpt_cost == "tiles", dynamic_claim=args.dynamic_claim, contiguous_ranks=contiguous)
    args_p = (w.sample_lens, w.anchors, w.block_size, Hq, Hkv, d, w.kv_chunk, W)
    o_parts = torch.empty((R, Nq, Hq, d), **f32)
    lse_parts = torch.empty((R, Nq, Hq), **f32)
    dq_parts = torch.empty((R, Nq, Hq, d), **f32)
    dk, dv = torch.zeros(t["k"].shape, **f32), torch.zeros(t["v"].shape, **f32)
    dkb, dvb = torch.zeros(t["kb"].shape, **f32), torch.zeros(t["vb"].shape, **f32)
    o = torch.empty((Nq, Hq, d), **f32)
    lse = torch.empty((Nq, Hq), **f32)

    def timed(fn):
        out = []
        for _ in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            out.append(a.elapsed_time(b))
        return float(np.median(out[1:]))

    fwd_ms, bwd_ms, loads = [], [], []
    full = skv.splitkv_plan(*args_p, **kw)
    full_pairs = full.export(skv.EXPORT_CHUNK_PAIRS)
    full.destroy()
    plans = []
    for r in range(R):
        plan = skv.splitkv_plan_shard(*args_p, R, r, **kw).upload(stream)
        owner = plan.export(skv.EXPORT_CHUNK_OWNER)
        loads.append(int(Hq * full_pairs[owner == r].sum()))
        ws_f = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_FWD), dtype=torch.uint8, device=dev)
        ws_b = torch.empty(skv.splitkv_workspace_size(plan, skv.WS_BWD), dtype=torch.uint8, device=dev)
        plans.append((plan, ws_f, ws_b))

        def fwd(plan=plan, ws_f=ws_f, r=r):
            skv.splitkv_attn_fwd(plan, t["q"], t["k"], t["v"], w.scale, ws_f, stream)
            skv.splitkv_merge(plan, t["q"], t["kb"], t["vb"], w.scale, ws_f, o_parts[r], lse_parts[r], stream)

        fwd_ms.append(timed(fwd))
    # the backward of every rank runs with the combined o, lse
    skv.splitkv_combine_ranks(o_parts, lse_parts, o, lse, stream)
    for r, (plan, ws_f, ws_b) in enumerate(plans):
        def bwd(plan=plan, ws_b=ws_b, r=r):
            skv.splitkv_attn_bwd(plan, t["q"], t["k"], t["v"], t["kb"], t["vb"], o, lse, t["dout"], dq_parts[r],
                                 dk, dv, dkb, dvb, w.scale, ws_b, stream)

        bwd_ms.append(timed(bwd))
        skv.splitkv_plan_status(plan, stream)
    for plan, _, _ in plans:
        plan.destroy()
    plans.clear()
    comb_ms = timed(lambda: skv.splitkv_combine_ranks(o_parts, lse_parts, o, lse, stream))
    dq = torch.empty((Nq, Hq, d), **f32)
    sum_ms = timed(lambda: skv.splitkv_sum_ranks(dq_parts, dq, stream))
    rows = Nq * Hq
    comb_bytes = (R + 1) * rows * (4 * d + 4)
    sum_bytes = 4 * (R + 1) * rows * d
    step = [f + b for f, b in zip(fwd_ms, bwd_ms)]

    def imb(x):
        x = np.asarray(x, dtype=np.float64)
        return float(x.max() / x.mean() - 1.0) if x.size and x.mean() > 0 else 0.0

    return {
        "ranks": R,
        "planned_loads": loads,
        "planned_imbalance_pct": 100 * imb(loads),
        "fwd_ms": fwd_ms,
        "bwd_ms": bwd_ms,
        "measured_imbalance_pct": 100 * imb(step),
        "combine": {"ms": comb_ms, "gbs": comb_bytes / (comb_ms * 1e-3) / 1e9,
                    "frac": comb_bytes / (comb_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "rows": rows},
        "sum": {"ms": sum_ms, "gbs": sum_bytes / (sum_ms * 1e-3) / 1e9,
                "frac": sum_bytes / (sum_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "note": "one GPU runs each rank plan in turn; combine / sum timed over all query rows at once",
    }


def run_e2e(args, w, plan, dev, stream, flops_step, world=1, out_bf16=True):
    """Same metric through the public API from pinned HOST buffers: every step copies its inputs in and
    its results (o, lse, dq, dk, dv, dkb, dvb) out inside the timed region, the copies overlapping the
    computation of the neighbouring steps (two device buffer sets, one stream per copy direction).
    out_bf16: o and the gradients come back as bf16 (the kernels accumulate in fp32; o is stored as
    bf16 by the merge, the gradients rounded on the GPU by splitkv_cast_bf16), lse as fp32."""
    import torch
    import torch.distributed as dist

    import context_block_sparse_b200 as skv
    from context_block_sparse_b200.torch_api import SplitKVAttention

    host = {n: torch.from_numpy(w.bits[n].view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "kb", "vb", "dout")}
    d, Hq, Nq = w.head_dim, w.num_q_heads, w.num_queries
    att = SplitKVAttention(w.sample_lens, w.anchors, w.block_size, Hq, w.num_kv_heads, d, w.kv_chunk,
                           num_workers=plan.problem.num_workers, num_bwd_workers=plan.problem.num_bwd_workers,
                           q_slice=plan.problem.q_slice, device=dev, partial_bf16=args.partial_bf16,
                           tile_cost=args.lpt_cost == "tiles", fwd_tile_cost=args.fwd_lpt_cost == "tiles",
                           dynamic_claim=args.dynamic_claim, contiguous_schedule=args.schedule == "contiguous")
    # two device sets of inputs and outputs, so that the next step's inputs go up and the
    # last step's results come down while a step computes; uploads and downloads on copy
    # streams of their own (the two PCIe directions run at once)
    dvs = [{n: torch.empty(x.shape, dtype=x.dtype, device=dev) for n, x in host.items()} for _ in range(2)]
    f32 = dict(dtype=torch.float32, device=dev)
    odt = torch.bfloat16 if out_bf16 else torch.float32
    outs_d = [{"o": torch.empty((Nq, Hq, d), dtype=odt, device=dev), "lse": torch.empty((Nq, Hq), **f32),
               **{"d" + n: torch.empty(host[n].shape, dtype=odt, device=dev) for n in ("q", "k", "v", "kb", "vb")}}
              for _ in range(2)]
    outs_h = {n: torch.empty(x.shape, dtype=x.dtype).pin_memory() for n, x in outs_d[0].items()}
    h2d = sum(x.numel() * x.element_size() for x in host.values()) + 4 * (w.sample_lens.size + w.anchors.size)
    d2h = sum(x.numel() * x.element_size() for x in outs_h.values())
    steps = max(1, min(args.steps, args.e2e_steps))
    up_s = torch.cuda.Stream(dev)
    down_s = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()   # noqa: E731
    computed = [None, None]   # per set: the step's kernels are done (its inputs and outputs are free)
    downloaded = [None, None]  # per set: its outputs have reached the host

    def step(k):
        b = k % 2
        x, y = dvs[b], outs_d[b]
        # inputs: after the kernels of step k - 2 have read this set
        if computed[b] is not None:
            up_s.wait_event(computed[b])
        with torch.cuda.stream(up_s):
            for n in host:
                x[n].copy_(host[n], non_blocking=True)
        uploaded = ev()
        uploaded.record(up_s)
        # compute: after the inputs landed and step k - 2's results left this set
        stream.wait_event(uploaded)
        if downloaded[b] is not None:
            stream.wait_event(downloaded[b])
        skv.splitkv_plan_update(att.plan, w.sample_lens, w.anchors)
        att.plan.upload(stream)
        o, lse = att.forward(x["q"], x["k"], x["v"], x["kb"], x["vb"], w.scale, o=y["o"], lse=y["lse"])
        att.backward(x["q"], x["k"], x["v"], x["kb"], x["vb"], o, lse, x["dout"], w.scale,
                     grads={n: y[n] for n in ("dq", "dk", "dv", "dkb", "dvb")}, grad_dtype=odt)
        computed[b] = ev()
        computed[b].record(stream)
        # results: down while the next step computes
        down_s.wait_event(computed[b])
        with torch.cuda.stream(down_s):
            for n, t in y.items():
                outs_h[n].copy_(t, non_blocking=True)
        downloaded[b] = ev()
        downloaded[b].record(down_s)

    for k in range(2):
        step(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    bev = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up_s.wait_event(a)      # the first upload of the timed steps starts after the start mark
    down_s.wait_event(a)
    for k in range(2, 2 + steps):
        step(k)
    stream.wait_event(downloaded[(1 + steps) % 2])   # the last results are on the host
    stream.wait_event(downloaded[steps % 2])
    bev.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(bev), dev)
    if world > 1:
        dist.barrier()
    return {"value": whole_job_tflops(world, steps, flops_step, ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms / steps,
            "outputs": ("bf16 o, dq, dk, dv, dkb, dvb (fp32 accumulation, rounded on the GPU); fp32 lse"
                        if out_bf16 else "fp32 o, lse, dq, dk, dv, dkb, dvb")}


# ---------------------------------------------------------------------------
# the fp64 CPU oracle, timed on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_blocks(w, budget_s: float, start: int = 0, stride: int = 37, keep=None):
    """Run the oracle forward + backward block by block until budget_s elapses; returns (flops, seconds, n).
    keep: a list that receives (block, O, LSE, dq, dkb, dvb) of every block's rows."""
    from oracle import attention as oatt
    from oracle import mask as omask
    f = {n: w.f64(n) for n in ("q", "k", "v", "kb", "vb", "dout")}
    iv = omask.context_interval(w.sample_lens, w.anchors)
    A = len(iv)
    flops = 0.0
    n = 0
    t0 = time.perf_counter()
    b = start % A
    while True:
        O, L = oatt.attention_fwd(f["q"], f["k"], f["v"], f["kb"], f["vb"], w.sample_lens, w.anchors,
                                  w.block_size, w.scale, blocks=[b])
        g = oatt.attention_bwd(f["q"], f["k"], f["v"], f["kb"], f["vb"], f["dout"], w.sample_lens, w.anchors,
                               w.block_size, w.scale, blocks=[b])
        if keep is not None:
            r = slice(b * w.block_size, (b + 1) * w.block_size)
            # copies: views would keep the oracle's full-size arrays of every block alive
            keep.append((b, O[r].copy(), L[r].copy(), g["dq"][r].copy(), g["dkb"][r].copy(), g["dvb"][r].copy()))
        S, a = iv[b]
        flops += 14.0 * w.head_dim * w.num_q_heads * w.block_size * ((a - S) + w.block_size)
        n += 1
        b = (b + stride) % A
        if time.perf_counter() - t0 >= budget_s:
            break
    return flops, time.perf_counter() - t0, n


def parity_chunks(w):
    """KV chunks whose dK, dV the oracle checks at full size, with the blocks that read them:
    the last chunk of the first and of a middle sample (few readers each) and the first chunk
    of the shortest sample (read by every block of that sample, so its gradient sums many
    blocks).  Returns (chunks, reader blocks, key positions)."""
    from oracle import mask as omask
    C = w.kv_chunk
    starts = list(omask.sample_starts(w.sample_lens)) + [w.context_len]

    def last_inside(s):     # the last chunk inside sample s (else the one holding its last key)
        c = starts[s + 1] // C - 1
        return c if c * C >= starts[s] else (starts[s + 1] - 1) // C

    def first_inside(s):    # the first chunk inside sample s (else the one holding its first key)
        c = -(-starts[s] // C)
        return c if (c + 1) * C <= starts[s + 1] else starts[s] // C

    mid = len(w.sample_lens) // 2
    short = int(np.argmin(w.sample_lens))
    chunks = sorted({last_inside(0), last_inside(mid), first_inside(short)})
    iv = omask.context_interval(w.sample_lens, w.anchors)
    readers = [b for b, (S, a) in enumerate(iv) if any(S < (c + 1) * C and a > c * C for c in chunks)]
    keys = np.concatenate([np.arange(c * C, min((c + 1) * C, w.context_len)) for c in chunks])
    return chunks, readers, keys


def _dkdv_parity(w, gpu_keys):
    """The GPU's dK, dV on the keys of parity_chunks(w) against the oracle's, which sums
    the backward of every block that reads them (untimed)."""
    from oracle import attention as oatt
    chunks, readers, keys = parity_chunks(w)
    f = {n: w.f64(n) for n in ("q", "k", "v", "kb", "vb", "dout")}
    g = oatt.attention_bwd(f["q"], f["k"], f["v"], f["kb"], f["vb"], f["dout"], w.sample_lens, w.anchors,
                           w.block_size, w.scale, blocks=readers)
    got = gpu_keys(keys)
    err = {n: float(np.abs(got[n] - g[n][keys]).max()) for n in ("dk", "dv")}
    ref = {n: float(np.abs(g[n][keys]).max()) for n in ("dk", "dv")}
    return {"chunks": [int(c) for c in chunks], "reader_blocks": len(readers), "keys": int(keys.size),
            "max_abs": err, "max_abs_over_max_oracle": {n: err[n] / ref[n] if ref[n] else 0.0 for n in err},
            "tolerance": {"dk": 2e-2, "dv": 2e-2}}


def cpu_baseline(w, budget_s=15.0, gpu_rows=None, gpu_keys=None):
    """The oracle timed on a bounded sample of the workload; with gpu_rows (rows -> the GPU's
    o, lse, dq, dkb, dvb on those query rows) also the GPU's error on the sampled blocks, and
    with gpu_keys (key positions -> the GPU's dk, dv there) its dK, dV error on the keys of a
    few chunks (parity_chunks)."""
    keep = [] if gpu_rows is not None else None
    flops, secs, n = _oracle_blocks(w, budget_s, keep=keep)
    out = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
           "sample": f"fp64 numpy oracle, forward + backward of {n} of {w.anchors.size} anchor blocks "
                     f"(every 37th, all {w.num_q_heads} heads), {secs:.1f} s; same masked-pair FLOP count",
           "host_cpu_count": os.cpu_count()}
    if keep:
        try:
            err = {n: 0.0 for n in ("o", "lse", "dq", "dkb", "dvb")}
            ref = dict(err)
            for b, *want in keep:
                got = gpu_rows(np.arange(b * w.block_size, (b + 1) * w.block_size))
                for name, x in zip(("o", "lse", "dq", "dkb", "dvb"), want):
                    err[name] = max(err[name], float(np.abs(got[name] - x).max()))
                    ref[name] = max(ref[name], float(np.abs(x).max()))
            out["parity_sample"] = {
                "blocks": len(keep), "max_abs": err,
                "max_abs_over_max_oracle": {k: err[k] / ref[k] if ref[k] else 0.0 for k in err},
                "tolerance": {"o": 2e-2, "dq": 2e-2, "dkb": 2e-2, "dvb": 2e-2, "lse": 1e-3},
                "what": "the last timed step's outputs against the fp64 oracle on the sampled blocks' rows"}
        except Exception as e:      # a report, never a reason to lose the bench line
            out["parity_sample"] = {"error": f"{type(e).__name__}: {e}"}
    if gpu_keys is not None and "parity_sample" in out:
        try:
            out["parity_sample"]["dkdv"] = _dkdv_parity(w, gpu_keys)
        except Exception as e:      # a report, never a reason to lose the bench line
            out["parity_sample"]["dkdv"] = {"error": f"{type(e).__name__}: {e}"}
    # the same oracle on one thread, on a shorter sample
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            f1, s1, n1 = _oracle_blocks(w, max(1.0, budget_s / 3), start=500)
        out["value_one_thread"] = f1 / s1 / 1e12
        out["sample_one_thread"] = f"{n1} anchor blocks, {s1:.1f} s, 1 BLAS thread"
    except ImportError:
        pass
    return out


def run_reference(args, world, rank):
    from synth import make_workload
    if rank != 0:
        return None
    w = make_workload(args.workload, num_anchors=args.anchors, seed=args.seed, with_grad=True)
    per_step = max(0.2, min(args.cpu_seconds, 120.0) / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        _oracle_blocks(w, per_step, start=i)
    flops = secs = 0.0
    n = 0
    for i in range(args.steps):
        f_, s_, n_ = _oracle_blocks(w, per_step, start=1000 + 7 * i)
        flops += f_
        secs += s_
        n += n_
    value = flops / secs / 1e12
    sample = (f"fp64 numpy oracle, forward + backward of {n} anchor blocks over {args.steps} steps "
              f"(about {per_step:.1f} s each) of the {args.workload} workload")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": bench_config(args, w, *_workers(args), world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="bwd", choices=["tiny", "drafter", "budget", "skew", "bwd"])
    ap.add_argument("--anchors", type=int, default=None)
    ap.add_argument("--seed", type=int, default=None,
                    help="input seed of the workload (default: the workload's own, 1000 + its index)")
    ap.add_argument("--workers", type=int, default=0, help="forward CTAs (default: SM count)")
    ap.add_argument("--bwd-workers", type=int, default=0, help="backward CTAs (default: SM count)")
    ap.add_argument("--q-slice", type=int, default=2,
                    help="forward items of at most this many 128-row query tiles (0 = whole chunks)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--lpt-cost", choices=["tiles", "pairs"], default="tiles",
                    help="LPT item cost of the backward (dK/dV) schedule: executed tile work (default) or "
                         "the allowed pairs of the pages' rule")
    ap.add_argument("--fwd-lpt-cost", choices=["tiles", "pairs"], default="pairs",
                    help="LPT item cost of the forward schedule (forward and dQ kernels): the allowed pairs "
                         "of the pages' rule (default) or the forward kernel's executed tile work")
    ap.add_argument("--claims", choices=["run-time", "static"], default="run-time",
                    help="how the CTAs of the partial kernels take their items: one at a time in LPT order at "
                         "run time (default; plan flag) or from the static LPT worker lists")
    ap.add_argument("--dump-cta-times", default=None, metavar="PATH",
                    help="write the measured per-CTA busy times of the last step (fwd partial and dK/dV "
                         "kernels, ns) with the schedule options to PATH as JSON")
    ap.add_argument("--schedule", choices=["lpt", "contiguous"], default="lpt",
                    help="contiguous: the pages' unbalanced baseline (chunks in order, equal counts) on the "
                         "kernels, static lists, to time what LPT saves")
    ap.add_argument("--dump-plan", default=None, metavar="PATH",
                    help="write the run's plan (problem, stats, every table) to PATH (.npz)")
    ap.add_argument("--split-kv", action="store_true",
                    help="under torchrun: Split-KV over the ranks (chunks owned by LPT, or in order with "
                         "--schedule contiguous), the whole workload split, strong scaling")
    ap.add_argument("--exchange", choices=["nccl", "p2p"], default="nccl",
                    help="with --split-kv: the forward exchange as an NCCL all-to-all, or fused into the "
                         "merge kernel as stores into the owners' peer-mapped buffers")
    ap.add_argument("--emulate-ranks", type=int, default=0, metavar="R",
                    help="also report Split-KV over R ranks, one GPU running each rank plan in turn")
    ap.add_argument("--partial-bf16", action="store_true",
                    help="store the partial records (O_c, dQ partials) as bf16 (plan flag; default float32)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    # the contiguous schedule is a CTA-level mode; under --split-kv --schedule contiguous names
    # the chunk ownership over ranks instead, and the CTAs keep LPT
    args.dynamic_claim = args.claims == "run-time" and (args.schedule == "lpt" or args.split_kv)
    return args


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = _dist()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    elif args.split_kv:
        res = run_split_kv(args, world, rank, local)
    else:
        res = run_ours(args, world, rank, local)
    if res is not None:
        # the per-kernel report and the imbalance figures close the line, so that a reader
        # that keeps only the end of a long line still sees them
        for k in ("kernels", "lpt_imbalance_pct"):
            if k in res:
                res[k] = res.pop(k)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
