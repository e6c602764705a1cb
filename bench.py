#!/usr/bin/env python
"""Hybrid-head layer prefill throughput on B200 (tokens/s) and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one forward pass of the whole hybrid-head layer (in_proj with the meta
prepend, x_proj, dt_proj, attention heads, selective scan + gate, branch
RMSNorm + beta, out_proj) over one batch of the seeded synthetic workload,
through the C ABI (hymba_layer_fwd).  Default workload: the Hymba-350M-shaped
layer (B=8, L=2048 + 32 meta tokens, d=1024, bf16).  W untimed warm-up steps,
then exactly K timed steps, each bracketed by CUDA events on the launching
stream with an L2 flush (256 MiB memset) between steps outside the events; a
barrier and a device synchronise on both sides of the timed loop; the time is
the max over ranks.  Under torchrun every rank runs its own batch (weak
scaling, no collective on the data path).  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores instead (each
step a bounded sample of the same workload), as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hybrid_attention_ssm_hymba_b200 import synth  # noqa: E402

METRIC = "hybrid-head layer prefill tokens/s at 1 B200; % of HBM/tensor roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _workload_config(wl: synth.Workload, extra=None):
    s = wl.first
    cfg = {"workload": wl.name, "description": wl.description, "batch": s.batch, "seq_len": s.seq_len,
           "n_meta": s.n_meta, "d_model": s.d_model, "n_q_heads": s.n_q_heads, "n_kv_heads": s.n_kv_heads,
           "head_dim": s.head_dim, "window": s.window, "d_inner": s.d_inner, "d_state": s.d_state,
           "dt_rank": s.dt_rank, "n_layers": len(wl.layers), "ffn_dim": s.ffn_dim, "seed": wl.seed}
    if extra:
        cfg.update(extra)
    return cfg


def _visible_pairs(T: int, M: int, W: int) -> int:
    """(query, key) pairs the attention mask admits in one sequence of T rows:
    key j <= query i and (i - j <= W or j < M); W = -1 is global causal."""
    if W < 0:
        return T * (T + 1) // 2
    i = np.arange(T, dtype=np.int64)
    return int((np.minimum(i + 1, W + 1) + np.maximum(0, np.minimum(M, i - W))).sum())


def stage_work(s: synth.LayerShape, dt_in_scan: bool = False):
    """Algorithmic work of each stage of one layer launch: (FLOPs, HBM bytes).

    FLOPs count the dense contractions only (2 per multiply-add; attention 4 dh per
    visible pair per query head).  Bytes are the compulsory traffic: every operand read
    once and every result written once (weights included), in the layer's dtype, with
    B|C in fp32.  dt_in_scan: the scan computes dt from dt_low itself (no dt_proj stage;
    the scan reads dt_low and W_dt instead of dt)."""
    es = 2 if s.dtype == "bf16" else 4
    rows = s.batch * s.T
    wa, di, n, r, d = s.attn_width, s.d_inner, s.d_state, s.dt_rank, s.d_model
    kv_out = 0 if s.kv_mode == synth.KV_CONSUME else 2 * s.kv_width
    pairs = s.batch * _visible_pairs(s.T, s.n_meta, s.window)
    work = {
        "in_proj": (2.0 * d * s.n_in * rows, es * (rows * d + s.n_in * d + rows * (wa + kv_out + 2 * di))),
        "x_proj": (2.0 * di * s.xproj_width * rows, es * (rows * di + s.xproj_width * di + rows * r) + 4 * rows * 2 * n),
        "dt_proj": (2.0 * r * di * rows, es * (rows * r + di * r + rows * di) + 4 * di),
        "attention": (4.0 * s.head_dim * s.n_q_heads * pairs,
                      es * (rows * wa + 2 * rows * s.kv_width + rows * wa)),
        "scan": (4.0 * n * di * rows, es * 4 * rows * di + 4 * rows * 2 * n + 4 * di),
        # bf16: the norm is fused into out_proj -- this stage reads Z once for the row sums of
        # squares and folds beta into a copy of W_out; fp32: Z is normalised in place
        "branch_norm": (0.0, (es * rows * (wa + di) + 8 * rows + 2 * es * d * (wa + di) + 4 * (wa + di))
                        if s.dtype == "bf16" else es * 2 * rows * (wa + di) + 4 * (wa + di)),
        "out_proj": (2.0 * (wa + di) * d * rows, es * (rows * (wa + di) + d * (wa + di) + rows * d)),
    }
    if dt_in_scan:
        fl_dt, _ = work.pop("dt_proj")
        fl, by = work["scan"]
        work["scan"] = (fl + fl_dt, by - es * rows * di + es * (rows * r + di * r) + 4 * di)
    return work


KERNEL_NAMES = {"in_proj": "gemm_bf16_tc, tcgen05", "x_proj": "gemm_bf16_tc, tcgen05",
                "dt_proj": "gemm_bf16_tc, tcgen05", "attention": "attn_fwd_tc, tcgen05",
                "scan": "scan_tc_kernel, tcgen05 tf32 (+ dt projection, bf16)", "branch_norm": "row_ssq_kernel + scale_cols_kernel",
                "out_proj": "gemm_bf16_tc, tcgen05, two accumulators"}

# dominant bound of each stage: a dense contraction on the tensor cores or HBM traffic
STAGE_BOUND = {"in_proj": "tensor", "x_proj": "hbm", "dt_proj": "hbm", "attention": "tensor",
               "scan": "hbm", "branch_norm": "hbm", "out_proj": "tensor"}


def _traffic(stage: str):
    """DRAM bytes per launch from the committed ncu capture of this stage's kernel,
    or None when there is none or the kernel's source changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(stage)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["sha256"]:
        return None
    return rec["dram_bytes_per_launch"]


def stage_rooflines(s: synth.LayerShape, stage_us, peaks, dt_in_scan=False):
    """Per stage: achieved work rate against its peak (measured peaks), and the layer's
    roofline time (sum over stages of the slower of its FLOP and byte times)."""
    out, t_roof = {}, 0.0
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops_sustained"] * 1e12
    for name, (fl, by) in stage_work(s, dt_in_scan).items():
        t = stage_us[name] * 1e-6
        t_roof += max(fl / tc, by / hbm)
        if STAGE_BOUND[name] == "tensor":
            ach = fl / t / 1e12
            out[name] = {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops_sustained"], 4),
                         "work_per_launch": fl, "us": stage_us[name]}
        else:
            ach = by / t / 1e9
            out[name] = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach / peaks["hbm_gbs"], 4), "work_per_launch": by, "us": stage_us[name]}
    return out, t_roof * 1e6


# --------------------------------------------------------------------------- clocks (NVML)

class ClockSampler:
    """Polls SM clock and clock-event reasons of one GPU on a thread while active."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x100: "display_clock_setting", 0x10: "sync_boost"}

    def __init__(self, device):
        self.samples, self.reasons, self.ok = [], set(), False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            try:   # NVML enumerates every GPU; match the CUDA device by UUID
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml unavailable" if not self.ok else "nvml"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------------------- CPU oracle legs

def _oracle_sample(wl: synth.Workload, x, meta, ps, b: int, L: int):
    """Run the oracle on sequence b, first L tokens, through every layer of the workload."""
    import dataclasses

    import oracle as O
    xb = x[b:b + 1, :L]
    shapes = [dataclasses.replace(s, batch=1, seq_len=L) for s in wl.layers]
    if wl.first.ffn_dim:
        return O.stack_forward(xb, meta, ps, shapes)
    h, kv = O.layer_forward(xb, meta, ps[0], shapes[0])
    for i in range(1, len(shapes)):
        h, _ = O.layer_forward(h, None, ps[i], shapes[i], kv_in=kv)
    return h


def _sample_len(wl: synth.Workload) -> int:
    s = wl.first
    if s.ffn_dim:
        return min(s.seq_len, 256)
    return min(s.seq_len, 2048)


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, x, meta, ps, budget_s=12.0):
    L = _sample_len(wl)
    done, t0 = 0, time.perf_counter()
    seqs = []
    for b in range(wl.first.batch):
        _oracle_sample(wl, x, meta, ps, b, L)
        done += L
        seqs.append(b)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle on sequences {seqs} of the workload, first {L} of "
                      f"{wl.first.seq_len} user tokens each ({dt:.1f} s wall)"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = synth.workload(args.workload)
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(len(wl.layers))]
    L = _sample_len(wl)
    B = wl.first.batch
    for i in range(args.warmup):
        _oracle_sample(wl, x, meta, ps, i % B, L)
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        _oracle_sample(wl, x, meta, ps, i % B, L)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * L / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _workload_config(wl, {"sample_tokens_per_step": L}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
                             "sample": f"each step: one sequence (rotating), first {L} user tokens, "
                                       "all layers of the workload, fp64 numpy oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- multi-process plumbing

class Ranks:
    """One process per GPU: the process group, its barrier and the max over ranks.
    World 1 needs no process group; the data path has no collective (each rank runs
    its own batch), so the only cross-rank traffic is timing."""

    def __init__(self, world: int, local_rank: int, backend: str, device, timeout_s: float = 180.0):
        import torch.distributed as dist
        self.world, self.local_rank, self.backend, self.device = world, local_rank, backend, device
        self.dist = dist
        if world > 1:
            from datetime import timedelta
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.local_rank])
            else:
                self.dist.barrier()

    def max(self, value: float) -> float:
        """The largest value over the ranks (every rank gets it)."""
        if self.world == 1:
            return float(value)
        import torch
        t = torch.tensor([float(value)], device=self.device, dtype=torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def weak_scaling_rate(world: int, steps: int, units_per_step_per_rank: float, max_total_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * steps * units_per_step_per_rank / (max_total_ms * 1e-3)


# --------------------------------------------------------------------------- native (CUDA) leg

def run_native(args, rank, world, local_rank):
    import torch

    import hybrid_attention_ssm_hymba_b200 as H
    from hybrid_attention_ssm_hymba_b200 import host

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ranks = Ranks(world, local_rank, "nccl", dev)
    barrier = ranks.barrier

    wl = synth.workload(args.workload)
    s0 = wl.first
    dtype = s0.dtype
    x_np, meta_np = synth.layer_inputs(wl)
    ps_np = [synth.layer_params(wl, i) for i in range(len(wl.layers))]
    dps = [host.params_to_device(p, dtype, dev) for p in ps_np]
    cfgs = [H.make_cfg(s) for s in wl.layers]
    weights = [H.make_weights(d) for d in dps]
    T = s0.T
    x = host.to_device(x_np, dtype, dev)
    meta = host.to_device(meta_np, dtype, dev)
    stack = bool(s0.ffn_dim)
    ws_bytes = H.hymba_stack_workspace_size(cfgs) if stack else max(H.hymba_workspace_size(c) for c in cfgs)
    ws = host.workspace(ws_bytes, dev)
    outs = [torch.empty((s0.batch, T, s0.d_model), dtype=x.dtype, device=dev) for _ in wl.layers]
    kv = torch.empty((2, s0.batch * T, s0.kv_width), dtype=x.dtype, device=dev) if len(wl.layers) > 1 \
        and not stack else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # this library's kernels per step: in_proj, x_proj, dt_proj (unless the scan computes dt),
    # attention, scan, out_proj and the norm stage (bf16: row sums + beta-scaled W_out; fp32:
    # in-place norm); a stack adds two pre-norms and the two FFN GEMMs per block, and the
    # meta prepend
    dt_in_scan = [H.hymba_layer_fuses_dt_proj(c) for c in cfgs]
    n_launch_per_step = sum((8 if dtype == "bf16" else 7) - int(f) for f in dt_in_scan) + \
        (4 * len(wl.layers) + 1 if stack else 0)

    def step(xin, stage_events=None, out_list=None):
        o = outs if out_list is None else out_list
        if stack:
            H.check(H.hymba_stack_fwd(xin, meta, weights, cfgs, o[0], ws, stream=stream), "stack")
            return o[0]
        if stage_events is not None:
            H.check(H.hymba_layer_fwd_events(xin, meta, weights[0], cfgs[0], None, kv, o[0], ws,
                                             stage_events, stream=stream), "layer")
        else:
            H.check(H.hymba_layer_fwd(xin, meta, weights[0], cfgs[0], None, kv, o[0], ws, stream=stream),
                    "layer")
        for i in range(1, len(wl.layers)):
            H.check(H.hymba_layer_fwd(o[i - 1], None, weights[i], cfgs[i], kv, None, o[i], ws,
                                      stream=stream), f"layer {i}")
        return o[-1]

    for _ in range(args.warmup):
        flush.zero_()
        step(x)
    torch.cuda.synchronize(dev)
    assert H.hymba_workspace_status(ws, stream) == H.HYMBA_OK

    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(dev)
    barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        for k in range(K):
            flush.zero_()
            ev_s[k].record(stream)
            step(x)
            ev_e[k].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    # Stage breakdown in a separate pass: events between the kernels of a step order
    # them fully (no programmatic overlap), so they are kept out of the timed steps.
    n_stage = max(3, min(K, 50))
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(n_stage)] \
        if not stack else None
    if stage_ev:
        for evs in stage_ev:   # torch creates the CUDA event lazily, at its first record
            for e in evs:
                e.record(stream)
        torch.cuda.synchronize(dev)
        for k in range(n_stage):
            flush.zero_()
            step(x, stage_ev[k])
        torch.cuda.synchronize(dev)
    step_ms = [ev_s[k].elapsed_time(ev_e[k]) for k in range(K)]
    total_ms = ranks.max(float(sum(step_ms)))
    status = H.hymba_workspace_status(ws, stream)
    tokens_per_step = s0.batch * s0.seq_len
    value = weak_scaling_rate(world, K, tokens_per_step, total_ms)

    peaks, peak_src = _peaks()
    roofline, stages, stage_roof, layer_roof = None, None, None, None
    if stage_ev:
        per_stage = {name: float(np.mean([stage_ev[k][i].elapsed_time(stage_ev[k][i + 1]) for k in range(n_stage)]))
                     for i, name in enumerate(H.STAGES)}
        stages = {n: round(v * 1e3, 2) for n, v in per_stage.items()}  # microseconds
        if dt_in_scan[0]:   # stage 2 launches nothing: dt is computed inside the scan
            stages.pop("dt_proj")
        stage_roof, t_roof_us = stage_rooflines(s0, stages, peaks, dt_in_scan[0])
        top = max(stages, key=stages.get)   # the dominant kernel of the step
        r = stage_roof[top]
        roofline = {"kernel": f"{top} ({KERNEL_NAMES[top]})", "bound": r["bound"], "achieved": r["achieved"],
                    "peak": r["peak"], "unit": r["unit"], "frac": r["frac"], "traffic": _traffic(top),
                    "peak_source": (f"{peak_src} bf16_tflops_sustained (kernel timed inside a continuous loop)"
                                    if r["bound"] == "tensor" else f"{peak_src} hbm_gbs (STREAM-style copy)"),
                    "us_per_launch": stages[top], "algorithmic_work_per_launch": r["work_per_launch"]}
        layer_roof = {"roofline_us": round(t_roof_us, 2), "measured_us": round(1e3 * total_ms / K, 2),
                      "frac": round(t_roof_us / (1e3 * total_ms / K), 4),
                      "definition": "sum over stages of max(FLOPs / bf16 sustained peak, bytes / HBM peak), "
                                    "against the timed step"}

    e2e = None
    if not args.no_e2e:
        # Through the public entry point with host buffers, as a serving loop runs it: each
        # step copies its input from pinned host memory and its output back, double-buffered
        # over three streams so that step k's input copy (host -> device), step k-1's layer
        # (the compute stream, with the same L2 flush before it) and step k-2's output copy
        # (device -> host) overlap.  Timed from the first timed input copy to the last output
        # copy, on the device.
        xh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
        xh.copy_(x.cpu())
        ohs = [torch.empty(outs[-1].shape, dtype=x.dtype).pin_memory() for _ in range(2)]
        xds = [torch.empty_like(x) for _ in range(2)]
        out_sets = [outs, [torch.empty_like(o) for o in outs]]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        n_e2e, n_warm = max(3, min(K, 50)), 3
        total = n_warm + n_e2e
        h2d = [torch.cuda.Event() for _ in range(total)]
        comp = [torch.cuda.Event() for _ in range(total)]
        d2h = [torch.cuda.Event() for _ in range(total)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        for k in range(total):
            j = k % 2
            if k == n_warm:
                torch.cuda.synchronize(dev)   # warm-up steps done; the timed pipeline starts empty
                t0.record(s_in)
            if k >= 2:
                s_in.wait_event(comp[k - 2])   # the layer that read xds[j] is done
            with torch.cuda.stream(s_in):
                xds[j].copy_(xh, non_blocking=True)
            h2d[k].record(s_in)
            stream.wait_event(h2d[k])
            if k >= 2:
                stream.wait_event(d2h[k - 2])  # out_sets[j] has been copied out
            flush.zero_()
            o = step(xds[j], out_list=out_sets[j])
            comp[k].record(stream)
            s_out.wait_event(comp[k])
            with torch.cuda.stream(s_out):
                ohs[j].copy_(o, non_blocking=True)
            d2h[k].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = ranks.max(float(t0.elapsed_time(t1)))
        e2e = {"value": weak_scaling_rate(world, n_e2e, tokens_per_step, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": ohs[0].numel() * ohs[0].element_size(), "steps": n_e2e,
               "path": "pinned host x -> device (copy stream), hymba_layer_fwd / hymba_stack_fwd (compute "
                       "stream, L2 flushed before each step), device out -> pinned host (copy stream); two "
                       "buffers each, so consecutive steps' copies and layers overlap"}

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
                "config": _workload_config(wl, {
                    "parallelism": f"replicas x{world} (batch per rank, no collective)" if world > 1 else "1 GPU",
                    "tokens_per_step_per_gpu": tokens_per_step, "rows_per_step_per_gpu": s0.batch * T,
                    "l2": "flushed between timed steps (256 MiB memset outside the events)"}),
                "roofline": roofline, "stages_us": stages, "stages_note": "stage events in a separate "
                f"{n_stage}-step pass (events between kernels disable their programmatic overlap)" if stages else None,
                "stage_roofline": stage_roof,
                "layer_roofline": layer_roof, "e2e": e2e,
                "gpu_launches": n_launch_per_step * K, "clocks": sampler.summary(),
                "device_status": H.hymba_status_string(status)}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, x_np, meta_np, ps_np)
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="hymba350m_layer", choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("note: fewer than 3 warm-up steps requested", file=sys.stderr)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_native(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
