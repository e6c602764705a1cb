#!/usr/bin/env python
"""Hybrid-head layer prefill throughput on B200 (tokens/s) and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one forward pass of every layer of the workload (in_proj with the meta
prepend, x_proj, dt_proj, attention heads, selective scan + gate, branch RMSNorm +
beta, out_proj; the stacked workload adds the pre-norms and the SwiGLU FFN) over one
batch of the seeded synthetic workload, through the C ABI.  Default workload: the
Hymba-1.5B-shaped producer + consumer layer pair sharing K/V (B=4, L=8192 + 128 meta
tokens, d=2048, SWA 1024, d_state 128, bf16) -- the largest single-GPU layer
configuration.  W untimed warm-up steps, then exactly K timed steps, each bracketed
by CUDA events on the launching stream with an L2 flush (256 MiB memset) between
steps outside the events; a barrier and a device synchronise on both sides of the
timed loop; the time is the max over ranks.  Under torchrun every rank runs its own
batch (weak scaling, no collective on the data path).  Rank 0 prints one JSON line;
at N = 1 it also carries `per_workload` (every other workload measured the same way
with fewer steps) and `decode` (the generation step of the layer pair).

--impl reference times the fp64 CPU oracle on the host cores instead (each step a
bounded sample of the same workload), as the reference arm.
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


def ffn_work(s: synth.LayerShape):
    """SwiGLU FFN and the two pre-norms of a stacked block: (FLOPs, HBM bytes)."""
    es = 2 if s.dtype == "bf16" else 4
    rows, d, F = s.batch * s.T, s.d_model, s.ffn_dim
    fl = 6.0 * d * F * rows
    by = es * (rows * d + 2 * F * d + rows * F) + es * (rows * F + F * d) + 4 * rows * d * 2
    by += 2 * (4 * rows * d + es * rows * d)          # pre-norms: read h (fp32), write the bf16 operand
    return fl, by


def scan_kernel_name(s: synth.LayerShape) -> str:
    """The scan kernel the library selects for a layer (mirrors the C++ choice)."""
    if s.dtype == "bf16" and not s.a_per_state:
        if s.d_state == 16:
            return "scan_tc_kernel, tcgen05 tf32"
        if s.d_state == 128 and s.dt_rank % 8 == 0 and 8 <= s.dt_rank <= 128:
            return "scan_tc128_kernel, tcgen05 tf32, state in TMEM"
    return "scan_w_kernel, fp32 FMA"


GEMM_STAGES = ("in_proj", "x_proj", "dt_proj", "out_proj")


def stage_bound(stage: str, s: synth.LayerShape, work=None, peaks=None) -> str:
    """The bound that binds each stage: a dense contraction on the tensor cores, HBM
    traffic, or (the CUDA-core scan) the fp32 FMA rate.  A GEMM stage is held to whichever
    of its FLOP time and its byte time is longer (x_proj's N = dt_rank + 2 d_state is
    narrow: byte-bound on some shapes, FLOP-bound on others); given no work and peaks it
    counts as a contraction."""
    if stage == "attention":
        return "tensor"
    if stage in GEMM_STAGES:
        if work is None or peaks is None:
            return "tensor"
        fl, by = work
        return "tensor" if fl / (peaks["bf16_tflops"] * 1e12) >= by / (peaks["hbm_gbs"] * 1e9) else "hbm"
    if stage == "scan" and not scan_kernel_name(s).startswith("scan_tc"):
        return "alu"
    return "hbm"


KERNEL_NAMES = {"in_proj": "gemm_bf16_tc, tcgen05", "x_proj": "gemm_bf16_tc, tcgen05",
                "dt_proj": "gemm_bf16_tc, tcgen05", "attention": "attn_fwd_tc2, tcgen05",
                "branch_norm": "row_ssq_bulk_kernel + scale_cols_kernel",
                "out_proj": "gemm_bf16_tc, tcgen05, two accumulators"}

PROFILE_COMMON = ("hybrid_attention_ssm_hymba_b200/csrc/hy_common.cuh",
                  "hybrid_attention_ssm_hymba_b200/csrc/hy_kernels.h")


def source_hash(sources) -> str:
    """sha256 over a kernel's source file and the headers every kernel includes."""
    import hashlib
    h = hashlib.sha256()
    for rel in list(sources) + list(PROFILE_COMMON):
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()


def _traffic(workload: str, stage: str):
    """DRAM bytes per launch from the committed ncu capture of this stage's kernel on this
    workload, or None when there is none or the kernel's sources (its file and the common
    headers) changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload, {}).get(stage)
    if not rec:
        return None
    try:
        if source_hash(rec["sources"]) != rec["sha256"]:
            return None
    except OSError:
        return None
    return rec["dram_bytes_per_launch"]


def alu_peak_tflops(peaks, sm_mhz=None):
    """fp32 FMA peak: 148 SMs x 128 lanes x 2 FLOP per clock at the SM clock (the sampled
    maximum, else 1965 MHz)."""
    return 148 * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def stage_rooflines(layers, stage_us, peaks, dt_in_scan, sm_max_mhz=None):
    """Per stage, summed over the layers of the workload: the achieved rate of its binding
    resource against that resource's measured peak (tensor: burst bf16 -- the layers run
    in sub-second steps; HBM: the measured copy bandwidth; fp32 FMA: derived), and the
    workload's roofline time (sum over stages of the slowest of its FLOP, byte and ALU
    times)."""
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops"] * 1e12
    alu = alu_peak_tflops(peaks, sm_max_mhz) * 1e12
    tot = {}
    t_roof = 0.0
    for s, fused in zip(layers, dt_in_scan):
        for name, (fl, by) in stage_work(s, fused).items():
            b = stage_bound(name, s, (fl, by), peaks)
            t_roof += max(fl / tc if b == "tensor" else 0.0, by / hbm, fl / alu if b == "alu" else 0.0)
            f0, b0, _ = tot.get(name, (0.0, 0.0, b))
            tot[name] = (f0 + fl, b0 + by, b)
    out = {}
    for name, (fl, by, b) in tot.items():
        t = stage_us[name] * 1e-6
        if b == "tensor":
            ach = fl / t / 1e12
            out[name] = {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4), "work": fl,
                         "us": stage_us[name]}
        elif b == "alu":
            ach = fl / t / 1e12
            pk = alu / 1e12
            out[name] = {"bound": "alu", "achieved": round(ach, 2), "peak": round(pk, 2), "unit": "TFLOP/s",
                         "frac": round(ach / pk, 4), "work": fl, "us": stage_us[name],
                         "hbm_frac": round(by / t / hbm, 4)}
        else:
            ach = by / t / 1e9
            out[name] = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach / peaks["hbm_gbs"], 4), "work": by, "us": stage_us[name]}
    return out, t_roof * 1e6


def stack_roofline_us(layers, peaks, dt_in_scan):
    """Roofline time of a stacked workload: every layer's stages plus its FFN and pre-norms."""
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops"] * 1e12
    alu = alu_peak_tflops(peaks) * 1e12
    t = 0.0
    for s, fused in zip(layers, dt_in_scan):
        for name, (fl, by) in stage_work(s, fused).items():
            b = stage_bound(name, s, (fl, by), peaks)
            t += max(fl / tc if b == "tensor" else 0.0, by / hbm, fl / alu if b == "alu" else 0.0)
        if s.ffn_dim:
            fl, by = ffn_work(s)
            t += max(fl / tc, by / hbm)
    return t * 1e6


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
    """User tokens of one oracle sample: about half a second of fp64 work on a host core
    set for every workload (its cost per token grows with width, state size and depth)."""
    s = wl.first
    if s.ffn_dim:
        return min(s.seq_len, 64)
    if s.d_state >= 128 or s.d_model >= 2048:
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

class Workbench:
    """Device-resident inputs, weights and buffers of one workload, and its step."""

    def __init__(self, name, dev, **overrides):
        import torch

        import hybrid_attention_ssm_hymba_b200 as H
        from hybrid_attention_ssm_hymba_b200 import host
        self.H, self.torch = H, torch
        self.wl = wl = synth.workload(name, **overrides)
        self.s0 = s0 = wl.first
        self.dtype = s0.dtype
        self.x_np, self.meta_np = synth.layer_inputs(wl)
        self.ps_np = [synth.layer_params(wl, i) for i in range(len(wl.layers))]
        self.dps = [host.params_to_device(p, self.dtype, dev) for p in self.ps_np]
        self.cfgs = [H.make_cfg(s) for s in wl.layers]
        self.weights = [H.make_weights(d) for d in self.dps]
        self.x = host.to_device(self.x_np, self.dtype, dev)
        self.meta = host.to_device(self.meta_np, self.dtype, dev)
        self.stack = bool(s0.ffn_dim)
        ws_bytes = H.hymba_stack_workspace_size(self.cfgs) if self.stack else \
            max(H.hymba_workspace_size(c) for c in self.cfgs)
        self.ws = host.workspace(ws_bytes, dev)
        T = s0.T
        self.outs = [torch.empty((s0.batch, T, s0.d_model), dtype=self.x.dtype, device=dev) for _ in wl.layers]
        self.kv = torch.empty((2, s0.batch * T, s0.kv_width), dtype=self.x.dtype, device=dev) \
            if len(wl.layers) > 1 and not self.stack else None
        self.stream = torch.cuda.current_stream(dev)
        self.dt_in_scan = [H.hymba_layer_fuses_dt_proj(c) for c in self.cfgs]
        bf16 = self.dtype == "bf16"
        # in_proj, x_proj, dt_proj (unless the scan computes dt), attention, scan, the branch norm
        # (bf16 whole-branch: row sums + beta-scaled W_out; else one in-place norm), out_proj;
        # the options add the conv and the D skip
        per_layer = [(8 if bf16 and not s.norm_group else 7) - int(f) + int(s.conv_width > 0) + int(bool(s.d_skip))
                     for f, s in zip(self.dt_in_scan, wl.layers)]
        if self.stack:   # the prepend; per block: the mixer's pre-norm (bf16 without the conv: + the
            # W_SSM transpose, the W_x W_SSM GEMM and its hi/lo split), the layer, and with an FFN
            # its pre-norm and two GEMMs
            self.launches = 1 + sum(n + (4 if bf16 and not s.conv_width else 1) + (3 if s.ffn_dim else 0)
                                    for n, s in zip(per_layer, wl.layers))
        else:
            self.launches = sum(per_layer)
        self.tokens = s0.batch * s0.seq_len

    def step(self, xin, stage_events=None, out_list=None):
        H = self.H
        o = self.outs if out_list is None else out_list
        st = self.stream
        if self.stack:
            H.check(H.hymba_stack_fwd(xin, self.meta, self.weights, self.cfgs, o[0], self.ws, stream=st), "stack")
            return o[0]
        meta = self.meta
        for i in range(len(self.cfgs)):
            kv_in = self.kv if i > 0 else None
            kv_out = self.kv if i == 0 else None
            if stage_events is not None:
                H.check(H.hymba_layer_fwd_events(xin, meta, self.weights[i], self.cfgs[i], kv_in, kv_out, o[i],
                                                 self.ws, stage_events[i], stream=st), f"layer {i}")
            else:
                H.check(H.hymba_layer_fwd(xin, meta, self.weights[i], self.cfgs[i], kv_in, kv_out, o[i], self.ws,
                                          stream=st), f"layer {i}")
            xin, meta = o[i], None
        return o[-1]


def measure(bench: Workbench, K: int, W: int, ranks, dev, flush, stages=True, e2e=False):
    """Time K steps of the workload (after W warm-up steps), then optionally the stage
    breakdown and the end-to-end path.  Returns (record, total_ms)."""
    import torch
    H = bench.H
    stream = bench.stream
    for _ in range(W):
        flush.zero_()
        bench.step(bench.x)
    torch.cuda.synchronize(dev)
    assert H.hymba_workspace_status(bench.ws, stream) == H.HYMBA_OK
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(dev)
    ranks.barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        for k in range(K):
            flush.zero_()
            ev_s[k].record(stream)
            bench.step(bench.x)
            ev_e[k].record(stream)
        torch.cuda.synchronize(dev)
        ranks.barrier()
        # clocks under load: keep stepping (untimed) until the sampler has a few hundred ms
        t_end = time.perf_counter() + 0.3
        while time.perf_counter() < t_end:
            bench.step(bench.x)
        torch.cuda.synchronize(dev)
    step_ms = [ev_s[k].elapsed_time(ev_e[k]) for k in range(K)]
    total_ms = ranks.max(float(sum(step_ms)))
    rec = {"ms_per_step": total_ms / K, "steps": K, "warmup": W, "clocks": sampler.summary(),
           "gpu_launches": bench.launches * K}
    peaks, peak_src = _peaks()
    wl = bench.wl
    if stages and not bench.stack:
        # Stage breakdown in a separate pass: events between the kernels of a step order them
        # fully (no programmatic overlap, the attention on the caller's stream), so they are
        # kept out of the timed steps.
        n_stage = max(3, min(K, 20))
        nl = len(bench.cfgs)
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(nl)] for _ in range(n_stage)]
        for per_step in ev:   # torch creates the CUDA event lazily, at its first record
            for evs in per_step:
                for e in evs:
                    e.record(stream)
        torch.cuda.synchronize(dev)
        for k in range(n_stage):
            flush.zero_()
            bench.step(bench.x, ev[k])
        torch.cuda.synchronize(dev)
        stages_us = {}
        by_layer = []
        for li in range(nl):
            per = {name: 1e3 * float(np.mean([ev[k][li][i].elapsed_time(ev[k][li][i + 1]) for k in range(n_stage)]))
                   for i, name in enumerate(H.STAGES)}
            if bench.dt_in_scan[li]:   # stage 2 launches nothing: dt is computed inside the scan
                per.pop("dt_proj")
            by_layer.append({k: round(v, 2) for k, v in per.items()})
            for k, v in per.items():
                stages_us[k] = stages_us.get(k, 0.0) + v
        stages_us = {k: round(v, 2) for k, v in stages_us.items()}
        stage_roof, t_roof_us = stage_rooflines(wl.layers, stages_us, peaks, bench.dt_in_scan,
                                                rec["clocks"].get("sm_max_mhz"))
        top = max(stages_us, key=stages_us.get)
        r = stage_roof[top]
        kname = KERNEL_NAMES.get(top) or scan_kernel_name(wl.first)
        n_launch = nl
        peak_note = {"tensor": f"{peak_src} bf16_tflops (burst: the kernel runs inside a sub-second step)",
                     "hbm": f"{peak_src} hbm_gbs (STREAM-style copy)",
                     "alu": "fp32 FMA peak derived from 148 SMs x 128 lanes x 2 FLOP x the SM clock"}[r["bound"]]
        traffic = _traffic(wl.name, top)
        rec["roofline"] = {"kernel": f"{top} ({kname})", "bound": r["bound"], "achieved": r["achieved"],
                           "peak": r["peak"], "unit": r["unit"], "frac": r["frac"],
                           "traffic": traffic if traffic is None else traffic,
                           "peak_source": peak_note, "launches_per_step": n_launch,
                           "us_per_launch": round(stages_us[top] / n_launch, 2),
                           "algorithmic_work_per_launch": r["work"] / n_launch}
        rec["stages_us"] = stages_us
        if nl > 1:
            rec["stages_us_by_layer"] = by_layer
        rec["stages_note"] = (f"stage events in a separate {n_stage}-step pass (events between kernels disable "
                              "their programmatic overlap and the second stream)")
        rec["stage_roofline"] = stage_roof
        rec["layer_roofline"] = {"roofline_us": round(t_roof_us, 2), "measured_us": round(1e3 * rec["ms_per_step"], 2),
                                 "frac": round(t_roof_us / (1e3 * rec["ms_per_step"]), 4),
                                 "definition": "sum over stages and layers of max(tensor FLOPs / burst bf16 peak, "
                                               "bytes / HBM peak, scan FMA FLOPs / fp32 peak where the CUDA-core "
                                               "scan runs), against the timed step"}
    elif bench.stack:
        t_roof_us = stack_roofline_us(wl.layers, peaks, bench.dt_in_scan)
        rec["layer_roofline"] = {"roofline_us": round(t_roof_us, 2), "measured_us": round(1e3 * rec["ms_per_step"], 2),
                                 "frac": round(t_roof_us / (1e3 * rec["ms_per_step"]), 4),
                                 "definition": "sum over the blocks of their stages' bounds plus the SwiGLU FFN and "
                                               "pre-norms (max of tensor FLOPs / burst bf16 peak and bytes / HBM "
                                               "peak), against the timed step"}
    if e2e:
        rec["e2e"] = measure_e2e(bench, ranks, dev, flush, K)
    return rec, total_ms


def measure_e2e(bench: Workbench, ranks, dev, flush, K):
    """Through the public entry point with host buffers, as a serving loop runs it: each step
    copies its input from pinned host memory and its output back, double-buffered over three
    streams so that step k's input copy (host -> device), step k-1's layers (the compute
    stream, with the same L2 flush before it) and step k-2's output copy (device -> host)
    overlap.  Timed from the first timed input copy to the last output copy, on the device."""
    import torch
    x, outs, stream = bench.x, bench.outs, bench.stream
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
    ranks.barrier()
    torch.cuda.synchronize(dev)
    for k in range(total):
        j = k % 2
        if k == n_warm:
            torch.cuda.synchronize(dev)   # warm-up steps done; the timed pipeline starts empty
            t0.record(s_in)
        if k >= 2:
            s_in.wait_event(comp[k - 2])   # the layers that read xds[j] are done
        with torch.cuda.stream(s_in):
            xds[j].copy_(xh, non_blocking=True)
        h2d[k].record(s_in)
        stream.wait_event(h2d[k])
        if k >= 2:
            stream.wait_event(d2h[k - 2])  # out_sets[j] has been copied out
        flush.zero_()
        o = bench.step(xds[j], out_list=out_sets[j])
        comp[k].record(stream)
        s_out.wait_event(comp[k])
        with torch.cuda.stream(s_out):
            ohs[j].copy_(o, non_blocking=True)
        d2h[k].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    e_ms = ranks.max(float(t0.elapsed_time(t1)))
    return {"value": weak_scaling_rate(ranks.world, n_e2e, bench.tokens, e_ms), "unit": UNIT,
            "h2d_bytes_per_step": xh.numel() * xh.element_size(),
            "d2h_bytes_per_step": ohs[0].numel() * ohs[0].element_size(), "steps": n_e2e,
            "path": "pinned host x -> device (copy stream), hymba_layer_fwd / hymba_stack_fwd (compute "
                    "stream, L2 flushed before each step), device out -> pinned host (copy stream); two "
                    "buffers each, so consecutive steps' copies and layers overlap"}


def measure_prefixed(bench: Workbench, K: int, W: int, dev, flush):
    """The workload's layers with their meta rows from records of hymba_meta_prefix (built
    once, outside the timed region): hymba_layer_fwd_prefixed runs the user rows only.
    Timed like the headline (K steps, L2 flushed between them)."""
    import torch
    H = bench.H
    from hybrid_attention_ssm_hymba_b200 import host
    s0, st = bench.s0, bench.stream
    if bench.stack or s0.n_meta == 0:
        return None
    es = 2 if bench.dtype == "bf16" else 4
    recs = [host.workspace(H.hymba_meta_prefix_size(c), dev) for c in bench.cfgs]
    meta_in = bench.meta
    for i, c in enumerate(bench.cfgs):
        H.check(H.hymba_meta_prefix(meta_in, bench.weights[i], c, recs[0] if i > 0 else None, recs[i], bench.ws,
                                    stream=st), "meta prefix")
        meta_in = recs[i][:s0.n_meta * s0.d_model * es].view(bench.x.dtype).view(s0.n_meta, s0.d_model)
    user_in = [None] + [o[:, s0.n_meta:] for o in bench.outs[:-1]]
    # a consumer's input rows: the producer's user rows, in a contiguous buffer
    user_bufs = [None] + [torch.empty((s0.batch, s0.seq_len, s0.d_model), dtype=bench.x.dtype, device=dev)
                          for _ in bench.outs[:-1]]

    def step():
        xin = bench.x
        for i, c in enumerate(bench.cfgs):
            if i > 0:
                user_bufs[i].copy_(user_in[i])
                xin = user_bufs[i]
            H.check(H.hymba_layer_fwd_prefixed(xin, recs[i], bench.weights[i], c, bench.kv if i > 0 else None,
                                               bench.kv if i == 0 else None, bench.outs[i], bench.ws, stream=st),
                    "prefixed")

    for _ in range(W):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush.zero_()
        ev[k][0].record(st)
        step()
        ev[k][1].record(st)
    torch.cuda.synchronize(dev)
    assert H.hymba_workspace_status(bench.ws, st) == H.HYMBA_OK
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    return {"ms_per_step": ms, "value": bench.tokens / (ms * 1e-3), "unit": UNIT,
            "note": "meta rows from hymba_meta_prefix records built once per weight set; each step runs "
                    "hymba_layer_fwd_prefixed on the user rows (a consumer's input copied out of the producer's "
                    "output rows inside the step)"}


def measure_decode(name: str, dev, flush, steps: int = 64, warmup: int = 8):
    """Generation steps of a layer workload after its full prompt: hymba_layer_prefill of every
    layer (untimed), then one new token per sequence per step through every layer
    (hymba_layer_decode), timed with CUDA events over `steps` steps."""
    import torch

    import hybrid_attention_ssm_hymba_b200 as H
    from hybrid_attention_ssm_hymba_b200 import host
    wl = synth.workload(name)
    s0 = wl.first
    dt = s0.dtype
    x_np, meta_np = synth.layer_inputs(wl)
    dps = [host.params_to_device(synth.layer_params(wl, i), dt, dev) for i in range(len(wl.layers))]
    cfgs = [H.make_cfg(s) for s in wl.layers]
    T = s0.T
    cap = T + warmup + steps
    ws = host.workspace(max(H.hymba_decode_workspace_size(c) for c in cfgs), dev)
    cache = torch.zeros((2, s0.batch, cap, s0.kv_width), dtype=host.torch_dtype(dt), device=dev)
    states = [torch.zeros((s0.batch, s.d_inner, s.d_state), dtype=torch.float32, device=dev) for s in wl.layers]
    weights = [H.make_weights(d) for d in dps]
    xin, meta = host.to_device(x_np, dt, dev), host.to_device(meta_np, dt, dev)
    for i, c in enumerate(cfgs):
        out = torch.empty((s0.batch, T, s0.d_model), dtype=host.torch_dtype(dt), device=dev)
        H.check(H.hymba_layer_prefill(xin, meta, weights[i], c, cache, cap, states[i], out, ws), "prefill")
        xin, meta = out, None
    toks = torch.randn((warmup + steps, s0.batch, s0.d_model), device=dev).to(host.torch_dtype(dt))
    bufs = [torch.empty((s0.batch, s0.d_model), dtype=host.torch_dtype(dt), device=dev) for _ in wl.layers]

    def one(k):
        xi = toks[k]
        for i, c in enumerate(cfgs):
            H.check(H.hymba_layer_decode(xi, weights[i], c, cache, cap, T + k, states[i], bufs[i], ws), "decode")
            xi = bufs[i]

    for k in range(warmup):
        one(k)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(warmup, warmup + steps):
        one(k)
    t1.record()
    torch.cuda.synchronize(dev)
    assert H.hymba_workspace_status(ws) == H.HYMBA_OK
    ms = t0.elapsed_time(t1)
    return {"workload": name, "tokens_per_s": s0.batch * steps / (ms * 1e-3), "unit": "tokens/s",
            "us_per_step": round(1e3 * ms / steps, 2), "steps": steps, "batch": s0.batch,
            "context_rows": [T + warmup, T + warmup + steps], "layers": len(cfgs),
            "launches_per_step": 8 * len(cfgs),
            "note": "one new token per sequence per step through every layer of the workload, after the "
                    "full prompt; K/V cache and SSM state resident; no L2 flush between steps (a generation "
                    "loop re-reads the same weights)"}


def run_native(args, rank, world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ranks = Ranks(world, local_rank, "nccl", dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    bench = Workbench(args.workload, dev, **({"batch": args.batch} if args.batch else {}))
    K = args.steps
    rec, total_ms = measure(bench, K, args.warmup, ranks, dev, flush, stages=True, e2e=not args.no_e2e)
    value = weak_scaling_rate(world, K, bench.tokens, total_ms)
    status = bench.H.hymba_workspace_status(bench.ws, bench.stream)
    wl, s0 = bench.wl, bench.s0

    line = None
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": bench.dtype, "data": "synthetic",
                "config": _workload_config(wl, {
                    "parallelism": f"replicas x{world} (batch per rank, no collective)" if world > 1 else "1 GPU",
                    "tokens_per_step_per_gpu": bench.tokens, "rows_per_step_per_gpu": s0.batch * s0.T,
                    "l2": "flushed between timed steps (256 MiB memset outside the events)"})}
        for k in ("roofline", "stages_us", "stages_us_by_layer", "stages_note", "stage_roofline", "layer_roofline",
                  "e2e", "gpu_launches", "clocks"):
            if k in rec:
                line[k] = rec[k]
        line["device_status"] = bench.H.hymba_status_string(status)
        try:
            pre = measure_prefixed(bench, K, args.warmup, dev, flush)
            if pre is not None:
                pre["saving_frac"] = round(1.0 - pre["ms_per_step"] / line["ms_per_step"], 4)
                line["meta_prefix"] = pre
        except Exception as ex:  # noqa: BLE001 -- reported in the line, the headline stands
            line["meta_prefix"] = {"error": f"{type(ex).__name__}: {ex}"}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, bench.x_np, bench.meta_np, bench.ps_np)
    del bench
    torch.cuda.empty_cache()
    # The secondary records (single GPU only): a failure in one of them is recorded in the
    # line and does not drop the headline.
    def secondary(fn):
        try:
            return fn()
        except Exception as ex:  # noqa: BLE001 -- reported, not hidden
            return {"error": f"{type(ex).__name__}: {ex}"}

    if world == 1 and not args.no_per_workload:
        per = {}

        def one(name):
            b = Workbench(name, dev)
            k = min(K, 10 if not b.stack else 3)
            r, t_ms = measure(b, k, 3, ranks, dev, flush, stages=True, e2e=False)
            r["value"] = weak_scaling_rate(1, k, b.tokens, t_ms)
            r["unit"] = UNIT
            r["dtype"] = b.dtype
            r["config"] = _workload_config(b.wl)
            if rank == 0 and not args.no_cpu_baseline:
                r["cpu_baseline"] = cpu_baseline(b.wl, b.x_np, b.meta_np, b.ps_np, budget_s=6.0)
            return r

        for name in synth.WORKLOAD_ORDER:
            if name != args.workload:
                per[name] = secondary(lambda: one(name))
                torch.cuda.empty_cache()
        if line is not None:
            line["per_workload"] = per
    if world == 1 and not args.no_decode and line is not None:
        line["decode"] = secondary(lambda: measure_decode("hymba1p5b_kvpair", dev, flush))
        torch.cuda.empty_cache()
    if world == 1 and not args.no_per_workload and line is not None:
        # the option paths (Mamba conv + D skip, per-group branch norm, difference fusion) on
        # the 350M-shaped layer, against the same layer without them
        def options():
            opts = dict(conv_width=4, d_skip=1, norm_group=128, fusion=1)
            b = Workbench("hymba350m_layer", dev, **opts)
            r, t_ms = measure(b, min(K, 10), 3, ranks, dev, flush, stages=True, e2e=False)
            r["value"] = weak_scaling_rate(1, min(K, 10), b.tokens, t_ms)
            r["unit"] = UNIT
            r["options"] = opts
            base = line.get("per_workload", {}).get("hymba350m_layer")
            if base and "ms_per_step" in base:
                r["overhead_frac"] = round(r["ms_per_step"] / base["ms_per_step"] - 1.0, 4)
            return r
        line["options"] = secondary(options)
        torch.cuda.empty_cache()
    if line is not None:
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="hymba1p5b_kvpair", choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--no-per-workload", action="store_true", help="skip the other workloads' lines")
    ap.add_argument("--no-decode", action="store_true", help="skip the generation-step measurement")
    ap.add_argument("--only-headline", action="store_true",
                    help="the headline workload only: no other workloads, decode, options, e2e or CPU baseline "
                         "(profiling runs)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("note: fewer than 3 warm-up steps requested", file=sys.stderr)
    if args.only_headline:
        args.no_per_workload = args.no_decode = args.no_e2e = args.no_cpu_baseline = True
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_native(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
