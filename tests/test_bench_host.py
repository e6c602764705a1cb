"""The bench's per-stage work accounting (host logic, CPU).

bench.py reports each stage's achieved rate against its roofline from stage_work(): the
algorithmic FLOPs and HBM bytes of one launch.  These checks pin that accounting to the
shapes: the visible-pair count against brute-force enumeration of the attention mask,
the contraction FLOPs against 2·K·N per row, and the dt projection moving into the scan
(its FLOPs move, its bytes change by exactly the dt round trip it saves)."""
import dataclasses
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from hybrid_attention_ssm_hymba_b200 import synth  # noqa: E402


@pytest.mark.parametrize("T,M,W", [(7, 0, -1), (13, 3, -1), (20, 4, 5), (33, 8, 0), (40, 0, 100), (64, 16, 9)])
def test_visible_pairs_match_the_mask(T, M, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = (j <= i) & ((W < 0) | (i - j <= W) | (j < M))
    assert bench._visible_pairs(T, M, W) == int(vis.sum())


def test_contraction_flops_are_two_k_n_per_row():
    s = synth.workload("hymba350m_layer").first
    w = bench.stage_work(s)
    rows = s.batch * s.T
    assert w["in_proj"][0] == 2.0 * s.d_model * s.n_in * rows
    assert w["x_proj"][0] == 2.0 * s.d_inner * s.xproj_width * rows
    assert w["dt_proj"][0] == 2.0 * s.dt_rank * s.d_inner * rows
    assert w["out_proj"][0] == 2.0 * (s.attn_width + s.d_inner) * s.d_model * rows


def test_dt_projection_moves_into_the_scan():
    s = synth.workload("hymba350m_layer").first
    plain, fused = bench.stage_work(s), bench.stage_work(s, dt_in_scan=True)
    assert "dt_proj" not in fused and set(fused) | {"dt_proj"} == set(plain)
    for k in fused:
        if k != "scan":
            assert fused[k] == plain[k]
    assert fused["scan"][0] == plain["scan"][0] + plain["dt_proj"][0]
    es, rows = 2, s.batch * s.T
    # the scan no longer reads dt; it reads dt_low, W_dt and b_dt instead, and dt is never written
    saved = es * rows * s.d_inner
    added = es * (rows * s.dt_rank + s.d_inner * s.dt_rank) + 4 * s.d_inner
    assert fused["scan"][1] == plain["scan"][1] - saved + added
    total_plain = sum(b for _, b in plain.values())
    total_fused = sum(b for _, b in fused.values())
    assert total_plain - total_fused == 2 * saved   # dt written once and read once


def test_stage_rooflines_sum_layers_and_pick_the_binding_resource():
    """The layer pair's stages add over both layers; the CUDA-core scan (here d_state 128
    with one decay per state, which has no tensor-core form) is held to the fp32 FMA peak,
    the tensor-core ones (d_state 16, and 128 with one decay per channel) to HBM; the
    workload's roofline time is the sum over stages and layers of the slowest term."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    wl = synth.workload("hymba1p5b_kvpair", a_per_state=True)
    fused = [False, False]
    names = list(bench.stage_work(wl.layers[0]).keys())
    us = {k: 100.0 for k in names}
    roof, t_us = bench.stage_rooflines(wl.layers, us, peaks, fused, 1965)
    assert roof["scan"]["bound"] == "alu" and roof["attention"]["bound"] == "tensor"
    fl0, _ = bench.stage_work(wl.layers[0])["in_proj"]
    fl1, _ = bench.stage_work(wl.layers[1])["in_proj"]
    assert roof["in_proj"]["work"] == fl0 + fl1 and fl1 < fl0   # the consumer has no K/V rows
    alu = 148 * 128 * 2 * 1965e6
    exp = 0.0
    for s in wl.layers:
        for k, (fl, by) in bench.stage_work(s).items():
            b = bench.stage_bound(k, s, (fl, by), peaks)
            exp += max(fl / 1600e12 if b == "tensor" else 0.0, by / 6000e9, fl / alu if b == "alu" else 0.0)
    assert abs(t_us - exp * 1e6) < 1e-6 * t_us
    s16 = synth.workload("hymba350m_layer").first
    assert bench.stage_bound("scan", s16) == "hbm" and bench.scan_kernel_name(s16).startswith("scan_tc_kernel")
    s128 = synth.workload("hymba1p5b_kvpair").first
    assert bench.stage_bound("scan", s128) == "hbm" and bench.scan_kernel_name(s128).startswith("scan_tc128")
    assert bench.scan_kernel_name(dataclasses.replace(s128, dt_rank=136)).startswith("scan_w")


def test_stack_roofline_counts_the_ffn():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    wl = synth.workload("hymba1p5b_stack24", n_layers=2)
    with_ffn = bench.stack_roofline_us(wl.layers, peaks, [False, False])
    no_ffn = bench.stack_roofline_us([dataclasses.replace(s, ffn_dim=0) for s in wl.layers], peaks, [False, False])
    fl, _ = bench.ffn_work(wl.layers[0])
    assert fl == 6.0 * 2048 * 5632 * wl.first.batch * wl.first.T
    assert with_ffn - no_ffn >= 2 * fl / 1600e12 * 1e6 * 0.999


def test_gemm_stage_bound_is_the_longer_of_flop_and_byte_time():
    """x_proj of the 1.5B pair (N = 128 + 2 x 128) is FLOP-bound at these peaks; a GEMM
    whose bytes dominate is held to HBM; with no work given a GEMM counts as tensor."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0}
    s = synth.workload("hymba1p5b_kvpair").first
    fl, by = bench.stage_work(s)["x_proj"]
    assert fl / 1600e12 > by / 6000e9
    assert bench.stage_bound("x_proj", s, (fl, by), peaks) == "tensor"
    assert bench.stage_bound("x_proj", s, (fl, 1e3 * by), peaks) == "hbm"
    assert bench.stage_bound("out_proj", s) == "tensor"
