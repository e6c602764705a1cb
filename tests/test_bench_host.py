"""The bench's per-stage work accounting (host logic, CPU).

bench.py reports each stage's achieved rate against its roofline from stage_work(): the
algorithmic FLOPs and HBM bytes of one launch.  These checks pin that accounting to the
shapes: the visible-pair count against brute-force enumeration of the attention mask,
the contraction FLOPs against 2·K·N per row, and the dt projection moving into the scan
(its FLOPs move, its bytes change by exactly the dt round trip it saves)."""
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
