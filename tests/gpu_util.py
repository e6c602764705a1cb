"""Shared helpers of the GPU parity tests: tolerances, device upload, oracle calls."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
from hybrid_attention_ssm_hymba_b200 import host

requires_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

# Acceptance: fp32 path |g - o| <= 1e-4 max(1, |o|) per element; bf16 path
# max|g - o| / max|o| <= 2e-2 per output tensor (fp32 accumulation and scan state).
F32_TOL = 1e-4
BF16_TOL = 2e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_max_err(g, o) -> float:
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


def assert_close(g, o, dtype: str, what: str = "", tol: float = None):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    assert g.shape == o.shape, f"{what}: shape {g.shape} vs {o.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    if dtype == "f32":
        t = F32_TOL if tol is None else tol
        bad = np.abs(g - o) > t * np.maximum(1.0, np.abs(o))
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond {t}; worst "
                               f"{float((np.abs(g - o) / np.maximum(1.0, np.abs(o))).max()):.3e}")
    else:
        t = BF16_TOL if tol is None else tol
        e = rel_max_err(g, o)
        assert e <= t, f"{what}: max|g-o|/max|o| = {e:.3e} > {t}"


def status_ok(ws):
    s = H.hymba_workspace_status(ws)
    assert s == H.HYMBA_OK, f"device status: {H.hymba_status_string(s)}"


def dev(a, dtype):
    return host.to_device(a, dtype)


def fp32(a):
    return host.to_device(a, "f32")
