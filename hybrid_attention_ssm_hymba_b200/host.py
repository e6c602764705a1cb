"""Host-side helpers around the binding: move seeded arrays to the GPU in the
layer's dtype and allocate caller-owned buffers (the library allocates
nothing).  Plumbing only -- no arithmetic of the layer."""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch

from . import _abi

FP32_KEYS = ("a_log", "b_dt", "beta1", "beta2", "norm1", "norm2", "b_conv", "d_skip")


def torch_dtype(dtype: str) -> torch.dtype:
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_device(a: np.ndarray, dtype: str, device="cuda", pin: bool = False) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch_dtype(dtype))
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device, non_blocking=False)


def params_to_device(p: Dict[str, np.ndarray], dtype: str, device="cuda") -> Dict[str, torch.Tensor]:
    """Projection weights in the layer's dtype; a_log, b_dt, beta1, beta2 (and the pre-norm
    gains norm1, norm2) in fp32."""
    return {k: to_device(v, "f32" if k in FP32_KEYS else dtype, device) for k, v in p.items()}


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device buffer of at least nbytes (torch allocations are)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def empty(shape, dtype: str, device="cuda") -> torch.Tensor:
    return torch.empty(shape, dtype=torch_dtype(dtype), device=device)


def run_layer(x, meta, dev_params, cfg, kv_in=None, kv_out=None, out=None, ws=None, stream=None):
    """Convenience wrapper: allocates `out` / workspace if not given, calls
    hymba_layer_fwd and raises on a non-OK status."""
    T = cfg.seq_len + cfg.n_meta
    if out is None:
        out = torch.empty((cfg.batch, T, cfg.d_model), dtype=x.dtype, device=x.device)
    if ws is None:
        ws = workspace(_abi.hymba_workspace_size(cfg), x.device)
    w = _abi.make_weights(dev_params)
    _abi.check(_abi.hymba_layer_fwd(x, meta, w, cfg, kv_in, kv_out, out, ws, stream=stream),
               "hymba_layer_fwd")
    return out
