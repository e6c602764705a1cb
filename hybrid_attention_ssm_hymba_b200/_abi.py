"""ctypes binding of the C ABI in include/hymba.h -- argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (or raw integer device pointers) and returns the C status code.  No
arithmetic of the layer happens in Python: all of it runs in the CUDA kernels
of ``libhymba.so``.  If the library is missing this module raises instead of
falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

HYMBA_OK, HYMBA_ERR_INVALID_ARG, HYMBA_ERR_UNSUPPORTED, HYMBA_ERR_WORKSPACE, HYMBA_ERR_CUDA, \
    HYMBA_ERR_TIMEOUT = range(6)
HYMBA_F32, HYMBA_BF16 = 0, 1
HYMBA_KV_OWN, HYMBA_KV_PRODUCE, HYMBA_KV_CONSUME = 0, 1, 2

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhymba.so")

# every entry point declared in include/hymba.h
ENTRY_POINTS = (
    "hymba_status_string", "hymba_workspace_size", "hymba_stack_workspace_size", "hymba_layer_fwd",
    "hymba_stack_fwd", "hymba_workspace_status", "hymba_layer_fwd_events", "hymba_gemm", "hymba_selective_scan",
    "hymba_selective_scan_dtproj_workspace_size", "hymba_selective_scan_dtproj",
    "hymba_attention", "hymba_branch_norm", "hymba_rmsnorm", "hymba_layer_fwd_noalloc", "hymba_layer_fuses_dt_proj",
    "hymba_check_wait_timeout", "hymba_decode_workspace_size", "hymba_layer_prefill", "hymba_layer_decode",
    "hymba_meta_prefix_size", "hymba_meta_prefix", "hymba_layer_fwd_prefixed",
)

# size of the library-owned scratch block behind hymba_layer_fwd_noalloc (HYMBA_NOALLOC_SCRATCH_BYTES)
HYMBA_NOALLOC_SCRATCH_BYTES = 16 << 20


class HymbaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {hymba_status_string(status)} ({status})" if what else
                         f"{hymba_status_string(status)} ({status})")


class hymba_cfg_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "seq_len", "n_meta", "d_model", "n_q_heads", "n_kv_heads", "head_dim", "window",
        "d_inner", "d_state", "n_ssm_heads", "dt_rank", "a_per_state", "kv_mode", "ffn_dim")] + [
        ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int), ("conv_width", ctypes.c_int),
        ("norm_group", ctypes.c_int), ("fusion", ctypes.c_int)]


class hymba_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt", "beta1", "beta2", "w_gate_up", "w_down",
        "norm1", "norm2", "w_conv", "b_conv", "d_skip")]


_VP, _SZ, _I, _F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_SIGS = {
    "hymba_status_string": (ctypes.c_char_p, [_I]),
    "hymba_workspace_size": (_SZ, [ctypes.POINTER(hymba_cfg_t)]),
    "hymba_layer_fuses_dt_proj": (ctypes.c_int, [ctypes.POINTER(hymba_cfg_t)]),
    "hymba_stack_workspace_size": (_SZ, [ctypes.POINTER(hymba_cfg_t), _I]),
    "hymba_layer_fwd": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                             _VP, _VP, _VP, _VP, _SZ, _VP]),
    "hymba_layer_fwd_events": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                                    _VP, _VP, _VP, _VP, _SZ, _VP, ctypes.POINTER(_VP)]),
    "hymba_layer_fwd_noalloc": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                                     _VP, _VP, _VP, _VP]),
    "hymba_stack_fwd": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                             _I, _VP, _VP, _SZ, _VP]),
    "hymba_workspace_status": (_I, [_VP, _VP]),
    "hymba_gemm": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "hymba_selective_scan": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "hymba_selective_scan_dtproj_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "hymba_selective_scan_dtproj": (_I, [_VP, _VP, _VP, _VP, _I, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP,
                                         _SZ, _VP]),
    "hymba_attention": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "hymba_branch_norm": (_I, [_VP, _VP, _VP, _I, _I, _I, _F, _I, _VP]),
    "hymba_rmsnorm": (_I, [_VP, _VP, _I, _I, _F, _I, _VP]),
    "hymba_check_wait_timeout": (_I, [_VP, _SZ, ctypes.c_uint, _VP]),
    "hymba_decode_workspace_size": (_SZ, [ctypes.POINTER(hymba_cfg_t)]),
    "hymba_meta_prefix_size": (_SZ, [ctypes.POINTER(hymba_cfg_t)]),
    "hymba_meta_prefix": (_I, [_VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t), _VP, _VP, _VP,
                               _SZ, _VP]),
    "hymba_layer_fwd_prefixed": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                                      _VP, _VP, _VP, _VP, _SZ, _VP]),
    "hymba_layer_prefill": (_I, [_VP, _VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                                 _VP, _I, _VP, _VP, _VP, _SZ, _VP]),
    "hymba_layer_decode": (_I, [_VP, ctypes.POINTER(hymba_weights_t), ctypes.POINTER(hymba_cfg_t),
                                _VP, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m hybrid_attention_ssm_hymba_b200.build` (no fallback exists)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------------------- marshalling helpers

def make_cfg(shape=None, **kw) -> hymba_cfg_t:
    """hymba_cfg_t from any object with the field names as attributes (e.g.
    synth.LayerShape, whose dtype is "bf16"/"f32") and/or keywords."""
    c = hymba_cfg_t()
    src = dict(kw)
    for f, _ in hymba_cfg_t._fields_:
        if f not in src and shape is not None and hasattr(shape, f):
            src[f] = getattr(shape, f)
    for f, _ in hymba_cfg_t._fields_:
        v = src.get(f, 0 if f != "rms_eps" else 1e-6)
        if f == "dtype" and isinstance(v, str):
            v = HYMBA_BF16 if v == "bf16" else HYMBA_F32
        setattr(c, f, v)
    return c


def make_weights(p: Dict[str, object]) -> hymba_weights_t:
    """hymba_weights_t from a dict of device tensors (keys as in hymba_weights_t)."""
    w = hymba_weights_t()
    for f, _ in hymba_weights_t._fields_:
        setattr(w, f, _ptr(p.get(f)))
    return w


# --------------------------------------------------------------------------- entry points

def hymba_status_string(status: int) -> str:
    return load().hymba_status_string(int(status)).decode()


def hymba_workspace_size(cfg: hymba_cfg_t) -> int:
    return load().hymba_workspace_size(ctypes.byref(cfg))


def hymba_layer_fuses_dt_proj(cfg: hymba_cfg_t) -> bool:
    return bool(load().hymba_layer_fuses_dt_proj(ctypes.byref(cfg)))


def hymba_stack_workspace_size(cfgs: Sequence[hymba_cfg_t]) -> int:
    arr = (hymba_cfg_t * len(cfgs))(*cfgs)
    return load().hymba_stack_workspace_size(arr, len(cfgs))


def hymba_layer_fwd(x, meta, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_in, kv_out, out,
                    workspace, ws_bytes: Optional[int] = None, stream=None) -> int:
    wsb = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    return load().hymba_layer_fwd(_ptr(x), _ptr(meta), ctypes.byref(weights), ctypes.byref(cfg),
                                  _ptr(kv_in), _ptr(kv_out), _ptr(out), _ptr(workspace), wsb,
                                  _stream(stream))


def hymba_layer_fwd_noalloc(x, meta, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_in, kv_out, out,
                            stream=None) -> int:
    """hymba_layer_fwd with the intermediates in the library's own static scratch block
    (no workspace argument; configs needing more than HYMBA_NOALLOC_SCRATCH_BYTES are
    rejected with HYMBA_ERR_WORKSPACE)."""
    return load().hymba_layer_fwd_noalloc(_ptr(x), _ptr(meta), ctypes.byref(weights), ctypes.byref(cfg),
                                          _ptr(kv_in), _ptr(kv_out), _ptr(out), _stream(stream))


STAGES = ("in_proj", "x_proj", "dt_proj", "attention", "scan", "branch_norm", "out_proj")


def hymba_layer_fwd_events(x, meta, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_in, kv_out, out,
                           workspace, events, ws_bytes: Optional[int] = None, stream=None) -> int:
    """hymba_layer_fwd recording events[i] before stage i (STAGES) and events[7] at the end;
    `events` is a sequence of 8 torch.cuda.Event (or raw cudaEvent_t ints)."""
    handles = [e if isinstance(e, int) else e.cuda_event for e in events]
    arr = (_VP * 8)(*handles)
    wsb = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    return load().hymba_layer_fwd_events(_ptr(x), _ptr(meta), ctypes.byref(weights), ctypes.byref(cfg),
                                         _ptr(kv_in), _ptr(kv_out), _ptr(out), _ptr(workspace), wsb,
                                         _stream(stream), arr)


def hymba_stack_fwd(x, meta, weights: Sequence[hymba_weights_t], cfgs: Sequence[hymba_cfg_t], out,
                    workspace, ws_bytes: Optional[int] = None, stream=None) -> int:
    n = len(cfgs)
    warr = (hymba_weights_t * n)(*weights)
    carr = (hymba_cfg_t * n)(*cfgs)
    wsb = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    return load().hymba_stack_fwd(_ptr(x), _ptr(meta), warr, carr, n, _ptr(out), _ptr(workspace), wsb,
                                  _stream(stream))


def hymba_workspace_status(workspace, stream=None) -> int:
    return load().hymba_workspace_status(_ptr(workspace), _stream(stream))


def hymba_gemm(a, w, c, M: int, N: int, K: int, dtype: int, workspace, stream=None) -> int:
    return load().hymba_gemm(_ptr(a), _ptr(w), _ptr(c), M, N, K, dtype, _ptr(workspace),
                             _nbytes(workspace), _stream(stream))


def hymba_selective_scan(x, dt, bc, gate, a_log, y, y_ld: int, batch: int, T: int, d_inner: int,
                         d_state: int, dtype: int, workspace, stream=None, a_per_state: int = 0) -> int:
    return load().hymba_selective_scan(_ptr(x), _ptr(dt), _ptr(bc), _ptr(gate), _ptr(a_log), _ptr(y),
                                       y_ld, batch, T, d_inner, d_state, int(a_per_state), dtype,
                                       _ptr(workspace), _nbytes(workspace), _stream(stream))


def hymba_selective_scan_dtproj_workspace_size(batch: int, T: int, d_inner: int, d_state: int, dt_rank: int,
                                               dtype: int) -> int:
    return load().hymba_selective_scan_dtproj_workspace_size(batch, T, d_inner, d_state, dt_rank, dtype)


def hymba_selective_scan_dtproj(x, dt_low, w_dt, b_dt, dt_rank: int, bc, gate, a_log, y, y_ld: int, batch: int,
                                T: int, d_inner: int, d_state: int, dtype: int, workspace, stream=None) -> int:
    return load().hymba_selective_scan_dtproj(_ptr(x), _ptr(dt_low), _ptr(w_dt), _ptr(b_dt), dt_rank, _ptr(bc),
                                              _ptr(gate), _ptr(a_log), _ptr(y), y_ld, batch, T, d_inner, d_state,
                                              dtype, _ptr(workspace), _nbytes(workspace), _stream(stream))


def hymba_attention(q, kv, out, out_ld: int, batch: int, T: int, n_q_heads: int, n_kv_heads: int,
                    head_dim: int, n_meta: int, window: int, dtype: int, workspace, stream=None) -> int:
    return load().hymba_attention(_ptr(q), _ptr(kv), _ptr(out), out_ld, batch, T, n_q_heads, n_kv_heads,
                                  head_dim, n_meta, window, dtype, _ptr(workspace), _nbytes(workspace),
                                  _stream(stream))


def hymba_branch_norm(z, beta1, beta2, rows: int, w_attn: int, w_ssm: int, eps: float, dtype: int,
                      stream=None) -> int:
    return load().hymba_branch_norm(_ptr(z), _ptr(beta1), _ptr(beta2), rows, w_attn, w_ssm, eps, dtype,
                                    _stream(stream))


def hymba_rmsnorm(x, y, rows: int, d: int, eps: float, dtype: int, stream=None) -> int:
    return load().hymba_rmsnorm(_ptr(x), _ptr(y), rows, d, eps, dtype, _stream(stream))


def hymba_meta_prefix_size(cfg: hymba_cfg_t) -> int:
    return load().hymba_meta_prefix_size(ctypes.byref(cfg))


def hymba_meta_prefix(meta_in, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_prefix_in, prefix, workspace,
                      stream=None) -> int:
    return load().hymba_meta_prefix(_ptr(meta_in), ctypes.byref(weights), ctypes.byref(cfg), _ptr(kv_prefix_in),
                                    _ptr(prefix), _ptr(workspace), _nbytes(workspace), _stream(stream))


def hymba_layer_fwd_prefixed(x, prefix, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_in, kv_out, out,
                             workspace, stream=None) -> int:
    return load().hymba_layer_fwd_prefixed(_ptr(x), _ptr(prefix), ctypes.byref(weights), ctypes.byref(cfg),
                                           _ptr(kv_in), _ptr(kv_out), _ptr(out), _ptr(workspace),
                                           _nbytes(workspace), _stream(stream))


def hymba_decode_workspace_size(cfg: hymba_cfg_t) -> int:
    return load().hymba_decode_workspace_size(ctypes.byref(cfg))


def hymba_layer_prefill(x, meta, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_cache, cache_rows: int,
                        ssm_state, out, workspace, stream=None) -> int:
    return load().hymba_layer_prefill(_ptr(x), _ptr(meta), ctypes.byref(weights), ctypes.byref(cfg),
                                      _ptr(kv_cache), int(cache_rows), _ptr(ssm_state), _ptr(out),
                                      _ptr(workspace), _nbytes(workspace), _stream(stream))


def hymba_layer_decode(x_t, weights: hymba_weights_t, cfg: hymba_cfg_t, kv_cache, cache_rows: int, pos: int,
                       ssm_state, out_t, workspace, stream=None) -> int:
    return load().hymba_layer_decode(_ptr(x_t), ctypes.byref(weights), ctypes.byref(cfg), _ptr(kv_cache),
                                     int(cache_rows), int(pos), _ptr(ssm_state), _ptr(out_t), _ptr(workspace),
                                     _nbytes(workspace), _stream(stream))


def hymba_check_wait_timeout(workspace, limit_us: int, stream=None) -> int:
    """Runs the bounded-wait failure path once (a wait that nothing ends, limited to
    limit_us); the workspace's status word then reads HYMBA_ERR_TIMEOUT."""
    return load().hymba_check_wait_timeout(_ptr(workspace), _nbytes(workspace), int(limit_us), _stream(stream))


def check(status: int, what: str = "") -> None:
    """Raise HymbaError unless status is HYMBA_OK."""
    if status != HYMBA_OK:
        raise HymbaError(status, what)
