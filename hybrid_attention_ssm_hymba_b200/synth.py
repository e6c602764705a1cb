"""Seeded synthetic workloads for the Hymba hybrid-head layer.

This module only draws random numbers and describes shapes.  It holds none of
the layer's arithmetic, imports nothing else from this package, and is the one
piece of code that both the CUDA path (through the tests and the bench) and the
fp64 oracle are fed from, so that both see bit-identical inputs.

Workloads (named by what they are):

* ``tiny_fp32``         B=1,  L=64    + 8 meta,   d=128,  fp32, global attention
* ``hymba350m_layer``   B=8,  L=2048  + 32 meta,  d=1024, bf16, global, GQA 2/1, N=16
* ``hymba1p5b_kvpair``  B=4,  L=8192  + 128 meta, d=2048, bf16, SWA 1024 + meta,
                        GQA 16/4, N=128, two layers sharing one K/V
* ``longctx_32k``       B=1,  L=32768 + 128 meta, d=1536, bf16, SWA 1024, N=128,
                        dt drawn down to 1e-4
* ``hymba1p5b_stack24`` 24 blocks, B=8, L=4096 + 128 meta, d=2048, SwiGLU FFN
                        5632, global in blocks {0, 11, 23}, SWA 1024 elsewhere,
                        adjacent blocks share K/V, N=16

Distributions (the same for every workload unless noted): X and meta ~ N(0,1);
every projection weight ~ N(0, 0.02); A_log ~ U(log 1, log 16); dt0 ~ U(dt_min,
0.1) per channel with b_dt the inverse softplus of dt0; beta1, beta2 = 1 for the
fp32 workload and ~ U(0.5, 1.5) otherwise.  Every tensor has its own
counter-free PCG64 stream keyed by (seed, layer, tensor id).  For bf16
workloads every tensor is rounded to bf16 (round to nearest even) once, here, so
the values handed to the oracle are exactly the values the GPU reads.
"""
from __future__ import annotations

import copy
import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

# Fixed per-tensor stream ids.  Never renumber: they define the workloads.
_STREAM = {
    "x": 1, "meta": 2,
    "w_in": 10, "w_x": 11, "w_dt": 12, "w_out": 13, "a_log": 14, "dt0": 15,
    "beta1": 16, "beta2": 17, "w_gate_up": 18, "w_down": 19, "norm1": 20, "norm2": 21,
    "w_conv": 22, "b_conv": 23, "d_skip": 24,
    # free-standing stage inputs used by the per-kernel tests
    "s_x": 40, "s_dt": 41, "s_bc": 42, "s_g": 43, "s_q": 44, "s_kv": 45,
    "s_z": 46, "s_a": 47, "s_w": 48, "s_dl": 49, "s_wd": 50, "s_bd": 51,
}

# kv_mode values (match hymba_kv_mode_t in include/hymba.h)
KV_OWN, KV_PRODUCE, KV_CONSUME = 0, 1, 2


@dataclasses.dataclass
class LayerShape:
    """Shapes of one hybrid-head layer (plus its FFN when ffn_dim > 0)."""
    batch: int
    seq_len: int          # L, user tokens
    n_meta: int           # M
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int           # -1 = global causal
    d_inner: int
    d_state: int
    n_ssm_heads: int
    dt_rank: int
    kv_mode: int = KV_OWN
    ffn_dim: int = 0
    a_per_state: int = 0
    rms_eps: float = 1e-6
    dtype: str = "bf16"   # "bf16" or "f32"
    conv_width: int = 0   # Mamba option: causal depthwise conv of this width + SiLU on X_ssm
    d_skip: int = 0       # Mamba option: 1 = the SSM output gets D * x before the gate
    norm_group: int = 0   # branch norm per group of this many features (0: whole branch)
    fusion: int = 0       # 0: sum of the branches; 1: difference (SSM branch subtracted)

    @property
    def T(self) -> int:
        return self.seq_len + self.n_meta

    @property
    def attn_width(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_width(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def n_in(self) -> int:
        kv = 0 if self.kv_mode == KV_CONSUME else 2 * self.kv_width
        return self.attn_width + kv + 2 * self.d_inner

    @property
    def xproj_width(self) -> int:
        return self.dt_rank + 2 * self.d_state


@dataclasses.dataclass
class Workload:
    name: str
    layers: List[LayerShape]
    seed: int
    dt_min: float
    beta_ones: bool
    description: str

    @property
    def first(self) -> LayerShape:
        return self.layers[0]

    def user_tokens(self) -> int:
        s = self.first
        return s.batch * s.seq_len


def _layer(**kw) -> LayerShape:
    return LayerShape(**kw)


def _make_workloads() -> Dict[str, Workload]:
    w: Dict[str, Workload] = {}
    w["tiny_fp32"] = Workload(
        "tiny_fp32",
        [_layer(batch=1, seq_len=64, n_meta=8, d_model=128, n_q_heads=2, n_kv_heads=2,
                head_dim=32, window=-1, d_inner=256, d_state=16, n_ssm_heads=2, dt_rank=8,
                dtype="f32")],
        seed=0, dt_min=1e-3, beta_ones=True,
        description="tiny fp32 hybrid-head layer, B1 L64+8 meta d128")
    w["hymba350m_layer"] = Workload(
        "hymba350m_layer",
        [_layer(batch=8, seq_len=2048, n_meta=32, d_model=1024, n_q_heads=2, n_kv_heads=1,
                head_dim=128, window=-1, d_inner=2048, d_state=16, n_ssm_heads=10, dt_rank=64)],
        seed=1, dt_min=1e-3, beta_ones=False,
        description="Hymba-350M-shaped layer, B8 L2048+32 meta d1024, bf16")
    prod = _layer(batch=4, seq_len=8192, n_meta=128, d_model=2048, n_q_heads=16, n_kv_heads=4,
                  head_dim=128, window=1024, d_inner=4096, d_state=128, n_ssm_heads=16,
                  dt_rank=128, kv_mode=KV_PRODUCE)
    cons = dataclasses.replace(prod, kv_mode=KV_CONSUME)
    w["hymba1p5b_kvpair"] = Workload(
        "hymba1p5b_kvpair", [prod, cons], seed=2, dt_min=1e-3, beta_ones=False,
        description="Hymba-1.5B-shaped producer+consumer layer pair sharing K/V, "
                    "B4 L8192+128 meta d2048, SWA 1024, bf16")
    w["longctx_32k"] = Workload(
        "longctx_32k",
        [_layer(batch=1, seq_len=32768, n_meta=128, d_model=1536, n_q_heads=12, n_kv_heads=2,
                head_dim=128, window=1024, d_inner=3072, d_state=128, n_ssm_heads=14,
                dt_rank=96)],
        seed=3, dt_min=1e-4, beta_ones=False,
        description="long-context layer, B1 L32768+128 meta d1536, SWA 1024, bf16")
    layers = []
    for i in range(24):
        layers.append(_layer(
            batch=8, seq_len=4096, n_meta=128, d_model=2048, n_q_heads=16, n_kv_heads=4,
            head_dim=128, window=-1 if i in (0, 11, 23) else 1024, d_inner=4096, d_state=16,
            n_ssm_heads=16, dt_rank=128, kv_mode=KV_PRODUCE if i % 2 == 0 else KV_CONSUME,
            ffn_dim=5632))
    w["hymba1p5b_stack24"] = Workload(
        "hymba1p5b_stack24", layers, seed=4, dt_min=1e-3, beta_ones=False,
        description="24-block Hymba-1.5B-shaped stack, B8 L4096+128 meta d2048, FFN 5632, bf16")
    return w


WORKLOADS: Dict[str, Workload] = _make_workloads()
WORKLOAD_ORDER = ["tiny_fp32", "hymba350m_layer", "hymba1p5b_kvpair", "longctx_32k",
                  "hymba1p5b_stack24"]


def workload(name: str, **overrides) -> Workload:
    """A copy of a named workload; keyword overrides apply to every layer
    (``batch``, ``seq_len``, ...).  ``n_layers`` truncates a stack."""
    wl = copy.deepcopy(WORKLOADS[name])
    n_layers = overrides.pop("n_layers", None)
    if n_layers is not None:
        wl.layers = wl.layers[:n_layers]
    if overrides:
        wl.layers = [dataclasses.replace(s, **overrides) for s in wl.layers]
    return wl


# ---------------------------------------------------------------------------
# random streams

def rng(seed: int, layer: int, tensor: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, _STREAM[tensor]])))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    nan = np.isnan(a)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    out = u.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return round_bf16(a) if dtype == "bf16" else a


def normal(seed, layer, tensor, shape, std=1.0, dtype="bf16") -> np.ndarray:
    g = rng(seed, layer, tensor)
    return _finish(g.standard_normal(size=shape, dtype=np.float32) * np.float32(std), dtype)


def uniform(seed, layer, tensor, shape, lo, hi, dtype="f32") -> np.ndarray:
    g = rng(seed, layer, tensor)
    return _finish(g.uniform(lo, hi, size=shape), dtype)


def inverse_softplus(y: np.ndarray) -> np.ndarray:
    """Initialisation recipe for b_dt: the value whose softplus is y."""
    y = y.astype(np.float64)
    return (y + np.log(-np.expm1(-y))).astype(np.float32)


def layer_inputs(wl: Workload, batch: Optional[int] = None, seq_len: Optional[int] = None):
    """x [B, L, d] and meta [M, d] (float32 arrays, bf16-exact for bf16 workloads).

    ``seq_len`` < L gives the exact prefix of the full draw (rows are drawn
    row-major per batch element), ``batch`` < B the leading batch elements."""
    s = wl.first
    B = s.batch if batch is None else batch
    L = s.seq_len if seq_len is None else seq_len
    # drawn per batch element (the same stream order as one [B, L, d] draw), so
    # that a shorter seq_len or batch gives the exact prefix of the full draw
    g = rng(wl.seed, 0, "x")
    rows = []
    for b in range(B):
        xb = g.standard_normal(size=(s.seq_len, s.d_model), dtype=np.float32)
        rows.append(xb[:L])
    full = _finish(np.stack(rows), s.dtype)
    meta = normal(wl.seed, 0, "meta", (s.n_meta, s.d_model), 1.0, s.dtype)
    return full, meta


def layer_params(wl: Workload, layer: int, norm_gains: bool = False) -> Dict[str, np.ndarray]:
    """Weights of one layer, as float32 arrays (bf16-exact for bf16 workloads).

    Layouts (row-major, nn.Linear convention [out_features, in_features]):
      w_in  [N_in, d]   rows ordered W_Q, W_K, W_V, W_SSM, W_G (no W_K/W_V rows
                        for a K/V-consuming layer)
      w_x   [R + 2N, Di]  rows ordered dt_low, B, C
      w_dt  [Di, R]
      w_out [d, Hq*dh + Di]
      a_log [Di] (or [Di, N] when a_per_state), b_dt [Di], beta1 [Hq*dh], beta2 [Di]: fp32
      w_gate_up [2F, d] (gate rows then up rows), w_down [d, F]   (ffn_dim > 0)
      w_conv [Di, K] (dtype), b_conv [Di] fp32 ~ U(+-1/sqrt(K)): with conv_width = K
      d_skip [Di] fp32 ~ U(0.5, 1.5): with d_skip
      norm1, norm2 [d] fp32 ~ U(0.5, 1.5): the stacked block's pre-norm gains, only with
                        norm_gains (the workloads use unit gains, their initial value)
    """
    s = wl.layers[layer]
    sd, dt = wl.seed, s.dtype
    p = {
        "w_in": normal(sd, layer, "w_in", (s.n_in, s.d_model), 0.02, dt),
        "w_x": normal(sd, layer, "w_x", (s.xproj_width, s.d_inner), 0.02, dt),
        "w_dt": normal(sd, layer, "w_dt", (s.d_inner, s.dt_rank), 0.02, dt),
        "w_out": normal(sd, layer, "w_out", (s.d_model, s.attn_width + s.d_inner), 0.02, dt),
    }
    a_shape = (s.d_inner, s.d_state) if s.a_per_state else (s.d_inner,)
    p["a_log"] = uniform(sd, layer, "a_log", a_shape, 0.0, math.log(16.0))
    dt0 = uniform(sd, layer, "dt0", (s.d_inner,), wl.dt_min, 0.1)
    p["b_dt"] = inverse_softplus(dt0)
    if wl.beta_ones:
        p["beta1"] = np.ones(s.attn_width, np.float32)
        p["beta2"] = np.ones(s.d_inner, np.float32)
    else:
        p["beta1"] = uniform(sd, layer, "beta1", (s.attn_width,), 0.5, 1.5)
        p["beta2"] = uniform(sd, layer, "beta2", (s.d_inner,), 0.5, 1.5)
    if s.ffn_dim:
        p["w_gate_up"] = normal(sd, layer, "w_gate_up", (2 * s.ffn_dim, s.d_model), 0.02, dt)
        p["w_down"] = normal(sd, layer, "w_down", (s.d_model, s.ffn_dim), 0.02, dt)
    if s.conv_width:   # the default init of a depthwise Conv1d: U(-1/sqrt(K), 1/sqrt(K))
        bound = 1.0 / math.sqrt(s.conv_width)
        p["w_conv"] = uniform(sd, layer, "w_conv", (s.d_inner, s.conv_width), -bound, bound, dt)
        p["b_conv"] = uniform(sd, layer, "b_conv", (s.d_inner,), -bound, bound)
    if s.d_skip:
        p["d_skip"] = uniform(sd, layer, "d_skip", (s.d_inner,), 0.5, 1.5)
    if norm_gains:
        p["norm1"] = uniform(sd, layer, "norm1", (s.d_model,), 0.5, 1.5)
        p["norm2"] = uniform(sd, layer, "norm2", (s.d_model,), 0.5, 1.5)
    return p


# ---------------------------------------------------------------------------
# free-standing stage inputs (per-kernel parity tests)

def scan_inputs(seed: int, B: int, T: int, Di: int, N: int, dt_min=1e-3, dtype="bf16",
                a_per_state=False):
    """Inputs in the layouts the scan stage reads: x, dt, g [B*T, Di] (dt already
    positive, drawn log-uniform in [dt_min, 0.15]); bc [B*T, 2N] fp32 (B then C);
    a_log [Di] fp32."""
    x = normal(seed, 0, "s_x", (B * T, Di), 0.6, dtype)
    g = rng(seed, 0, "s_dt")
    dt = np.exp(g.uniform(math.log(dt_min), math.log(0.15), size=(B * T, Di))).astype(np.float32)
    dt = _finish(dt, dtype)
    bc = normal(seed, 0, "s_bc", (B * T, 2 * N), 0.6, "f32")
    gate = normal(seed, 0, "s_g", (B * T, Di), 0.5, dtype)
    a_shape = (Di, N) if a_per_state else (Di,)
    a_log = uniform(seed, 0, "s_a", a_shape, 0.0, math.log(16.0))
    return dict(x=x, dt=dt, bc=bc, g=gate, a_log=a_log)


def scan_dtproj_inputs(seed: int, B: int, T: int, Di: int, N: int, R: int, dt_min=1e-3, dtype="bf16"):
    """scan_inputs with dt given through its low-rank projection, as the layer forms it:
    dt_low [B*T, R] ~ N(0, 0.5) (dtype), w_dt [Di, R] ~ N(0, 0.02) (dtype), b_dt [Di] fp32
    the inverse softplus of dt0 ~ U(dt_min, 0.1).  No dt entry."""
    d = scan_inputs(seed, B, T, Di, N, dt_min=dt_min, dtype=dtype)
    del d["dt"]
    d["dt_low"] = normal(seed, 0, "s_dl", (B * T, R), 0.5, dtype)
    d["w_dt"] = normal(seed, 0, "s_wd", (Di, R), 0.02, dtype)
    d["b_dt"] = inverse_softplus(uniform(seed, 0, "s_bd", (Di,), dt_min, 0.1)).astype(np.float32)
    return d


def attention_inputs(seed: int, B: int, T: int, Hq: int, Hkv: int, dh: int, dtype="bf16",
                     std=0.64):
    """q [B*T, Hq*dh]; kv [2, B*T, Hkv*dh] (K then V)."""
    q = normal(seed, 0, "s_q", (B * T, Hq * dh), std, dtype)
    kv = normal(seed, 0, "s_kv", (2, B * T, Hkv * dh), std, dtype)
    return q, kv


def matrix(seed: int, tensor: str, shape, std=1.0, dtype="bf16") -> np.ndarray:
    return normal(seed, 0, tensor, shape, std, dtype)
