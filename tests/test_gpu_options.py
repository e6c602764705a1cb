"""Option paths of the layer on the GPU through the C ABI, against the oracle.

Mamba options of the SSM head (the pages print neither): the causal depthwise conv +
SiLU on X_ssm (conv_width) and the D skip (weights d_skip).  Fusion variants of the
intra-layer hybrid study: the branch norm per group of features (norm_group) and
difference fusion (fusion = 1).  Each alone and together, in the tensor-core scan
(d_state 16) and the CUDA-core scan (d_state 128), bf16 and fp32, and the generation
step with the options it supports."""
import dataclasses

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
import oracle as O
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]

SMALL_PAIR = dict(batch=2, seq_len=300, window=64, d_model=512, n_q_heads=8, n_kv_heads=2, d_inner=512,
                  dt_rank=32)


def _layer(wl):
    s = dataclasses.replace(wl.first, kv_mode=H.HYMBA_KV_OWN)
    wl.layers = [s]
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    dp = host.params_to_device(p, s.dtype)
    cfg = H.make_cfg(s)
    ws = host.workspace(H.hymba_workspace_size(cfg))
    out = host.empty((s.batch, s.T, s.d_model), s.dtype)
    H.check(H.hymba_layer_fwd(dev(x, s.dtype), dev(meta, s.dtype), H.make_weights(dp), cfg, None, None, out, ws),
            "layer")
    status_ok(ws)
    ref, _ = O.layer_forward(x, meta, p, s)
    return to_np(out), ref, s


@pytest.mark.parametrize("opts", [dict(conv_width=4), dict(d_skip=1), dict(conv_width=4, d_skip=1),
                                  dict(norm_group=128), dict(fusion=1), dict(norm_group=128, fusion=1),
                                  dict(conv_width=3, d_skip=1, norm_group=64, fusion=1)])
def test_options_hymba350m_shaped(opts):
    g, ref, s = _layer(synth.workload("hymba350m_layer", batch=2, seq_len=300, **opts))
    assert_close(g, ref, "bf16", f"350M-shaped layer {opts}")


@pytest.mark.parametrize("opts", [dict(conv_width=4, d_skip=1), dict(norm_group=256, fusion=1)])
def test_options_dstate128_swa(opts):
    g, ref, s = _layer(synth.workload("hymba1p5b_kvpair", **SMALL_PAIR, **opts))
    assert_close(g, ref, "bf16", f"d_state 128 layer {opts}")


@pytest.mark.parametrize("opts", [dict(conv_width=2, d_skip=1), dict(norm_group=64, fusion=1),
                                  dict(conv_width=4, d_skip=1, norm_group=64, fusion=1, a_per_state=1)])
def test_options_fp32(opts):
    g, ref, s = _layer(synth.workload("tiny_fp32", batch=2, **opts))
    assert_close(g, ref, "f32", f"fp32 layer {opts}")


def test_options_full_size_350m_layer_every_option():
    """The 350M-shaped workload at full size with every option on; sequences 0 and 7 in full."""
    wl = synth.workload("hymba350m_layer", conv_width=4, d_skip=1, norm_group=128, fusion=1)
    s = wl.first
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    dp = host.params_to_device(p, "bf16")
    cfg = H.make_cfg(s)
    ws = host.workspace(H.hymba_workspace_size(cfg))
    out = host.empty((s.batch, s.T, s.d_model), "bf16")
    H.check(H.hymba_layer_fwd(dev(x, "bf16"), dev(meta, "bf16"), H.make_weights(dp), cfg, None, None, out, ws), "l")
    status_ok(ws)
    g = to_np(out)
    for b in (0, 7):
        ref, _ = O.layer_forward(x[b:b + 1], meta, p, dataclasses.replace(s, batch=1))
        assert_close(g[b], ref[0], "bf16", f"sequence {b}")


@pytest.mark.parametrize("name,kw", [("hymba350m_layer", dict(batch=2, seq_len=200)),
                                     ("tiny_fp32", dict(batch=2))])
def test_decode_with_skip_group_norm_difference(name, kw):
    wl = synth.workload(name, d_skip=1, norm_group=64, fusion=1, **kw)
    s = wl.first
    dt = s.dtype
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    dp = host.params_to_device(p, dt)
    cfg = H.make_cfg(s)
    cap = s.T + 3
    ws = host.workspace(H.hymba_decode_workspace_size(cfg))
    cache = host.empty((2, s.batch, cap, s.kv_width), dt)
    state = torch.empty((s.batch, s.d_inner, s.d_state), dtype=torch.float32, device="cuda")
    out = host.empty((s.batch, s.T, s.d_model), dt)
    W = H.make_weights(dp)
    H.check(H.hymba_layer_prefill(dev(x, dt), dev(meta, dt), W, cfg, cache, cap, state, out, ws), "prefill")
    ref, kv, h = O.layer_prefill_state(x, meta, p, s)
    assert_close(to_np(out), ref, dt, "prefill")
    for step in range(3):
        xt = synth.normal(wl.seed, 200 + step, "x", (s.batch, s.d_model), 1.0, dt)
        ot = host.empty((s.batch, s.d_model), dt)
        H.check(H.hymba_layer_decode(dev(xt, dt), W, cfg, cache, cap, s.T + step, state, ot, ws), "decode")
        r, kv, h = O.layer_decode_step(xt, p, s, kv, h, s.T + step)
        assert_close(to_np(ot), r, dt, f"decode step {step}")
    status_ok(ws)


def test_conv_is_rejected_where_no_state_is_carried():
    s = synth.workload("hymba350m_layer", batch=1, seq_len=64, conv_width=4).first
    cfg = H.make_cfg(s)
    assert H.hymba_decode_workspace_size(cfg) == 0
    assert H.hymba_meta_prefix_size(cfg) > 0
    dummy = host.workspace(1 << 20)
    w = H.make_weights(host.params_to_device(synth.layer_params(synth.workload("hymba350m_layer", batch=1,
                                                                               seq_len=64, conv_width=4), 0), "bf16"))
    assert H.hymba_layer_fwd_prefixed(dummy, dummy, w, cfg, None, None, dummy, dummy) == H.HYMBA_ERR_UNSUPPORTED
