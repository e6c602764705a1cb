"""The generation step on the GPU through the C ABI, against the oracle's.

hymba_layer_prefill runs the prompt and leaves the K/V cache and the SSM state;
hymba_layer_decode then takes one new token per sequence per call.  Each step's output,
and the state and cache the prefill leaves, are compared with oracle.layer_prefill_state
and oracle.layer_decode_step (pinned on the CPU against the longer prefill they must
reproduce).  Cases: the 350M-shaped layer (global attention, GQA, d_state 16); a
1.5B-shaped KV-sharing pair shrunk in width, with a window shorter than the history and
meta rows that stay visible, d_state 128 (the consumer reads the producer's cache); the
fp32 path, also with one decay per channel and state."""
import dataclasses

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
import oracle as O
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]

STEPS = 4


def _tokens(wl, step):
    s = wl.first
    return synth.normal(wl.seed, 100 + step, "x", (s.batch, s.d_model), 1.0, s.dtype)


def _run(wl, norm_tol=None):
    layers = wl.layers
    s0 = layers[0]
    dtype = s0.dtype
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(len(layers))]
    dps = [host.params_to_device(p, dtype) for p in ps]
    cfgs = [H.make_cfg(s) for s in layers]
    T = s0.T
    cap = T + STEPS + 3
    ws = host.workspace(max(H.hymba_decode_workspace_size(c) for c in cfgs))
    cache = host.empty((2, s0.batch, cap, s0.kv_width), dtype)
    cache.fill_(float("nan"))     # rows past pos must never be read
    states = [torch.full((s0.batch, s.d_inner, s.d_state), float("nan"), dtype=torch.float32, device="cuda")
              for s in layers]
    # prefill: the producer (or own-K/V layer) fills the cache; a consumer reads it
    outs = []
    inp, inp_meta = dev(x, dtype), dev(meta, dtype)
    for i, (c, s) in enumerate(zip(cfgs, layers)):
        out = host.empty((s0.batch, T, s0.d_model), dtype)
        H.check(H.hymba_layer_prefill(inp, inp_meta, H.make_weights(dps[i]), c, cache, cap, states[i], out, ws),
                f"prefill layer {i}")
        outs.append(out)
        inp, inp_meta = out, None
    status_ok(ws)
    # the oracle layer by layer, each on the input the GPU layer saw: X and meta for the
    # first, the previous GPU layer's output after that, and for a consumer the K/V the
    # GPU cache holds (a chained fp64 comparison would measure how much the layer pair
    # amplifies bf16 rounding of its input, ~1e-2 here, not the layer)
    refs, kv_ref, h_ref = [], None, []
    xin, min_ = x, meta
    for i, s in enumerate(layers):
        kv_in = None
        if s.kv_mode == O.KV_CONSUME:
            kc = to_np(cache[:, :, :T])
            kv_in = (kc[0], kc[1])
        o, kv_l, h = O.layer_prefill_state(xin, min_, ps[i], s, kv_in=kv_in)
        if s.kv_mode != O.KV_CONSUME:
            kv_ref = kv_l
        refs.append(o)
        h_ref.append(h)
        xin, min_ = to_np(outs[i]), None
    for i in range(len(layers)):
        assert_close(to_np(outs[i]), refs[i], dtype, f"prefill out, layer {i}")
        assert_close(to_np(states[i]), h_ref[i], dtype, f"SSM state after the prefill, layer {i}")
    kc = to_np(cache[:, :, :T])
    assert_close(kc[0], kv_ref[0], dtype, "cached K")
    assert_close(kc[1], kv_ref[1], dtype, "cached V")
    # decode steps
    hs = list(h_ref)
    for step in range(STEPS):
        pos = T + step
        xt = _tokens(wl, step)
        g_in = dev(xt, dtype)
        r_in = xt
        for i, (c, s) in enumerate(zip(cfgs, layers)):
            out_t = host.empty((s0.batch, s0.d_model), dtype)
            H.check(H.hymba_layer_decode(g_in, H.make_weights(dps[i]), c, cache, cap, pos, states[i], out_t, ws),
                    f"decode layer {i} step {step}")
            kv_step = kv_ref
            if s.kv_mode == O.KV_CONSUME:
                kc = to_np(cache[:, :, :pos + 1])
                kv_step = (kc[0], kc[1])
            r_out, kv_new, hs[i] = O.layer_decode_step(r_in, ps[i], s, kv_step, hs[i], pos)
            if s.kv_mode != O.KV_CONSUME:
                kv_ref = kv_new
                kc = to_np(cache[:, :, pos])
                assert_close(kc[0], kv_new[0][:, pos], dtype, f"cached K row {pos}, layer {i}")
                assert_close(kc[1], kv_new[1][:, pos], dtype, f"cached V row {pos}, layer {i}")
            assert_close(to_np(out_t), r_out, dtype, f"decode step {step}, layer {i}")
            g_in, r_in = out_t, to_np(out_t)
        status_ok(ws)
    for i in range(len(layers)):
        assert_close(to_np(states[i]), hs[i], dtype, f"SSM state after {STEPS} steps, layer {i}")


def test_decode_hymba350m_shaped():
    _run(synth.workload("hymba350m_layer", batch=2, seq_len=200))


def test_decode_kv_pair_window_meta_dstate128():
    _run(synth.workload("hymba1p5b_kvpair", batch=2, seq_len=300, window=64, d_model=512, n_q_heads=8,
                        n_kv_heads=2, d_inner=512, dt_rank=32))


@pytest.mark.parametrize("a_per_state", [0, 1])
def test_decode_fp32(a_per_state):
    _run(synth.workload("tiny_fp32", batch=2, a_per_state=a_per_state))


def test_decode_long_global_history_splits_keys():
    """Global attention over a 4K-row history: the key range is split over many CTAs."""
    _run(synth.workload("hymba350m_layer", batch=1, seq_len=4000, d_model=512, d_inner=512, dt_rank=32))
