"""Meta-prefix precompute on the GPU through the C ABI.

hymba_meta_prefix computes what the layer does for the M meta rows -- identical for every
sequence under the causal mask -- once into a record; hymba_layer_fwd_prefixed then runs
only the user rows.  Checked: with d_state 16 and M a multiple of the scan's 64-row block
the prefixed layer is bit-identical to hymba_layer_fwd (the same kernels see the same
values in the same order); a KV-sharing pair with SWA and d_state 128 (the consumer's
record built from the producer's) and the fp32 path match the oracle."""
import dataclasses

import numpy as np
import pytest

import hybrid_attention_ssm_hymba_b200 as H
import oracle as O
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]

# Two GPU paths over the same input (prefixed call vs the full layer) agree to fp32 rounding
# before the bf16 stores; the largest output can still land one bf16 unit apart, 2^-7 of
# its magnitude.
PATH_TOL = 2.0 ** -7


def _prefixed_chain(wl, x, meta, dps, every_layer=False):
    """Every layer of the workload through records + prefixed calls (a pair: the consumer's
    record from the producer's record rows and K/V).  The last layer's output, or
    (every_layer) each layer's output and the shared K/V."""
    layers = wl.layers
    s0 = layers[0]
    dt = s0.dtype
    cfgs = [H.make_cfg(s) for s in layers]
    ws = host.workspace(max(H.hymba_workspace_size(c) for c in cfgs))
    recs = [host.workspace(H.hymba_meta_prefix_size(c)) for c in cfgs]
    tm = dev(meta, dt)
    meta_in = tm
    for i, c in enumerate(cfgs):
        H.check(H.hymba_meta_prefix(meta_in, H.make_weights(dps[i]), c, recs[0] if i > 0 else None, recs[i], ws),
                f"prefix {i}")
        # the next layer's meta rows are this layer's meta output rows (the record's first M rows)
        meta_in = recs[i][:s0.n_meta * s0.d_model * (2 if dt == "bf16" else 4)].view(
            host.torch_dtype(dt)).view(s0.n_meta, s0.d_model)
    kv = host.empty((2, s0.batch * s0.T, s0.kv_width), dt) if len(layers) > 1 else None
    out = host.empty((s0.batch, s0.T, s0.d_model), dt)
    H.check(H.hymba_layer_fwd_prefixed(dev(x, dt), recs[0], H.make_weights(dps[0]), cfgs[0], None, kv, out, ws),
            "prefixed 0")
    outs = [out]
    for i in range(1, len(layers)):
        # the consumer takes the producer's user rows; its meta rows come from its record
        o2 = host.empty((s0.batch, s0.T, s0.d_model), dt)
        H.check(H.hymba_layer_fwd_prefixed(outs[-1][:, s0.n_meta:].contiguous(), recs[i], H.make_weights(dps[i]),
                                           cfgs[i], kv, None, o2, ws), f"prefixed {i}")
        outs.append(o2)
    status_ok(ws)
    if every_layer:
        return [to_np(o) for o in outs], (None if kv is None else to_np(kv))
    return to_np(outs[-1])


def _plain_chain(wl, x, meta, dps, every_layer=False):
    """hymba_layer_fwd over every layer: the last layer's output, or (every_layer) each
    layer's output and the shared K/V."""
    layers = wl.layers
    s0 = layers[0]
    dt = s0.dtype
    cfgs = [H.make_cfg(s) for s in layers]
    ws = host.workspace(max(H.hymba_workspace_size(c) for c in cfgs))
    kv = host.empty((2, s0.batch * s0.T, s0.kv_width), dt) if len(layers) > 1 else None
    out = host.empty((s0.batch, s0.T, s0.d_model), dt)
    H.check(H.hymba_layer_fwd(dev(x, dt), dev(meta, dt), H.make_weights(dps[0]), cfgs[0], None, kv, out, ws), "0")
    outs = [out]
    for i in range(1, len(layers)):
        o2 = host.empty((s0.batch, s0.T, s0.d_model), dt)
        H.check(H.hymba_layer_fwd(outs[-1], None, H.make_weights(dps[i]), cfgs[i], kv, None, o2, ws), f"{i}")
        outs.append(o2)
    status_ok(ws)
    if every_layer:
        return [to_np(o) for o in outs], (None if kv is None else to_np(kv))
    return to_np(outs[-1])


def _setup(wl):
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(len(wl.layers))]
    return x, meta, ps, [host.params_to_device(p, wl.first.dtype) for p in ps]


def test_prefixed_layer_is_bit_identical_to_the_full_layer():
    wl = synth.workload("hymba350m_layer", batch=3, seq_len=333, n_meta=128)
    x, meta, ps, dps = _setup(wl)
    np.testing.assert_array_equal(_prefixed_chain(wl, x, meta, dps), _plain_chain(wl, x, meta, dps))


def test_prefixed_kv_pair_swa_dstate128_matches_oracle_and_full_path():
    """Each layer of the pair on the inputs that layer saw.  Against the oracle (2e-2): the
    producer on X and meta, the consumer on the producer's GPU output rows and K/V (fed the
    oracle's own fp64 producer output instead, the consumer differs by ~1e-2 from
    bf16-rounding that input alone: the pair amplifies input rounding).  Against the full
    path (one bf16 unit of the largest output): the prefixed producer with hymba_layer_fwd on the same X, the prefixed
    consumer with hymba_layer_fwd on the prefixed producer's output and K/V."""
    wl = synth.workload("hymba1p5b_kvpair", batch=2, seq_len=400, window=96, d_model=512, n_q_heads=8,
                        n_kv_heads=2, d_inner=512, dt_rank=32)
    x, meta, ps, dps = _setup(wl)
    s0, s1 = wl.layers
    (p0, p1), kv_p = _prefixed_chain(wl, x, meta, dps, every_layer=True)
    (h_gpu, _), _ = _plain_chain(wl, x, meta, dps, every_layer=True)
    h, _ = O.layer_forward(x, meta, ps[0], s0)
    assert_close(h_gpu, h, "bf16", "producer (full path) vs oracle")
    assert_close(p0, h, "bf16", "prefixed producer vs oracle")
    assert_close(p0, h_gpu, "bf16", "prefixed producer vs the full path", tol=PATH_TOL)
    kv_b = kv_p.reshape(2, s0.batch, s0.T, s0.kv_width)
    ref, _ = O.layer_forward(p0, None, ps[1], s1, kv_in=(kv_b[0], kv_b[1]))
    assert_close(p1, ref, "bf16", "prefixed consumer vs oracle")
    cfg1 = H.make_cfg(s1)
    ws = host.workspace(H.hymba_workspace_size(cfg1))
    full1 = host.empty((s0.batch, s0.T, s0.d_model), "bf16")
    H.check(H.hymba_layer_fwd(dev(p0, "bf16"), None, H.make_weights(dps[1]), cfg1, dev(kv_p, "bf16"), None, full1, ws),
            "consumer full path")
    status_ok(ws)
    assert_close(p1, to_np(full1), "bf16", "prefixed consumer vs the full path on the same input", tol=PATH_TOL)


@pytest.mark.parametrize("a_per_state", [0, 1])
def test_prefixed_fp32(a_per_state):
    wl = synth.workload("tiny_fp32", batch=2, a_per_state=a_per_state)
    x, meta, ps, dps = _setup(wl)
    ref, _ = O.layer_forward(x, meta, ps[0], wl.first)
    assert_close(_prefixed_chain(wl, x, meta, dps), ref, "f32", "prefixed fp32 layer")


@pytest.mark.parametrize("window,d_state", [(-1, 16), (96, 16), (-1, 128), (96, 128)])
def test_prefixed_single_layer_window_and_state_size(window, d_state):
    """One layer with its own K/V, global or windowed, tensor-core (d_state 16) or CUDA-core
    (d_state 128) scan: the prefixed call against the full path and the oracle."""
    wl = synth.workload("hymba1p5b_kvpair", n_layers=1, batch=2, seq_len=400, window=window, d_model=512,
                        n_q_heads=8, n_kv_heads=2, d_inner=512, dt_rank=32, d_state=d_state, kv_mode=H.HYMBA_KV_OWN)
    x, meta, ps, dps = _setup(wl)
    g = _prefixed_chain(wl, x, meta, dps)
    full = _plain_chain(wl, x, meta, dps)
    ref, _ = O.layer_forward(x, meta, ps[0], wl.first)
    assert_close(full, ref, "bf16", "full path vs oracle")
    assert_close(g, full, "bf16", "prefixed vs the full path", tol=PATH_TOL)
    assert_close(g, ref, "bf16", "prefixed vs oracle")
