"""hymba_layer_fwd_noalloc: the layer forward for callers that cannot allocate device
memory -- for example a plugin whose execute step runs inside a framework that owns
every allocation, or a latency-critical path where cudaMalloc would synchronise the
device.  It keeps the intermediates in the library's own static scratch block instead
of a caller workspace.

Checked here through the C ABI: two calls in a row, each on fresh inputs, give exactly
the output of hymba_layer_fwd with a caller workspace (the same kernels run on the same
inputs, so the results agree bit for bit); the second call must not see anything the
first one left in the shared block; a KV-sharing pair (producer, then consumer) gives
the same outputs and the same K/V as the workspace entry point.  This file is collected
last on purpose."""
import dataclasses

import numpy as np
import pytest

import hybrid_attention_ssm_hymba_b200 as H
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import dev, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]


def _with_workspace(x, meta, w, cfg, out_shape, dtype, kv_in=None, kv_out=None):
    out = host.empty(out_shape, dtype)
    ws = host.workspace(H.hymba_workspace_size(cfg))
    H.check(H.hymba_layer_fwd(x, meta, w, cfg, kv_in, kv_out, out, ws), "hymba_layer_fwd")
    status_ok(ws)
    return to_np(out)


@pytest.mark.parametrize("name,kw", [
    ("tiny_fp32", {}),
    ("hymba350m_layer", dict(batch=1, seq_len=224)),
    ("hymba1p5b_kvpair", dict(n_layers=1, batch=1, seq_len=120, window=48, d_model=512, n_q_heads=4,
                              n_kv_heads=2, d_inner=512, dt_rank=32)),
])
def test_noalloc_matches_workspace_entry_point_two_calls(name, kw):
    wl = synth.workload(name, **kw)
    s = dataclasses.replace(wl.first, kv_mode=H.HYMBA_KV_OWN)
    cfg = H.make_cfg(s)
    assert 0 < H.hymba_workspace_size(cfg) <= H.HYMBA_NOALLOC_SCRATCH_BYTES
    dps = host.params_to_device(synth.layer_params(wl, 0), s.dtype)   # kept alive for the calls
    w = H.make_weights(dps)
    x1, meta = synth.layer_inputs(wl)
    x2 = synth.normal(wl.seed, 1, "x", x1.shape, 1.0, s.dtype)   # another stream of the same recipe
    tm = dev(meta, s.dtype)
    shape = (s.batch, s.T, s.d_model)
    outs = []
    for x in (x1, x2):   # two calls in a row on the shared block, different inputs
        out = host.empty(shape, s.dtype)
        out.fill_(float("nan"))
        H.check(H.hymba_layer_fwd_noalloc(dev(x, s.dtype), tm, w, cfg, None, None, out), "noalloc")
        outs.append(to_np(out))
    for i, x in enumerate((x1, x2)):
        ref = _with_workspace(dev(x, s.dtype), tm, w, cfg, shape, s.dtype)
        np.testing.assert_array_equal(outs[i], ref, err_msg=f"{name} noalloc call {i + 1}")
    assert not np.allclose(outs[0], outs[1]), "the two calls must see their own inputs"


def test_noalloc_kv_sharing_pair_matches_workspace_entry_point():
    """HYMBA_KV_PRODUCE then HYMBA_KV_CONSUME through the scratch block: K/V go to the
    caller's kv buffer and come back from it; outputs and K/V equal the workspace path."""
    wl = synth.workload("hymba1p5b_kvpair", batch=1, seq_len=120, window=48, d_model=512, n_q_heads=4,
                        n_kv_heads=2, d_inner=512, dt_rank=32)
    sp, sc = wl.layers
    cp, cc = H.make_cfg(sp), H.make_cfg(sc)
    assert max(H.hymba_workspace_size(cp), H.hymba_workspace_size(cc)) <= H.HYMBA_NOALLOC_SCRATCH_BYTES
    dps = [host.params_to_device(synth.layer_params(wl, i), "bf16") for i in range(2)]
    ws_ = [H.make_weights(d) for d in dps]
    x, meta = synth.layer_inputs(wl)
    tx, tm = dev(x, "bf16"), dev(meta, "bf16")
    T = sp.T
    shape = (1, T, sp.d_model)
    res = []
    for noalloc in (True, False):
        kv = host.empty((2, T, sp.kv_width), "bf16")
        kv.fill_(float("nan"))
        o1, o2 = host.empty(shape, "bf16"), host.empty(shape, "bf16")
        if noalloc:
            H.check(H.hymba_layer_fwd_noalloc(tx, tm, ws_[0], cp, None, kv, o1), "noalloc producer")
            H.check(H.hymba_layer_fwd_noalloc(o1, None, ws_[1], cc, kv, None, o2), "noalloc consumer")
        else:
            ws = host.workspace(max(H.hymba_workspace_size(cp), H.hymba_workspace_size(cc)))
            H.check(H.hymba_layer_fwd(tx, tm, ws_[0], cp, None, kv, o1, ws), "producer")
            H.check(H.hymba_layer_fwd(o1, None, ws_[1], cc, kv, None, o2, ws), "consumer")
            status_ok(ws)
        res.append((to_np(o1), to_np(o2), to_np(kv)))
    for a, b, what in zip(res[0], res[1], ("producer out", "consumer out", "K/V")):
        np.testing.assert_array_equal(a, b, err_msg=what)


def test_noalloc_rejects_configs_beyond_the_scratch_block():
    wl = synth.workload("hymba350m_layer")   # B=8, L=2048: ~300 MB of intermediates
    cfg = H.make_cfg(wl.first)
    assert H.hymba_workspace_size(cfg) > H.HYMBA_NOALLOC_SCRATCH_BYTES
    dps = host.params_to_device(synth.layer_params(synth.workload("tiny_fp32"), 0), "f32")
    w = H.make_weights(dps)
    out = host.empty((1, 1, 8), "bf16")
    assert H.hymba_layer_fwd_noalloc(out, out, w, cfg, None, None, out) == H.HYMBA_ERR_WORKSPACE
