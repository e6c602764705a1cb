"""Whole-layer and whole-stack parity on the GPU against the fp64 oracle, through
the C ABI, on the five seeded workloads.

The GPU always runs the full workload (the launch configuration the bench
times).  The oracle runs the full batch where it finishes in seconds and
otherwise a causal prefix of chosen sequences: output rows [0, t) depend only
on input rows [0, t), so the oracle on the truncated input gives those rows
exactly.  Prefixes are longer than window + meta, so the sliding window and the
always-visible meta tokens are exercised."""
import dataclasses

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
import oracle as O
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]


def _upload(wl, layers=None):
    layers = range(len(wl.layers)) if layers is None else layers
    ps = [synth.layer_params(wl, i) for i in layers]
    return ps, [host.params_to_device(p, wl.layers[i].dtype) for i, p in zip(layers, ps)]


def _oracle_layer(wl, ps, x, meta, batch_ids, L):
    """Oracle output rows [0, M + L) of the listed sequences (layer pairs chained)."""
    outs = []
    for b in batch_ids:
        xb = x[b:b + 1, :L]
        kv = None
        h = None
        for i, s in enumerate(wl.layers):
            si = dataclasses.replace(s, batch=1, seq_len=L)
            if i == 0:
                h, kv = O.layer_forward(xb, meta, ps[i], si)
            else:   # the consumer reads the producer's output and K/V
                h, _ = O.layer_forward(h, None, ps[i], si, kv_in=kv)
        outs.append(h[0])
    return outs


def _gpu_layers(wl, dps, x, meta):
    s0 = wl.first
    T = s0.T
    dtype = s0.dtype
    cfgs = [H.make_cfg(s) for s in wl.layers]
    ws = host.workspace(max(H.hymba_workspace_size(c) for c in cfgs))
    kv = host.empty((2, s0.batch * T, s0.kv_width), dtype) if len(wl.layers) > 1 else None
    tx, tm = dev(x, dtype), dev(meta, dtype)
    out = host.empty((s0.batch, T, s0.d_model), dtype)
    H.check(H.hymba_layer_fwd(tx, tm, H.make_weights(dps[0]), cfgs[0], None, kv, out, ws), "layer 0")
    outs = [out]
    for i in range(1, len(wl.layers)):
        o2 = host.empty((s0.batch, T, s0.d_model), dtype)
        H.check(H.hymba_layer_fwd(outs[-1], None, H.make_weights(dps[i]), cfgs[i], kv, None, o2, ws),
                f"layer {i}")
        outs.append(o2)
    status_ok(ws)
    return to_np(outs[-1])


def test_tiny_fp32_layer_full():
    wl = synth.workload("tiny_fp32")
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    ref, _ = O.layer_forward(x, meta, ps[0], wl.first)
    assert_close(g, ref, "f32", "tiny fp32 layer")


def test_hymba350m_layer_full_batch():
    wl = synth.workload("hymba350m_layer")
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    ref, _ = O.layer_forward(x, meta, ps[0], wl.first)
    for b in range(wl.first.batch):
        assert_close(g[b], ref[b], "bf16", f"350M layer, sequence {b}")


@pytest.mark.parametrize("name,prefixes", [
    ("hymba1p5b_kvpair", {0: 1300, 3: 200}),
    ("longctx_32k", {0: 1420}),
])
def test_large_layers_prefix(name, prefixes):
    wl = synth.workload(name)
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    M = wl.first.n_meta
    for b, L in prefixes.items():
        ref = _oracle_layer(wl, ps, x, meta, [b], L)[0]
        assert_close(g[b, :M + L], ref, "bf16", f"{name} sequence {b} rows [0, {M + L})")


def test_longctx_32k_layer_last_rows():
    """The 32K-context layer (dt down to 1e-4: long decay products) at full size; the
    last 128 of its 32,896 rows against the oracle, which runs the projections and the
    scan over every row and the attention and out_proj for those rows only."""
    wl = synth.workload("longctx_32k")
    s = wl.first
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    rows = np.arange(s.T - 128, s.T)
    ref = O.layer_forward_rows(x[:1], meta, ps[0], s, rows)
    assert_close(g[0, rows], ref, "bf16", "longctx_32k rows [T-128, T)")


def test_kvpair_last_rows_of_last_sequence():
    """The 1.5B-shaped producer + consumer pair at full size; the last 64 rows of
    sequence 3 against the oracle (the producer over every row, since the consumer reads
    its output and K/V; the consumer's attention and out_proj for those rows only)."""
    wl = synth.workload("hymba1p5b_kvpair")
    sp, sc = wl.layers
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    b = sp.batch - 1
    s1 = dataclasses.replace(sp, batch=1)
    h, kv = O.layer_forward(x[b:b + 1], meta, ps[0], s1)
    rows = np.arange(sp.T - 64, sp.T)
    ref = O.layer_forward_rows(h, None, ps[1], dataclasses.replace(sc, batch=1), rows, kv_in=kv)
    assert_close(g[b, rows], ref, "bf16", f"kvpair sequence {b} rows [T-64, T)")


def test_meta_rows_identical_across_batch_and_meta_mode_equals_explicit_xtilde():
    """Meta output rows are the same for every sequence; passing meta separately
    equals passing X~ = [meta; X] with meta = NULL."""
    wl = synth.workload("hymba350m_layer", batch=3, seq_len=500)
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta)
    M = wl.first.n_meta
    for b in range(1, 3):
        np.testing.assert_array_equal(g[b, :M], g[0, :M])
    xt = np.concatenate([np.broadcast_to(meta, (3,) + meta.shape), x], axis=1)
    cfg = H.make_cfg(wl.first)
    out = host.empty((3, wl.first.T, wl.first.d_model), "bf16")
    ws = host.workspace(H.hymba_workspace_size(cfg))
    H.check(H.hymba_layer_fwd(dev(xt, "bf16"), None, H.make_weights(dps[0]), cfg, None, None, out, ws), "X~")
    np.testing.assert_array_equal(to_np(out), g)


@pytest.mark.parametrize("kw", [dict(n_meta=0, window=0), dict(n_meta=8, window=0), dict(window=300),
                                dict(seq_len=1), dict(n_meta=136, window=64)])
def test_layer_edge_configs(kw):
    """No meta / self-only window / meta + zero window / one token / meta not a
    multiple of the 128-row tile."""
    kw = dict(kw)
    wl = synth.workload("hymba350m_layer", batch=2, seq_len=kw.pop("seq_len", 333), **kw)
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _gpu_layers(wl, dps, x, meta if wl.first.n_meta else np.zeros((0, wl.first.d_model), np.float32))
    ref, _ = O.layer_forward(x, meta if wl.first.n_meta else None, ps[0], wl.first)
    assert_close(g, ref, "bf16", f"edge {kw}")


@pytest.mark.parametrize("name,kw", [("tiny_fp32", {}), ("hymba350m_layer", dict(batch=2, seq_len=300))])
def test_layer_per_state_decay(name, kw):
    """a_per_state = 1: A_log [d_inner, d_state], the SSM head with one decay per channel and
    state, through the whole layer."""
    wl = synth.workload(name, a_per_state=1, **kw)
    assert wl.first.a_per_state == 1
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    assert ps[0]["a_log"].shape == (wl.first.d_inner, wl.first.d_state)
    g = _gpu_layers(wl, dps, x, meta)
    ref, _ = O.layer_forward(x, meta, ps[0], wl.first)
    assert_close(g, ref, wl.first.dtype, f"{name} per-state A")


def test_kv_sharing_consumer_equals_standalone_layer():
    """A consumer fed the producer's K/V equals a standalone layer whose W_K, W_V
    rows would produce that K/V (same Q, SSM and output weights)."""
    wl = synth.workload("hymba1p5b_kvpair", batch=1, seq_len=700)
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    s0 = wl.first
    T, wa, wkv = s0.T, s0.attn_width, s0.kv_width
    kv = host.empty((2, T, wkv), "bf16")
    cfg_p = H.make_cfg(s0)
    ws = host.workspace(H.hymba_workspace_size(cfg_p))
    out_p = host.empty((1, T, s0.d_model), "bf16")
    tx, tm = dev(x, "bf16"), dev(meta, "bf16")
    H.check(H.hymba_layer_fwd(tx, tm, H.make_weights(dps[0]), cfg_p, None, kv, out_p, ws), "producer")
    # consumer weights = producer's weights without the W_K, W_V rows
    w_in_c = torch.cat([dps[0]["w_in"][:wa], dps[0]["w_in"][wa + 2 * wkv:]]).contiguous()
    dpc = dict(dps[0], w_in=w_in_c)
    cfg_c = H.make_cfg(dataclasses.replace(s0, kv_mode=H.HYMBA_KV_CONSUME))
    out_c = host.empty((1, T, s0.d_model), "bf16")
    H.check(H.hymba_layer_fwd(tx, tm, H.make_weights(dpc), cfg_c, kv, None, out_c, ws), "consumer")
    status_ok(ws)
    np.testing.assert_array_equal(to_np(out_c), to_np(out_p))


def _run_stack(wl, x, meta, dps):
    s0 = wl.first
    cfgs = [H.make_cfg(s) for s in wl.layers]
    ws = host.workspace(H.hymba_stack_workspace_size(cfgs))
    out = host.empty((s0.batch, s0.T, s0.d_model), "bf16")
    H.check(H.hymba_stack_fwd(dev(x, "bf16"), dev(meta, "bf16"), [H.make_weights(d) for d in dps], cfgs, out,
                              ws), "stack")
    status_ok(ws)
    return to_np(out)


@pytest.mark.parametrize("pair", range(12))
def test_stack24_block_pair_full_size(pair):
    """Every block pair (2k, 2k+1) of the 24-block workload -- producer and consumer
    of one shared K/V, global or SWA as scheduled, SwiGLU FFN -- run as a 2-block
    stack on the full batch; sequence 0 checked over a causal prefix longer than
    window + meta, sequence 7 over a short prefix.  Bound: 2e-2 for every pair and
    sequence (tests/golden/stack24_tolerance.json also lists the deviation that the
    oracle with the path's storage roundings shows for each)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "stack24_tolerance.json")) as f:
        bounds = json.load(f)["block_pairs"]
    full = synth.workload("hymba1p5b_stack24")
    wl = synth.workload("hymba1p5b_stack24")
    wl.layers = full.layers[2 * pair:2 * pair + 2]
    s0 = wl.first
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(full, 2 * pair + i) for i in range(2)]
    dps = [host.params_to_device(p, "bf16") for p in ps]
    g = _run_stack(wl, x, meta, dps)
    for b, L in ((0, 1100), (7, 160)):
        shapes = [dataclasses.replace(s, batch=1, seq_len=L) for s in wl.layers]
        ref = O.stack_forward(x[b:b + 1, :L], meta, ps, shapes)
        bound = bounds[f"{pair}/{b}"]
        assert bound["prefix_user_tokens"] == L and bound["tolerance"] == 2e-2
        assert_close(g[b, :s0.n_meta + L], ref[0], "bf16", f"blocks {2 * pair},{2 * pair + 1} sequence {b}",
                     tol=bound["tolerance"])


def test_stack24_full_depth_prefix():
    """All 24 blocks at full size on the GPU; sequence 0's causal prefix against the
    oracle.  Bound: the depth-24 tolerance derived in tests/golden/stack24_tolerance.json
    by a procedure fixed in advance (the exact oracle vs the oracle with rounding at the
    path's storage points, largest over 8 placements of the rounding errors, x1.5); every
    block pair is held at 2e-2 (block-pair test above)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "stack24_tolerance.json")) as f:
        tol = json.load(f)
    wl = synth.workload("hymba1p5b_stack24")
    s0 = wl.first
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _run_stack(wl, x, meta, dps)
    L = tol["prefix_user_tokens"]
    shapes = [dataclasses.replace(s, batch=1, seq_len=L) for s in wl.layers]
    ref = O.stack_forward(x[:1, :L], meta, ps, shapes)
    assert_close(g[0, :s0.n_meta + L], ref[0], "bf16", "24-block stack, sequence 0 prefix",
                 tol=tol["tolerance_24_blocks"])


def test_stack_two_blocks_with_prenorm_gains_every_row():
    """Two blocks with non-unit pre-norm gains (norm1, norm2 ~ U(0.5, 1.5)), SWA producer and
    global consumer, ragged T: every output row at 2e-2."""
    wl = synth.workload("hymba1p5b_stack24", n_layers=2, batch=2, seq_len=700, d_model=1024,
                        n_q_heads=8, n_kv_heads=2, d_inner=2048, dt_rank=64, ffn_dim=2816)
    wl.layers[0] = dataclasses.replace(wl.layers[0], window=200)
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i, norm_gains=True) for i in range(2)]
    dps = [host.params_to_device(p, "bf16") for p in ps]
    g = _run_stack(wl, x, meta, dps)
    ref = O.stack_forward(x, meta, ps, wl.layers)
    assert_close(g, ref, "bf16", "2-block stack with pre-norm gains")


def test_stack_two_blocks_every_row():
    """Two blocks (global producer, SWA consumer), ragged T, two sequences, every
    output row checked at 2e-2."""
    wl = synth.workload("hymba1p5b_stack24", n_layers=2, batch=2, seq_len=1300, d_model=1024,
                        n_q_heads=8, n_kv_heads=2, d_inner=2048, dt_rank=64, ffn_dim=2816)
    wl.layers[1] = dataclasses.replace(wl.layers[1], window=300)
    x, meta = synth.layer_inputs(wl)
    ps, dps = _upload(wl)
    g = _run_stack(wl, x, meta, dps)
    ref = O.stack_forward(x, meta, ps, wl.layers)
    assert_close(g, ref, "bf16", "2-block stack")


def test_stack_fp32_two_blocks_with_gains():
    """The fp32 path of the stack (residual stream in `out`, fp32 pre-norms with gains):
    two blocks sharing K/V, every element at 1e-4."""
    s = dataclasses.replace(synth.workload("tiny_fp32").first, ffn_dim=96)
    layers = [dataclasses.replace(s, kv_mode=H.HYMBA_KV_PRODUCE, window=20),
              dataclasses.replace(s, kv_mode=H.HYMBA_KV_CONSUME)]
    wl = synth.Workload("tiny_fp32_stack", layers, 0, 1e-3, True, "two fp32 blocks")
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i, norm_gains=True) for i in range(2)]
    dps = [host.params_to_device(p, "f32") for p in ps]
    cfgs = [H.make_cfg(l) for l in layers]
    ws = host.workspace(H.hymba_stack_workspace_size(cfgs))
    out = host.empty((s.batch, s.T, s.d_model), "f32")
    H.check(H.hymba_stack_fwd(dev(x, "f32"), dev(meta, "f32"), [H.make_weights(d) for d in dps], cfgs, out, ws),
            "fp32 stack")
    status_ok(ws)
    assert_close(to_np(out), O.stack_forward(x, meta, ps, layers), "f32", "fp32 2-block stack")
