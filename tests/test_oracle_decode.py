"""Pins of the oracle's generation step (CPU).

Generating one token from the attention heads' K/V cache and the SSM heads' state must
give exactly what the prefill gives for that row: layer_decode_step after a prefill of
L tokens equals row M + L of the prefill of L + 1 tokens, and the grown cache and the
advanced state equal the longer prefill's.  Checked for global attention, for a window
shorter than the history (with meta tokens that stay visible), over several steps, and
for a KV-sharing pair (the consumer reads the producer's grown cache)."""
import numpy as np
import pytest

import oracle as O
from hybrid_attention_ssm_hymba_b200 import synth

SMALL = dict(d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, d_inner=48, d_state=8, dt_rank=8)


def _rel(a, b):
    return float(np.abs(np.asarray(a) - np.asarray(b)).max() / max(np.abs(np.asarray(b)).max(), 1e-300))


@pytest.mark.parametrize("name,kw", [
    ("tiny_fp32", dict(batch=2)),
    ("hymba350m_layer", dict(batch=2, d_model=96, d_inner=64, n_q_heads=2, n_kv_heads=1, head_dim=32,
                             dt_rank=8)),
    ("hymba350m_layer", dict(batch=1, window=5, n_meta=3, **{k: v for k, v in SMALL.items()})),
])
@pytest.mark.parametrize("steps", [1, 3])
def test_decode_steps_equal_the_longer_prefill(name, kw, steps):
    L = 21
    wl = synth.workload(name, seq_len=L + steps, **kw)
    s = wl.first
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    M = s.n_meta
    full, (kf, vf), hf = O.layer_prefill_state(x, meta, p, s)
    _, kv, h = O.layer_prefill_state(x[:, :L], meta, p, s)
    for i in range(steps):
        out_t, kv, h = O.layer_decode_step(x[:, L + i], p, s, kv, h, M + L + i)
        assert _rel(out_t, full[:, M + L + i]) < 1e-10
    assert _rel(kv[0], kf) < 1e-12 and _rel(kv[1], vf) < 1e-12
    assert _rel(h, hf) < 1e-10


def test_decode_reaches_only_meta_and_the_window():
    """With window W, the new token's output does not change when keys outside
    [pos - W, pos] that are not meta rows are altered in the cache."""
    L = 30
    wl = synth.workload("hymba350m_layer", batch=1, seq_len=L + 1, window=4, n_meta=3, **SMALL)
    s = wl.first
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    _, (k, v), h = O.layer_prefill_state(x[:, :L], meta, p, s)
    pos = s.n_meta + L
    out_a, _, _ = O.layer_decode_step(x[:, L], p, s, (k, v), h, pos)
    k2, v2 = k.copy(), v.copy()
    far = np.arange(s.n_meta, pos - s.window)          # neither meta nor inside the window
    k2[:, far] += 3.0
    v2[:, far] -= 2.0
    out_b, _, _ = O.layer_decode_step(x[:, L], p, s, (k2, v2), h, pos)
    assert _rel(out_b, out_a) < 1e-12
    k3 = k.copy()
    k3[:, 0] += 3.0                                     # a meta row is always visible
    out_c, _, _ = O.layer_decode_step(x[:, L], p, s, (k3, v), h, pos)
    assert _rel(out_c, out_a) > 1e-6


def test_decode_through_a_kv_sharing_pair():
    L = 17
    wl = synth.workload("hymba1p5b_kvpair", batch=2, seq_len=L + 1, window=6, n_meta=4, **SMALL)
    assert [l.kv_mode for l in wl.layers] == [O.KV_PRODUCE, O.KV_CONSUME]
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(2)]
    s0, s1 = wl.layers
    # the longer prefill: producer, then consumer on the producer's output and K/V
    out0, kv0, _ = O.layer_prefill_state(x, meta, ps[0], s0)
    out1, _, h1f = O.layer_prefill_state(out0, None, ps[1], s1, kv_in=kv0)
    # prefill L tokens, then one decode step through both layers
    p0, kv, h0 = O.layer_prefill_state(x[:, :L], meta, ps[0], s0)
    _, _, h1 = O.layer_prefill_state(p0, None, ps[1], s1, kv_in=kv)
    pos = s0.n_meta + L
    o0, kv, h0 = O.layer_decode_step(x[:, L], ps[0], s0, kv, h0, pos)
    o1, _, h1 = O.layer_decode_step(o0, ps[1], s1, kv, h1, pos)
    assert _rel(o0, out0[:, pos]) < 1e-10
    assert _rel(o1, out1[:, pos]) < 1e-10
    assert _rel(h1, h1f) < 1e-10
