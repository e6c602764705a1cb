"""Pins for the fp64 oracle: closed forms, hand-worked examples, brute force,
library special cases and the invariants the Hymba pages imply.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one window) fails it.
CPU only, seconds in total.
"""
import dataclasses
import math

import numpy as np
import pytest
import scipy.special

import oracle as O
from hybrid_attention_ssm_hymba_b200 import synth

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# SSM: recurrence vs the materialised alpha_ij form, closed forms, hand examples

@pytest.mark.parametrize("per_state", [False, True])
@pytest.mark.parametrize("T,Di,N", [(1, 3, 2), (7, 4, 3), (33, 5, 4)])
def test_scan_equals_alpha_matrix_form(per_state, T, Di, N):
    """Recurrence == alpha_ij = C_i (prod_{k=j+1..i} exp(A dt_k)) B_j dt_j form
    (Hymba review, "Design formulation"), to fp64 rounding."""
    x = RNG.standard_normal((T, Di))
    dt = RNG.uniform(1e-3, 0.3, (T, Di))
    A = -RNG.uniform(0.5, 4.0, (Di, N) if per_state else (Di,))
    Bm, Cm = RNG.standard_normal((T, N)), RNG.standard_normal((T, N))
    y = O.selective_scan(x, dt, A, Bm, Cm)
    y_alpha = O.ssm_from_alpha(x, O.ssm_alpha_matrix(dt, A, Bm, Cm))
    np.testing.assert_allclose(y, y_alpha, rtol=0, atol=1e-12 * max(1.0, np.abs(y).max()))


def test_scan_cumsum_special_case():
    """N = 1, A = 0 (no decay), dt = 1, B = C = 1: y = cumsum(x)."""
    T = 50
    x = RNG.standard_normal((T, 3))
    y = O.selective_scan(x, np.ones((T, 3)), np.zeros(3), np.ones((T, 1)), np.ones((T, 1)))
    np.testing.assert_allclose(y, np.cumsum(x, axis=0), rtol=1e-13, atol=1e-13)


def test_scan_constant_decay_closed_form():
    """Constant a = exp(A dt), B = C = 1: y_i = dt sum_j a^(i-j) x_j, and for x = 1
    the geometric series y_i = dt (1 - a^(i+1)) / (1 - a)."""
    T, dt, A = 40, 0.25, -1.3
    a = math.exp(A * dt)
    x = RNG.standard_normal((T, 1))
    y = O.selective_scan(x, np.full((T, 1), dt), np.array([A]), np.ones((T, 1)), np.ones((T, 1)))
    powers = np.array([[a ** (i - j) if j <= i else 0.0 for j in range(T)] for i in range(T)])
    np.testing.assert_allclose(y[:, 0], dt * powers @ x[:, 0], rtol=1e-12, atol=1e-14)
    y1 = O.selective_scan(np.ones((T, 1)), np.full((T, 1), dt), np.array([A]), np.ones((T, 1)),
                          np.ones((T, 1)))
    i = np.arange(T)
    np.testing.assert_allclose(y1[:, 0], dt * (1 - a ** (i + 1)) / (1 - a), rtol=1e-12)


def test_scan_impulse_response():
    """x = impulse at j0: y_i = C_i . (prod_{k=j0+1..i} exp(A dt_k)) B_{j0} dt_{j0}
    for i >= j0 and 0 before (per-state decay, so the product stays per state)."""
    T, N, j0 = 12, 3, 4
    dt = RNG.uniform(0.05, 0.4, (T, 1))
    A = -np.array([[0.3, 1.1, 2.5]])
    Bm, Cm = RNG.standard_normal((T, N)), RNG.standard_normal((T, N))
    x = np.zeros((T, 1)); x[j0] = 1.0
    y = O.selective_scan(x, dt, A, Bm, Cm)[:, 0]
    for i in range(T):
        if i < j0:
            assert y[i] == 0.0
        else:
            decay = np.exp(A[0] * dt[j0 + 1:i + 1, 0].sum())
            assert y[i] == pytest.approx(float(Cm[i] @ (decay * Bm[j0])) * dt[j0, 0], rel=1e-12, abs=1e-15)


def test_scan_hand_example():
    """Worked by hand: N = 2, A = -ln 2, dt = 1 so a = 1/2, B_0 = (1, 2), B_1 = (0, 1),
    C_0 = (1, 1), C_1 = (2, 0), x = (1, 1):
      t=0: h = (1, 2),                  y_0 = 1 + 2 = 3
      t=1: h = (0.5, 1) + (0, 1) = (0.5, 2), y_1 = 2*0.5 + 0*2 = 1
    and the alpha form: alpha_00 = 3, alpha_10 = C_1 . (1/2) B_0 = 1, alpha_11 = 0."""
    x = np.array([[1.0], [1.0]])
    dt = np.ones((2, 1))
    A = np.array([-math.log(2.0)])
    Bm = np.array([[1.0, 2.0], [0.0, 1.0]])
    Cm = np.array([[1.0, 1.0], [2.0, 0.0]])
    np.testing.assert_allclose(O.selective_scan(x, dt, A, Bm, Cm)[:, 0], [3.0, 1.0], atol=1e-15)
    al = O.ssm_alpha_matrix(dt, A, Bm, Cm)[0]
    np.testing.assert_allclose(al, [[3.0, 0.0], [1.0, 0.0]], atol=1e-15)


def test_scan_three_step_hand_example():
    """N = 1, a = 1/2, dt = B = C = 1, x = (1, 2, 3): h = 1, 2.5, 4.25."""
    y = O.selective_scan(np.array([[1.0], [2.0], [3.0]]), np.ones((3, 1)), np.array([-math.log(2)]),
                         np.ones((3, 1)), np.ones((3, 1)))
    np.testing.assert_allclose(y[:, 0], [1.0, 2.5, 4.25], atol=1e-15)


def test_scan_states_are_independent_and_additive():
    """y = sum over states of one-state scans (C_t . h_t is a sum over n)."""
    T, Di, N = 20, 2, 4
    x, dt = RNG.standard_normal((T, Di)), RNG.uniform(0.01, 0.3, (T, Di))
    A = -RNG.uniform(0.5, 3, Di)
    Bm, Cm = RNG.standard_normal((T, N)), RNG.standard_normal((T, N))
    y = O.selective_scan(x, dt, A, Bm, Cm)
    ysum = sum(O.selective_scan(x, dt, A, Bm[:, n:n + 1], Cm[:, n:n + 1]) for n in range(N))
    np.testing.assert_allclose(y, ysum, rtol=1e-12, atol=1e-14)


def test_scan_batched_equals_per_sequence_and_state_carry():
    """Leading batch axes are independent; splitting T and carrying h gives the same y."""
    B, T, Di, N = 3, 17, 4, 5
    x, dt = RNG.standard_normal((B, T, Di)), RNG.uniform(0.01, 0.3, (B, T, Di))
    A = -RNG.uniform(0.5, 3, Di)
    Bm, Cm = RNG.standard_normal((B, T, N)), RNG.standard_normal((B, T, N))
    y = O.selective_scan(x, dt, A, Bm, Cm)
    for b in range(B):
        np.testing.assert_allclose(y[b], O.selective_scan(x[b], dt[b], A, Bm[b], Cm[b]), rtol=1e-14)
        y1, h = O.selective_scan(x[b, :9], dt[b, :9], A, Bm[b, :9], Cm[b, :9], return_state=True)
        y2 = O.selective_scan(x[b, 9:], dt[b, 9:], A, Bm[b, 9:], Cm[b, 9:], h0=h)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y[b], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# elementwise pieces

def test_softplus_silu_rms_closed_forms():
    assert O.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    z = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(O.softplus(z), np.log1p(np.exp(z)), rtol=1e-13)
    assert O.softplus(800.0) == pytest.approx(800.0)
    np.testing.assert_allclose(O.silu(z), z * scipy.special.expit(z), rtol=1e-13, atol=1e-300)
    assert O.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    # RMSNorm of (3, 4): rms = sqrt(12.5)
    np.testing.assert_allclose(O.rms_normalize(np.array([3.0, 4.0]), 0.0),
                               [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15)
    # RMSNorm of a constant vector c*1 is sign(c)*1 up to eps
    for c in (-3.0, 0.7):
        v = np.full(64, c)
        np.testing.assert_allclose(O.rms_normalize(v, 1e-6), np.sign(c) / np.sqrt(1 + 1e-6 / c ** 2),
                                   rtol=1e-14)


def test_generator_dt_recipe_inverts_softplus():
    """b_dt = inverse softplus of dt0, so softplus(b_dt) gives dt0 back."""
    dt0 = np.array([1e-4, 1e-3, 0.01, 0.05, 0.1])
    np.testing.assert_allclose(O.softplus(synth.inverse_softplus(dt0)), dt0, rtol=2e-6)


def test_linear_against_triple_loop():
    x, w = RNG.standard_normal((5, 7)), RNG.standard_normal((3, 7))
    ref = np.array([[sum(x[i, k] * w[n, k] for k in range(7)) for n in range(3)] for i in range(5)])
    np.testing.assert_allclose(O.linear(x, w), ref, rtol=1e-13)


def test_meta_prepend():
    x, meta = RNG.standard_normal((2, 3, 4)), RNG.standard_normal((5, 4))
    xt = O.meta_prepend(x, meta)
    assert xt.shape == (2, 8, 4)
    for b in range(2):
        np.testing.assert_array_equal(xt[b, :5], meta)
        np.testing.assert_array_equal(xt[b, 5:], x[b])


# ---------------------------------------------------------------------------
# attention

def _enumerated_visible(T, M, W):
    """The visible set from its definition, by enumeration."""
    s = set()
    for i in range(T):
        for j in range(T):
            if j <= i and (W < 0 or i - j <= W or j < M):
                s.add((i, j))
    return s


@pytest.mark.parametrize("M", [0, 3, 8])
@pytest.mark.parametrize("W", [-1, 0, 1, 3, 7, 100])
def test_visibility_set_and_row_sums(M, W):
    T = 24
    m = O.visibility_mask(T, M, W)
    got = {(i, j) for i in range(T) for j in range(T) if m[i, j]}
    assert got == _enumerated_visible(T, M, W)
    assert all(O.visible(i, j, M, W) == ((i, j) in got) for i in range(T) for j in range(T))
    q, k = RNG.standard_normal((T, 8)), RNG.standard_normal((T, 8))
    p = O.attention_probs(q, k, M, W)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p[~m] == 0.0)
    assert np.all(p[m] > 0.0)


def test_window_examples_by_hand():
    """T = 4, M = 1 meta token, W = 1, zero queries (uniform weights over the
    visible keys), v = (1, 10, 100, 1000):
      row 0 sees {0}       -> 1
      row 1 sees {0, 1}    -> 5.5
      row 2 sees {0, 1, 2} -> 37   (key 0 through the meta rule, key 1 through the window)
      row 3 sees {0, 2, 3} -> 367  (key 1 is outside the window and not meta)"""
    v = np.array([[1.0], [10.0], [100.0], [1000.0]])
    out = O.attention(np.zeros((4, 1)), np.zeros((4, 1)), v, 1, 1, n_meta=1, window=1)
    np.testing.assert_allclose(out[:, 0], [1.0, 5.5, 37.0, 367.0], rtol=1e-14)


def test_attention_hand_example():
    """dh = 4 (scale 1/2); q_1 . k_1 / 2 = ln 3 and q_1 . k_0 = 0, so row 1
    weights are (1/4, 3/4); v_0 = (4,0,0,0), v_1 = (0,4,0,0) -> out_1 = (1,3,0,0);
    row 0 sees only key 0 -> out_0 = v_0."""
    q = np.array([[1.0, 1.0, 1.0, 1.0], [2 * math.log(3.0), 0, 0, 0]])
    k = np.array([[0.0, 0, 0, 0], [1.0, 0, 0, 0]])
    v = np.array([[4.0, 0, 0, 0], [0, 4.0, 0, 0]])
    out = O.attention(q, k, v, 1, 1, n_meta=0, window=-1)
    np.testing.assert_allclose(out, [[4, 0, 0, 0], [1, 3, 0, 0]], atol=1e-14)


def test_self_only_when_zero_window_and_no_meta():
    """W = 0 and M = 0: each query sees only itself, so out = V_i."""
    T = 20
    q, k, v = RNG.standard_normal((T, 16)), RNG.standard_normal((T, 16)), RNG.standard_normal((T, 16))
    np.testing.assert_allclose(O.attention(q, k, v, 1, 1, 0, 0), v, rtol=1e-14)


def test_large_window_equals_global_and_single_key():
    T = 30
    q, k, v = (RNG.standard_normal((T, 2 * 8)) for _ in range(3))
    g = O.attention(q, k, v, 2, 2, 5, -1)
    for W in (T - 1, T + 10):
        np.testing.assert_allclose(O.attention(q, k, v, 2, 2, 5, W), g, rtol=1e-14)
    np.testing.assert_allclose(g[0], v[0], rtol=1e-14)      # the first query sees one key


def test_attention_matches_library_softmax_brute_force():
    """Per row: softmax over the visible keys (scipy) of q.k/sqrt(dh), times V."""
    T, dh, M, W = 19, 8, 2, 4
    q, k, v = (RNG.standard_normal((T, dh)) for _ in range(3))
    out = O.attention(q, k, v, 1, 1, M, W)
    for i in range(T):
        js = [j for j in range(T) if j <= i and (i - j <= W or j < M)]
        w = scipy.special.softmax(np.array([q[i] @ k[j] for j in js]) / math.sqrt(dh))
        np.testing.assert_allclose(out[i], sum(wj * v[j] for wj, j in zip(w, js)), rtol=1e-12)


def test_gqa_equals_mha_with_replicated_kv():
    T, dh, Hq, Hkv = 15, 4, 6, 2
    q = RNG.standard_normal((T, Hq * dh))
    k, v = RNG.standard_normal((T, Hkv * dh)), RNG.standard_normal((T, Hkv * dh))
    rep = lambda a: np.concatenate([a[:, (h // 3) * dh:(h // 3 + 1) * dh] for h in range(Hq)], axis=1)
    np.testing.assert_allclose(O.attention(q, k, v, Hq, Hkv, 3, 5),
                               O.attention(q, rep(k), rep(v), Hq, Hq, 3, 5), rtol=1e-14)


def test_attention_row_subset_equals_full():
    T = 40
    q, k, v = (RNG.standard_normal((T, 8)) for _ in range(3))
    full = O.attention(q, k, v, 1, 1, 4, 6)
    rows = np.array([0, 5, 39, 17])
    np.testing.assert_allclose(O.attention(q[rows], k, v, 1, 1, 4, 6, rows=rows), full[rows], rtol=1e-14)


# ---------------------------------------------------------------------------
# layer-level invariants

def _tiny_shape(**kw):
    base = dict(batch=2, seq_len=11, n_meta=3, d_model=16, n_q_heads=2, n_kv_heads=1, head_dim=4,
                window=-1, d_inner=12, d_state=4, n_ssm_heads=2, dt_rank=2, dtype="f32")
    base.update(kw)
    return synth.LayerShape(**base)


def _tiny(seed=7, **kw):
    s = _tiny_shape(**kw)
    wl = synth.Workload("t", [s], seed, 1e-3, False, "tiny")
    x, meta = synth.layer_inputs(wl)
    return s, x, meta, synth.layer_params(wl, 0)


def test_beta2_zero_gives_attention_only_and_beta1_zero_ssm_only():
    """beta2 = 0 -> W_out,a (beta1 n(Y_attn)); beta1 = 0 -> W_out,s (beta2 n(Y_ssm))."""
    s, x, meta, p = _tiny()
    _, _, parts = O.layer_forward(x, meta, p, s, return_parts=True)
    wa = s.n_q_heads * s.head_dim

    def nrm(v):     # an independent RMS: |v| / sqrt(width)
        return v / np.sqrt(np.linalg.norm(v, axis=-1, keepdims=True) ** 2 / v.shape[-1] + s.rms_eps)

    p0 = dict(p, beta2=np.zeros_like(p["beta2"]))
    out, _ = O.layer_forward(x, meta, p0, s)
    np.testing.assert_allclose(out, (p["beta1"] * nrm(parts["y_attn"])) @ p["w_out"][:, :wa].T.astype(float),
                               rtol=1e-12, atol=1e-13)
    p1 = dict(p, beta1=np.zeros_like(p["beta1"]))
    out, _ = O.layer_forward(x, meta, p1, s)
    np.testing.assert_allclose(out, (p["beta2"] * nrm(parts["y_ssm"])) @ p["w_out"][:, wa:].T.astype(float),
                               rtol=1e-12, atol=1e-13)


def test_half_beta_reproduces_averaged_fusion():
    """beta1 = beta2 = 0.5 with equal branch widths and a tied out projection
    reproduces the averaged fusion out_proj(0.5 (ssm_norm + attn_norm)) of the
    metaphor-xennon HymbaLayer pseudocode."""
    s, x, meta, p = _tiny(d_inner=8)          # Hq*dh = 8 = d_inner
    w = p["w_out"][:, :8].astype(np.float64)
    p = dict(p, w_out=np.concatenate([w, w], axis=1), beta1=np.full(8, 0.5), beta2=np.full(8, 0.5))
    out, _, parts = O.layer_forward(x, meta, p, s, return_parts=True)
    fused = 0.5 * (O.rms_normalize(parts["y_ssm"], s.rms_eps) + O.rms_normalize(parts["y_attn"], s.rms_eps))
    np.testing.assert_allclose(out, fused @ w.T, rtol=1e-12, atol=1e-13)


def test_batch_independence_and_meta_rows():
    """Batch rows are independent; meta output rows are the same for every
    sequence and do not depend on X (meta tokens are fixed at inference)."""
    s, x, meta, p = _tiny(window=4)
    out, _ = O.layer_forward(x, meta, p, s)
    for b in range(2):
        ob, _ = O.layer_forward(x[b:b + 1], meta, p, s)
        np.testing.assert_allclose(ob[0], out[b], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(out[0, :3], out[1, :3], rtol=1e-13, atol=1e-14)
    out2, _ = O.layer_forward(x * 3.0 + 1.0, meta, p, s)
    np.testing.assert_allclose(out2[:, :3], out[:, :3], rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("window", [-1, 3])
def test_causality_prefix(window):
    """Rows [0, t) of the output depend only on rows [0, t) of X~."""
    s, x, meta, p = _tiny(window=window)
    out, _ = O.layer_forward(x, meta, p, s)
    for L in (1, 4, 9):
        outp, _ = O.layer_forward(x[:, :L], meta, p, s)
        np.testing.assert_allclose(outp, out[:, :3 + L], rtol=1e-12, atol=1e-13)


def test_kv_sharing_equivalence():
    """A consuming layer fed the K/V its own (absent) W_K, W_V rows would produce
    equals the standalone layer with those rows."""
    s, x, meta, p = _tiny(window=5)
    out_own, (k, v) = O.layer_forward(x, meta, p, s)
    wa, wkv = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
    w_in_c = np.concatenate([p["w_in"][:wa], p["w_in"][wa + 2 * wkv:]], axis=0)
    sc = dataclasses.replace(s, kv_mode=O.KV_CONSUME)
    out_c, _ = O.layer_forward(x, meta, dict(p, w_in=w_in_c), sc, kv_in=(k, v))
    np.testing.assert_allclose(out_c, out_own, rtol=1e-13, atol=1e-14)


def test_layer_matches_stagewise_hand_composition():
    """The layer equals its stages composed by hand for one sequence: in_proj split
    Q|K|V|X_ssm|G, attention, SSM with dt = softplus(...), gate, fusion, out_proj."""
    s, x, meta, p = _tiny(window=2)
    out, _ = O.layer_forward(x, meta, p, s)
    xt = np.concatenate([meta, x[1]], axis=0).astype(float)
    w_in = p["w_in"].astype(float)
    wa, wkv, di = 8, 4, 12
    q, k, v = xt @ w_in[:wa].T, xt @ w_in[wa:wa + wkv].T, xt @ w_in[wa + wkv:wa + 2 * wkv].T
    xs, g = xt @ w_in[wa + 2 * wkv:wa + 2 * wkv + di].T, xt @ w_in[wa + 2 * wkv + di:].T
    ya = O.attention(q, k, v, 2, 1, 3, 2)
    xdbc = xs @ p["w_x"].T.astype(float)
    dt = np.log1p(np.exp(xdbc[:, :2] @ p["w_dt"].T.astype(float) + p["b_dt"]))
    y = O.selective_scan(xs, dt, -np.exp(p["a_log"].astype(float)), xdbc[:, 2:6], xdbc[:, 6:10])
    ys = g * scipy.special.expit(g) * y
    z = np.concatenate([p["beta1"] * O.rms_normalize(ya, 1e-6), p["beta2"] * O.rms_normalize(ys, 1e-6)], 1)
    np.testing.assert_allclose(out[1], z @ p["w_out"].T.astype(float), rtol=1e-12, atol=1e-13)


def test_stack_residual_identities():
    """Zero out_proj and zero FFN down weights leave h = X~; one block equals
    h + mixer(norm h) then + ffn(norm h) composed by hand."""
    s = _tiny_shape(window=3, ffn_dim=10)
    wl = synth.Workload("t", [s, dataclasses.replace(s, kv_mode=O.KV_CONSUME)], 3, 1e-3, False, "t")
    wl.layers[0] = dataclasses.replace(s, kv_mode=O.KV_PRODUCE)
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(2)]
    zero = [dict(p, w_out=np.zeros_like(p["w_out"]), w_down=np.zeros_like(p["w_down"])) for p in ps]
    np.testing.assert_allclose(O.stack_forward(x, meta, zero, wl.layers), O.meta_prepend(x, meta), rtol=0)
    h = O.meta_prepend(x, meta)
    mix, _ = O.layer_forward(O.rms_normalize(h, 1e-6), None, ps[0], wl.layers[0])
    h1 = h + mix
    h1 = h1 + O.swiglu_ffn(O.rms_normalize(h1, 1e-6), ps[0]["w_gate_up"], ps[0]["w_down"])
    np.testing.assert_allclose(O.stack_forward(x, meta, ps[:1], wl.layers[:1]), h1, rtol=1e-13)


def test_swiglu_by_hand():
    x = RNG.standard_normal((3, 4))
    wgu, wd = RNG.standard_normal((6, 4)), RNG.standard_normal((4, 3))
    gate, up = x @ wgu[:3].T, x @ wgu[3:].T
    ref = (gate / (1 + np.exp(-gate)) * up) @ wd.T
    np.testing.assert_allclose(O.swiglu_ffn(x, wgu, wd), ref, rtol=1e-13)


def test_stack_kv_pairing_uses_producer_kv():
    """The consuming block reads the K/V of the block before it: changing the
    producer's W_K rows changes the consumer's attention input."""
    s = _tiny_shape(window=-1, ffn_dim=6)
    layers = [dataclasses.replace(s, kv_mode=O.KV_PRODUCE), dataclasses.replace(s, kv_mode=O.KV_CONSUME)]
    wl = synth.Workload("t", layers, 5, 1e-3, False, "t")
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i) for i in range(2)]
    h, hidden = O.stack_forward(x, meta, ps, layers, return_hidden=True)
    ps2 = [dict(ps[0]), ps[1]]
    w = ps2[0]["w_in"].copy(); w[8:12] *= 2.0          # producer's W_K rows
    ps2[0]["w_in"] = w
    ps2[0]["w_out"] = np.zeros_like(ps[0]["w_out"]); ps2[0]["w_down"] = np.zeros_like(ps[0]["w_down"])
    ps3 = [dict(ps2[0], w_in=ps[0]["w_in"]), ps[1]]
    a = O.stack_forward(x, meta, ps2, layers)
    b = O.stack_forward(x, meta, ps3, layers)
    assert np.abs(a - b).max() > 1e-6


def test_stack_prenorm_gains_fold_into_the_following_weights():
    """Gains g1, g2 of the two pre-norms of a block equal unit gains with g1 folded into the
    columns of W_in and g2 into the columns of W_gate_up (W (g * u) = (W diag g) u): two
    stacks that differ only in where the gain sits give the same output; a gain of c * 1
    on a block's pre-norm is not a no-op (the norm's output is rescaled, not re-normalised)."""
    s = _tiny_shape(window=3, ffn_dim=10)
    layers = [dataclasses.replace(s, kv_mode=O.KV_PRODUCE), dataclasses.replace(s, kv_mode=O.KV_CONSUME)]
    wl = synth.Workload("t", layers, 6, 1e-3, False, "t")
    x, meta = synth.layer_inputs(wl)
    ps = [synth.layer_params(wl, i, norm_gains=True) for i in range(2)]
    assert ps[0]["norm1"].shape == (s.d_model,) and not np.allclose(ps[0]["norm1"], 1.0)
    folded = []
    for p in ps:
        q = {k: v for k, v in p.items() if k not in ("norm1", "norm2")}
        q["w_in"] = p["w_in"].astype(float) * p["norm1"][None, :]
        q["w_gate_up"] = p["w_gate_up"].astype(float) * p["norm2"][None, :]
        folded.append(q)
    np.testing.assert_allclose(O.stack_forward(x, meta, ps, layers), O.stack_forward(x, meta, folded, layers),
                               rtol=1e-11, atol=1e-12)
    unit = [{k: v for k, v in p.items() if k not in ("norm1", "norm2")} for p in ps]
    scaled = [dict(u, norm1=np.full(s.d_model, 2.0)) for u in unit]
    assert np.abs(O.stack_forward(x, meta, scaled, layers) - O.stack_forward(x, meta, unit, layers)).max() > 1e-3
    np.testing.assert_allclose(O.rms_norm(np.full((1, 4), -3.0), 0.0, np.array([1.0, 2.0, 3.0, 4.0])),
                               [[-1.0, -2.0, -3.0, -4.0]], rtol=1e-15)


@pytest.mark.parametrize("window,kv", [(-1, O.KV_OWN), (3, O.KV_PRODUCE), (2, O.KV_CONSUME)])
def test_layer_forward_rows_equals_the_full_layer_rows(window, kv):
    """The row-subset layer (projections and scan over every row, attention and out_proj
    for the listed rows only) returns exactly those rows of the full layer, including
    rows past window + meta and the last row."""
    s = dataclasses.replace(_tiny_shape(window=window, batch=1), kv_mode=kv)
    wl = synth.Workload("t", [s], 7, 1e-3, False, "t")
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    kv_in = None
    if kv == O.KV_CONSUME:
        T = s.T
        kv_in = (RNG.standard_normal((1, T, s.kv_width)), RNG.standard_normal((1, T, s.kv_width)))
    full, _ = O.layer_forward(x, meta, p, s, kv_in=kv_in)
    rows = np.array([0, 1, s.n_meta, s.T // 2, s.T - 1])
    np.testing.assert_allclose(O.layer_forward_rows(x, meta, p, s, rows, kv_in=kv_in), full[0][rows],
                               rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# Mamba options (causal conv + SiLU, D skip) and the fusion variants (group norm, difference)

def test_causal_conv_equals_a_library_fir_filter_per_channel():
    """out[:, c] = b[c] + FIR filter of x[:, c] with taps w[c, ::-1] (scipy.signal.lfilter),
    i.e. a causal convolution whose rows before the first read as zero."""
    import scipy.signal
    T, Di, K = 19, 5, 4
    x = RNG.standard_normal((T, Di))
    w = RNG.standard_normal((Di, K))
    b = RNG.standard_normal(Di)
    out = O.causal_conv1d(x, w, b)
    for c in range(Di):
        np.testing.assert_allclose(out[:, c], b[c] + scipy.signal.lfilter(w[c, ::-1], [1.0], x[:, c]), rtol=1e-12,
                                   atol=1e-13)


def test_causal_conv_is_causal_and_width_one_identity():
    T, Di, K = 12, 3, 4
    x = RNG.standard_normal((2, T, Di))
    w, b = RNG.standard_normal((Di, K)), RNG.standard_normal(Di)
    a = O.causal_conv1d(x, w, b)
    x2 = x.copy()
    x2[:, 7] += 5.0
    c2 = O.causal_conv1d(x2, w, b)
    np.testing.assert_array_equal(a[:, :7], c2[:, :7])
    assert np.abs(a[:, 7:7 + K] - c2[:, 7:7 + K]).min() > 0       # rows t..t+K-1 see row t
    np.testing.assert_array_equal(a[:, 7 + K:], c2[:, 7 + K:])     # and no later row
    np.testing.assert_allclose(O.causal_conv1d(x, np.ones((Di, 1)), np.zeros(Di)), x, rtol=0)


def test_d_skip_alone_when_c_is_zero_and_conv_feeds_x_proj_and_scan():
    """With W_x's C rows zero the scan output is 0, so Y = SiLU(G) * D * x with x the head's
    input -- SiLU(conv(X_ssm) + b) when the conv is on; without D and conv the branch is
    unchanged."""
    T, Di, N, R = 9, 6, 3, 2
    xs, g = RNG.standard_normal((T, Di)), RNG.standard_normal((T, Di))
    w_x = RNG.standard_normal((R + 2 * N, Di))
    w_x[R + N:] = 0.0
    w_dt, b_dt, a_log = RNG.standard_normal((Di, R)), RNG.standard_normal(Di), RNG.uniform(0, 2, Di)
    D = RNG.uniform(0.5, 1.5, Di)
    w_c, b_c = RNG.standard_normal((Di, 4)), RNG.standard_normal(Di)
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    y = O.ssm_branch(xs, g, w_x, w_dt, b_dt, a_log, N, R, d_skip=D)
    np.testing.assert_allclose(y, g * sig(g) * D * xs, rtol=1e-12)
    xc = O.causal_conv1d(xs, w_c, b_c)
    y = O.ssm_branch(xs, g, w_x, w_dt, b_dt, a_log, N, R, w_conv=w_c, b_conv=b_c, d_skip=D)
    np.testing.assert_allclose(y, g * sig(g) * D * xc * sig(xc), rtol=1e-12)
    w_x2 = RNG.standard_normal((R + 2 * N, Di))
    np.testing.assert_array_equal(O.ssm_branch(xs, g, w_x2, w_dt, b_dt, a_log, N, R),
                                  O.ssm_branch(xs, g, w_x2, w_dt, b_dt, a_log, N, R, d_skip=None))


def test_group_norm_closed_forms():
    """Groups of constant values c_j normalise to sign(c_j) (eps 0); every group has unit RMS;
    one group over the whole width is the plain RMSNorm."""
    c = np.array([3.0, -0.5, 2.0, -7.0])
    v = np.repeat(c, 4)[None, :]
    np.testing.assert_allclose(O.rms_normalize_groups(v, 0.0, 4), np.repeat(np.sign(c), 4)[None, :], rtol=1e-15)
    z = RNG.standard_normal((5, 24))
    n = O.rms_normalize_groups(z, 0.0, 8).reshape(5, 3, 8)
    np.testing.assert_allclose(np.sqrt((n * n).mean(-1)), 1.0, rtol=1e-13)
    np.testing.assert_array_equal(O.rms_normalize_groups(z, 1e-6, 24), O.rms_normalize(z, 1e-6))
    np.testing.assert_array_equal(O.rms_normalize_groups(z, 1e-6, 0), O.rms_normalize(z, 1e-6))


def test_difference_fusion_identity():
    """out(difference) + out(sum) = 2 out(beta2 = 0): the SSM branch enters with the opposite
    sign and the attention branch is unchanged (eps tiny, so both branches normalise to
    unit RMS)."""
    s, x, meta, p = _tiny(rms_eps=1e-14)
    sd = dataclasses.replace(s, fusion=1)
    o_sum, _ = O.layer_forward(x, meta, p, s)
    o_dif, _ = O.layer_forward(x, meta, p, sd)
    o_att, _ = O.layer_forward(x, meta, dict(p, beta2=np.zeros_like(p["beta2"])), s)
    np.testing.assert_allclose(o_sum + o_dif, 2.0 * o_att, rtol=1e-11, atol=1e-12)
    assert np.abs(o_sum - o_dif).max() > 1e-3


def test_layer_with_every_option_matches_its_hand_composition():
    """Conv + D skip + group norm + difference through layer_forward equal the stages
    composed by hand for one sequence."""
    s = _tiny_shape(batch=1, conv_width=4, d_skip=1, norm_group=4, fusion=1, window=3)
    wl = synth.Workload("t", [s], 8, 1e-3, False, "t")
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    assert p["w_conv"].shape == (s.d_inner, 4) and p["d_skip"].shape == (s.d_inner,)
    out, _ = O.layer_forward(x, meta, p, s)
    xt = O.meta_prepend(x, meta)[0]
    parts = O.split_in_proj(xt @ p["w_in"].T.astype(float), s)
    ya = O.attention(parts["q"], parts["k"], parts["v"], s.n_q_heads, s.n_kv_heads, s.n_meta, s.window)
    xc = O.causal_conv1d(parts["x_ssm"], p["w_conv"], p["b_conv"])
    xc = xc / (1.0 + np.exp(-xc))
    xdbc = xc @ p["w_x"].T.astype(float)
    dt = np.log1p(np.exp(xdbc[:, :s.dt_rank] @ p["w_dt"].T.astype(float) + p["b_dt"]))
    y = O.selective_scan(xc, dt, -np.exp(p["a_log"].astype(float)), xdbc[:, s.dt_rank:s.dt_rank + s.d_state],
                         xdbc[:, s.dt_rank + s.d_state:])
    ys = parts["g_raw"] * scipy.special.expit(parts["g_raw"]) * (y + p["d_skip"] * xc)
    grp = lambda v: (v.reshape(v.shape[0], -1, 4) / np.sqrt((v.reshape(v.shape[0], -1, 4) ** 2).mean(-1, keepdims=True)
                                                                + 1e-6)).reshape(v.shape)
    z = np.concatenate([p["beta1"] * grp(ya), -p["beta2"] * grp(ys)], 1)
    np.testing.assert_allclose(out[0], z @ p["w_out"].T.astype(float), rtol=1e-11, atol=1e-12)
