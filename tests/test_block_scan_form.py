"""The block form of the selective scan that the tensor-core kernel evaluates (CPU).

The SSM head's output is the mixing-matrix product of the Hymba review's "Design
formulation": y_i = G_i . sum_{j<=i} C_i (prod_{k=j+1..i} exp(A dt_k)) B_j dt_j x_j.
With one decay rate per channel, inside a block of Q steps the decay product factors as
2^(r - lambda_t) 2^(lambda_s - r) (lambda the block's running sum of |A| dt / ln 2, r a
reference inside the block), so a block's output is two small matrix products shared by
all channels plus a carried state:

    y[t,c] = W[c,t] (sum_s V[c,s] M[t,s] + sum_n G'[c,n] C[t,n]),
    V = dt x 2^(lambda - r),  W = gate 2^(r - lambda),  M = tril(C B^T),  G' = h_in 2^(-r),
    h_out = 2^(-lambda_last) h_in + 2^(r - lambda_last) V B.

This file writes that algorithm out in numpy and checks it against the oracle's plain
recurrence: to rounding in fp64, and within the bound the parity tests allow when the
products take tf32 operands (as the kernel's do).  It also checks the guard the kernel
uses: a block whose half-block decay sums leave the range of the factors runs the plain
recurrence instead.  Nothing here imports the CUDA path."""
import numpy as np
import pytest

import oracle as O
from hybrid_attention_ssm_hymba_b200 import synth

Q = 64
RANGE = 100.0   # max half-block decay sum (log2 units) for the factored form


def _tf32(a):
    """Round to the tf32 significand (10 explicit bits), ties away from zero."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x1000) & 0xFFFFE000).astype(np.uint32)).view(np.float32).astype(np.float64)


def block_scan(x, dt, a_log, Bm, Cm, gate, tf32=False):
    """The block algorithm for one sequence: x, dt, gate [T, Di]; Bm, Cm [T, N]; a_log
    [Di].  Returns (y [T, Di], number of blocks run as the plain recurrence)."""
    rnd = _tf32 if tf32 else (lambda v: v)
    T, Di = x.shape
    N = Bm.shape[1]
    A2 = np.exp(a_log) / np.log(2.0)          # |A| / ln 2: exp(A dt) = 2^(-A2 dt)
    h = np.zeros((Di, N))
    y = np.zeros((T, Di))
    plain = 0
    for t0 in range(0, T, Q):
        n = min(Q, T - t0)
        pad = lambda a: np.concatenate([a[t0:t0 + n], np.zeros((Q - n,) + a.shape[1:])])  # noqa: E731
        d, xx, g, B, C = pad(dt), pad(x), pad(gate), pad(Bm), pad(Cm)
        S0, S1 = (A2 * d[:Q // 2]).sum(0), (A2 * d[Q // 2:]).sum(0)
        if (S0 > RANGE).any() or (S1 > RANGE).any():
            plain += 1
            for t in range(n):
                h = np.exp2(-A2 * d[t])[:, None] * h + (d[t] * xx[t])[:, None] * B[t][None]
                y[t0 + t] = g[t] * (h @ C[t])
            continue
        mu = np.cumsum(A2 * d, 0) - S0[None]   # lambda - r, r = lambda after Q/2 steps
        V = rnd(d * xx * np.exp2(mu))          # [s, c]
        W = g * np.exp2(-mu)                   # [t, c]
        M = rnd(np.tril(rnd(C) @ rnd(B).T))    # [t, s]
        Gp = rnd(h * np.exp2(-S0)[:, None])    # [c, n]
        Y = M @ V + rnd(C) @ Gp.T              # [t, c]
        y[t0:t0 + n] = (W * Y)[:n]
        h = np.exp2(-(S0 + S1))[:, None] * h + np.exp2(-S1)[:, None] * (V.T @ rnd(B))
    return y, plain


def _case(T, Di, seed, dt_hi=None):
    inp = synth.scan_inputs(seed, 1, T, Di, 16, dtype="bf16")
    if dt_hi is not None:   # runs of very large dt: the guard's plain recurrence
        dt = inp["dt"].copy()
        dt[T // 3:T // 3 + 20, 1] = dt_hi
        inp["dt"] = dt
    f = lambda k: inp[k].astype(np.float64)  # noqa: E731
    bc = f("bc")
    ref = f("g") * O.selective_scan(f("x"), f("dt"), O.ssm_decay_rate(inp["a_log"]), bc[:, :16], bc[:, 16:])
    return inp, f, bc, ref


@pytest.mark.parametrize("T,Di", [(64, 8), (150, 12), (300, 16)])
def test_block_form_equals_the_recurrence_in_fp64(T, Di):
    inp, f, bc, ref = _case(T, Di, 31)
    y, plain = block_scan(f("x"), f("dt"), f("a_log"), bc[:, :16], bc[:, 16:], f("g"))
    assert plain == 0
    assert np.abs(y - ref).max() <= 1e-10 * np.abs(ref).max()


def test_block_form_with_tf32_operands_stays_within_the_bf16_bound():
    inp, f, bc, ref = _case(700, 24, 32)
    y, plain = block_scan(f("x"), f("dt"), f("a_log"), bc[:, :16], bc[:, 16:], f("g"), tf32=True)
    e = np.abs(y - ref).max() / np.abs(ref).max()
    assert plain == 0 and 1e-6 < e < 2e-3   # tf32-sized error, far inside the 2e-2 bound


def test_blocks_beyond_the_factored_range_run_the_recurrence():
    inp, f, bc, ref = _case(400, 8, 33, dt_hi=6.0)
    y, plain = block_scan(f("x"), f("dt"), f("a_log"), bc[:, :16], bc[:, 16:], f("g"))
    assert plain >= 1
    assert np.abs(y - ref).max() <= 1e-10 * np.abs(ref).max()
