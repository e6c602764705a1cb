"""Per-kernel parity on the GPU against the fp64 oracle, through the C ABI.

Small and ragged shapes are compared element by element; the full workload
shapes run in the same launch configuration as the layer and are compared on
sampled outputs the oracle computes one by one (rows of a GEMM, channels of the
scan, query rows of the attention)."""
import math

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
import oracle as O
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, fp32, requires_cuda, status_ok, to_np

pytestmark = [pytest.mark.gpu, requires_cuda]

DT = {"bf16": H.HYMBA_BF16, "f32": H.HYMBA_F32}


# --------------------------------------------------------------------------- GEMM

@pytest.mark.parametrize("dtype,M,N,K", [
    ("bf16", 128, 256, 64), ("bf16", 333, 96, 1000), ("bf16", 1000, 4608, 1024), ("bf16", 257, 352, 96),
    ("bf16", 130, 128, 64), ("bf16", 1, 16, 8), ("bf16", 4099, 512, 136),
    ("f32", 100, 70, 50), ("f32", 72, 704, 128), ("f32", 1, 1, 1),
])
def test_gemm_parity(dtype, M, N, K):
    a = synth.matrix(11, "s_x", (M, K), 1.0, dtype)
    w = synth.matrix(12, "s_w", (N, K), 0.05, dtype)
    ta, tw = dev(a, dtype), dev(w, dtype)
    c = host.empty((M, N), dtype)
    ws = host.workspace(256)
    H.check(H.hymba_gemm(ta, tw, c, M, N, K, DT[dtype], ws), "gemm")
    status_ok(ws)
    assert_close(to_np(c), O.linear(a, w), dtype, f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(16640, 4608, 1024), (33280, 2048, 6144), (33792, 11264, 2048)])
def test_gemm_full_size_sampled_rows(M, N, K):
    """in_proj / out_proj shapes of the workloads; 48 sampled rows checked exactly."""
    rng = np.random.default_rng(0)
    a = synth.matrix(13, "s_x", (M, K), 1.0, "bf16")
    w = synth.matrix(14, "s_w", (N, K), 0.02, "bf16")
    c = host.empty((M, N), "bf16")
    ws = host.workspace(256)
    H.check(H.hymba_gemm(dev(a, "bf16"), dev(w, "bf16"), c, M, N, K, H.HYMBA_BF16, ws), "gemm")
    status_ok(ws)
    rows = np.unique(np.concatenate([rng.integers(0, M, 44), [0, 127, 128, M - 1]]))
    assert_close(to_np(c)[rows], O.linear(a[rows], w), "bf16", "gemm sampled rows")


# --------------------------------------------------------------------------- scan

def _scan_ref(inp, B, T, Di, N, chans=None):
    chans = np.arange(Di) if chans is None else np.asarray(chans)
    # a_log is [Di] or [Di, N] (per-state decay); ssm_decay_rate keeps the shape
    x = inp["x"].reshape(B, T, Di)[:, :, chans]
    dt = inp["dt"].reshape(B, T, Di)[:, :, chans]
    g = inp["g"].reshape(B, T, Di)[:, :, chans]
    bc = inp["bc"].reshape(B, T, 2 * N)
    y = O.selective_scan(x, dt, O.ssm_decay_rate(inp["a_log"][chans]), bc[..., :N], bc[..., N:])
    return (g * y).reshape(B * T, len(chans))


def _run_scan(inp, B, T, Di, N, dtype):
    y = host.empty((B * T, Di), dtype)
    ws = host.workspace(256)
    H.check(H.hymba_selective_scan(dev(inp["x"], dtype), dev(inp["dt"], dtype), fp32(inp["bc"]),
                                   dev(inp["g"], dtype), fp32(inp["a_log"]), y, Di, B, T, Di, N,
                                   DT[dtype], ws, a_per_state=int(inp["a_log"].ndim == 2)), "scan")
    status_ok(ws)
    return to_np(y)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T,Di,N", [(2, 300, 64, 16), (1, 1000, 48, 128), (1, 72, 256, 16),
                                      (3, 129, 40, 32), (1, 517, 24, 64), (1, 33, 16, 256),
                                      (1, 5, 32, 16)])
def test_scan_parity(dtype, B, T, Di, N):
    inp = synth.scan_inputs(21, B, T, Di, N, dtype=dtype)
    assert_close(_run_scan(inp, B, T, Di, N, dtype), _scan_ref(inp, B, T, Di, N), dtype, "scan")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,T", [(16, 1100), (32, 1500)])
def test_scan_extreme_decay_and_segments(dtype, N, T):
    """dt up to 6 with |A| up to 16: single steps decaying by more than 2^-60 and long
    runs of strong decay (the scaled-state fold and restart paths), over several
    512-step segments; plus a channel count that is not a multiple of 64."""
    B, Di = 2, 96
    inp = synth.scan_inputs(24, B, T, Di, N, dtype=dtype)
    g = np.random.default_rng(5)
    dt = np.exp(g.uniform(np.log(1e-3), np.log(6.0), size=(B * T, Di))).astype(np.float32)
    inp["dt"] = synth.round_bf16(dt) if dtype == "bf16" else dt
    assert_close(_run_scan(inp, B, T, Di, N, dtype), _scan_ref(inp, B, T, Di, N), dtype, "scan extreme decay")


def test_scan_block_form_hands_large_decay_blocks_to_the_recurrence():
    """bf16, d_state 16 (the tensor-core block form): a 64-step block in which some
    channel's half-block decay sum leaves the range of the factored form runs the plain
    recurrence for every channel of its 128-channel tile, and the state chain resumes
    after it.  Such blocks here sit between ordinary ones, in the first and in the second
    half of a block, in the second (partial) channel tile and in the ragged last block."""
    B, T, Di, N = 2, 700, 192, 16
    inp = synth.scan_inputs(25, B, T, Di, N)
    dt = inp["dt"].reshape(B, T, Di).astype(np.float32).copy()
    dt[0, 130:150, 7] = 6.0      # block 2, first half, tile 0
    dt[0, 360:380, 150] = 6.0    # block 5, second half, tile 1
    dt[1, 650:670, 100] = 6.0    # block 10 (60 steps), tile 0
    inp["dt"] = synth.round_bf16(dt.reshape(B * T, Di))
    assert_close(_run_scan(inp, B, T, Di, N, "bf16"), _scan_ref(inp, B, T, Di, N), "bf16", "scan mixed blocks")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T,Di,N", [(2, 300, 64, 16), (1, 200, 40, 32), (1, 130, 24, 128), (1, 33, 16, 256)])
def test_scan_per_state_decay(dtype, B, T, Di, N):
    """A_log [Di, N]: every state component decays at its own rate (the recurrence kernel),
    including channel counts that are not a multiple of the channels per block."""
    inp = synth.scan_inputs(26, B, T, Di, N, dtype=dtype, a_per_state=True)
    assert inp["a_log"].shape == (Di, N)
    assert_close(_run_scan(inp, B, T, Di, N, dtype), _scan_ref(inp, B, T, Di, N), dtype, "scan per-state A")


def test_scan_long_decay_small_dt():
    """dt down to 1e-4 over 32K steps: fp32 state keeps the long decay products."""
    B, T, Di, N = 1, 32896, 16, 128
    inp = synth.scan_inputs(22, B, T, Di, N, dt_min=1e-4)
    assert_close(_run_scan(inp, B, T, Di, N, "bf16"), _scan_ref(inp, B, T, Di, N), "bf16", "scan 32K")


@pytest.mark.parametrize("B,T,Di,N", [(8, 2080, 2048, 16), (1, 32896, 3072, 128)])
def test_scan_full_size_sampled_channels(B, T, Di, N):
    inp = synth.scan_inputs(23, B, T, Di, N)
    y = _run_scan(inp, B, T, Di, N, "bf16")
    chans = np.array([0, 1, 31, 32, 777, Di - 1])
    assert_close(y[:, chans], _scan_ref(inp, B, T, Di, N, chans), "bf16", "scan sampled channels")


# --------------------------------------------------------------------------- attention

def _attn_ref(q, kv, B, T, Hq, Hkv, dh, M, W, rows=None):
    out = []
    for b in range(B):
        qb = q[b * T:(b + 1) * T]
        kb, vb = kv[0, b * T:(b + 1) * T], kv[1, b * T:(b + 1) * T]
        r = np.arange(T) if rows is None else rows
        out.append(O.attention(qb[r], kb, vb, Hq, Hkv, M, W, rows=r))
    return np.concatenate(out)


def _run_attn(q, kv, B, T, Hq, Hkv, dh, M, W, dtype):
    out = host.empty((B * T, Hq * dh), dtype)
    out.fill_(float("nan"))
    ws = host.workspace(256)
    H.check(H.hymba_attention(dev(q, dtype), dev(kv, dtype), out, Hq * dh, B, T, Hq, Hkv, dh, M, W, DT[dtype],
                              ws), "attention")
    status_ok(ws)
    return to_np(out)


@pytest.mark.parametrize("B,T,Hq,Hkv,M,W", [
    (1, 72, 1, 1, 8, -1), (2, 300, 2, 1, 32, -1), (1, 700, 4, 2, 16, 100), (1, 1200, 2, 2, 128, 256),
    (1, 520, 1, 1, 0, 0), (1, 256, 2, 1, 8, 0), (1, 128, 1, 1, 0, -1), (1, 1, 1, 1, 0, -1),
    (2, 390, 4, 4, 24, 130), (1, 1300, 2, 1, 128, 1024),
])
def test_attention_parity_bf16(B, T, Hq, Hkv, M, W):
    dh = 128
    q, kv = synth.attention_inputs(31, B, T, Hq, Hkv, dh)
    assert_close(_run_attn(q, kv, B, T, Hq, Hkv, dh, M, W, "bf16"),
                 _attn_ref(q, kv, B, T, Hq, Hkv, dh, M, W), "bf16", f"attention T={T} M={M} W={W}")


@pytest.mark.parametrize("B,T,Hq,Hkv,dh,M,W", [(1, 72, 2, 2, 32, 8, -1), (2, 50, 4, 2, 64, 3, 5),
                                               (1, 33, 1, 1, 128, 0, 0), (1, 40, 2, 1, 16, 4, 7)])
def test_attention_parity_f32(B, T, Hq, Hkv, dh, M, W):
    q, kv = synth.attention_inputs(32, B, T, Hq, Hkv, dh, dtype="f32")
    assert_close(_run_attn(q, kv, B, T, Hq, Hkv, dh, M, W, "f32"),
                 _attn_ref(q, kv, B, T, Hq, Hkv, dh, M, W), "f32", "attention f32")


@pytest.mark.parametrize("B,T,Hq,Hkv,M,W", [(4, 8320, 16, 4, 128, 1024), (1, 32896, 12, 2, 128, 1024),
                                            (8, 2080, 2, 1, 32, -1)])
def test_attention_full_size_sampled_rows(B, T, Hq, Hkv, M, W):
    dh = 128
    q, kv = synth.attention_inputs(33, B, T, Hq, Hkv, dh)
    g = _run_attn(q, kv, B, T, Hq, Hkv, dh, M, W, "bf16")
    rows = np.array([0, 1, M - 1, M, 1000, 1151, 1152, 1153, 4095, T - 129, T - 1])
    rows = np.unique(rows[(rows >= 0) & (rows < T)])
    for b in sorted({0, B - 1}):
        ref = _attn_ref(q[b * T:(b + 1) * T], kv[:, b * T:(b + 1) * T], 1, T, Hq, Hkv, dh, M, W, rows)
        assert_close(g[b * T + rows], ref, "bf16", f"attention sampled rows b={b}")


# --------------------------------------------------------------------------- norms

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,wa,ws_", [(7, 256, 2048), (300, 64, 256), (33, 2048, 4096)])
def test_branch_norm_parity(dtype, rows, wa, ws_):
    z = synth.matrix(41, "s_z", (rows, wa + ws_), 0.7, dtype)
    b1 = synth.uniform(41, 0, "beta1", (wa,), 0.5, 1.5)
    b2 = synth.uniform(41, 0, "beta2", (ws_,), 0.5, 1.5)
    tz = dev(z, dtype)
    H.check(H.hymba_branch_norm(tz, fp32(b1), fp32(b2), rows, wa, ws_, 1e-6, DT[dtype]), "branch_norm")
    ref = O.branch_fusion(z[:, :wa], z[:, wa:], b1, b2, 1e-6)
    assert_close(to_np(tz), ref, dtype, "branch norm")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_rmsnorm_parity(dtype):
    x = synth.matrix(42, "s_z", (513, 2048), 2.0, dtype)
    tx = dev(x, dtype)
    y = host.empty(x.shape, dtype)
    H.check(H.hymba_rmsnorm(tx, y, 513, 2048, 1e-6, DT[dtype]), "rmsnorm")
    assert_close(to_np(y), O.rms_normalize(x, 1e-6), dtype, "rmsnorm")


# ------------------------------------------------------------------ scan with the dt projection

def _dtproj_ref(inp, B, T, Di, N, chans=None):
    chans = np.arange(Di) if chans is None else np.asarray(chans)
    dt = O.softplus(O.linear(inp["dt_low"], inp["w_dt"][chans]) + inp["b_dt"][chans].astype(np.float64))
    x = inp["x"].reshape(B, T, Di)[:, :, chans]
    g = inp["g"].reshape(B, T, Di)[:, :, chans]
    bc = inp["bc"].reshape(B, T, 2 * N)
    y = O.selective_scan(x, dt.reshape(B, T, len(chans)), O.ssm_decay_rate(inp["a_log"][chans]), bc[..., :N],
                         bc[..., N:])
    return (g * y).reshape(B * T, len(chans))


def _run_dtproj(inp, B, T, Di, N, dtype, y_ld=None):
    R = inp["dt_low"].shape[1]
    y_ld = Di if y_ld is None else y_ld
    y = host.empty((B * T, y_ld), dtype)
    y.zero_()   # columns past Di are not written
    ws = host.workspace(H.hymba_selective_scan_dtproj_workspace_size(B, T, Di, N, R, DT[dtype]))
    H.check(H.hymba_selective_scan_dtproj(dev(inp["x"], dtype), dev(inp["dt_low"], dtype), dev(inp["w_dt"], dtype),
                                          fp32(inp["b_dt"]), R, fp32(inp["bc"]), dev(inp["g"], dtype),
                                          fp32(inp["a_log"]), y, y_ld, B, T, Di, N, DT[dtype], ws), "scan dtproj")
    status_ok(ws)
    return to_np(y)[:, :Di]


@pytest.mark.parametrize("dtype,B,T,Di,N,R", [
    ("bf16", 2, 300, 256, 128, 128),   # tensor-core form, d_state 128: two dt atoms, ragged last block
    ("bf16", 1, 517, 200, 128, 96),    # second channel tile partial, dt_rank 96 (zero-filled atom tail)
    ("bf16", 3, 65, 128, 128, 64),     # one dt atom, three sequences
    ("bf16", 1, 31, 136, 128, 8),      # a single partial block, 8-wide dt projection
    ("bf16", 2, 64, 128, 128, 128),    # exactly one dt pair (two full blocks)
    ("bf16", 1, 33, 128, 128, 128),    # two blocks, the second a single step
    ("bf16", 2, 333, 192, 16, 64),     # d_state 16 tensor-core form
    ("bf16", 1, 100, 64, 64, 32),      # no tensor-core form: dt through the GEMM, then the scan
    ("f32", 2, 90, 48, 128, 40),
])
def test_scan_dtproj_parity(dtype, B, T, Di, N, R):
    inp = synth.scan_dtproj_inputs(31, B, T, Di, N, R, dtype=dtype)
    assert_close(_run_dtproj(inp, B, T, Di, N, dtype), _dtproj_ref(inp, B, T, Di, N), dtype, "scan dtproj")


def test_scan_dtproj_d128_output_row_stride():
    """y written into the SSM columns of a wider row (the layer's Z layout)."""
    B, T, Di, N, R = 2, 150, 256, 128, 128
    inp = synth.scan_dtproj_inputs(32, B, T, Di, N, R)
    assert_close(_run_dtproj(inp, B, T, Di, N, "bf16", y_ld=Di + 64), _dtproj_ref(inp, B, T, Di, N), "bf16",
                 "scan dtproj y_ld")


def test_scan_dtproj_d128_hands_large_decay_blocks_to_the_recurrence():
    """d_state 128 tensor-core form: a 32-step block where some channel's half-block decay
    sum leaves the factored form's range runs the plain recurrence on the state held in
    TMEM, and the block products resume after it.  dt is pushed up (to ~10) for one channel
    per case by a run of large dt_low rows times a positive W_dt row: in the first and in the
    second half of a block, in the second (partial) channel tile, in the ragged last block,
    and over a run spanning two blocks."""
    B, T, Di, N, R = 2, 300, 200, 128, 128
    inp = synth.scan_dtproj_inputs(33, B, T, Di, N, R)
    dl = inp["dt_low"].reshape(B, T, R).copy()
    wd = inp["w_dt"].copy()
    for c in (7, 150, 100, 60):
        wd[c] = np.abs(wd[c]) + 0.05
    # dt_low runs: rows are shared by all channels, so every channel with a positive-leaning
    # W_dt row sees them, the four above most strongly
    dl[0, 36:44] = 2.0     # block 1, first half
    dl[0, 120:124] = 2.0   # block 3, second half
    dl[1, 290:298] = 2.0   # block 9 (12 steps), ragged
    dl[1, 60:70] = 2.0     # across blocks 1 and 2
    inp["dt_low"] = synth.round_bf16(dl.reshape(B * T, R))
    inp["w_dt"] = synth.round_bf16(wd)
    dt = O.softplus(O.linear(inp["dt_low"], inp["w_dt"]) + inp["b_dt"].astype(np.float64))
    assert dt.max() > 5.0, "the runs must produce large dt"
    assert_close(_run_dtproj(inp, B, T, Di, N, "bf16"), _dtproj_ref(inp, B, T, Di, N), "bf16",
                 "scan dtproj mixed blocks")


@pytest.mark.parametrize("B,T,Di,N,R,dt_min", [(4, 8320, 4096, 128, 128, 1e-3), (1, 32896, 3072, 128, 96, 1e-4)])
def test_scan_dtproj_full_size_sampled_channels(B, T, Di, N, R, dt_min):
    """The 1.5B-shaped pair's and the 32K layer's scan shapes in the layer's launch
    configuration; channels from both ends of several 128-channel tiles checked exactly."""
    inp = synth.scan_dtproj_inputs(34, B, T, Di, N, R, dt_min=dt_min)
    y = _run_dtproj(inp, B, T, Di, N, "bf16")
    chans = np.array([0, 1, 127, 128, 777, Di - 1])
    assert_close(y[:, chans], _dtproj_ref(inp, B, T, Di, N, chans), "bf16", "scan dtproj sampled channels")


# ------------------------------------------------------------------ run-to-run repeatability

@pytest.mark.parametrize("N,R", [(128, 128), (16, 64)])
def test_scan_dtproj_is_repeatable_bit_for_bit(N, R):
    """The tensor-core scans are deterministic: the same inputs give the same bits on every
    call (a race between the state products and the state's rescale, or between an MMA
    reading TMEM and a later one writing it, shows up here first)."""
    B, T, Di = 3, 1200, 384
    inp = synth.scan_dtproj_inputs(42, B, T, Di, N, R)
    first = _run_dtproj(inp, B, T, Di, N, "bf16")
    for _ in range(4):
        np.testing.assert_array_equal(_run_dtproj(inp, B, T, Di, N, "bf16"), first)


def test_attention_is_repeatable_bit_for_bit():
    B, T, Hq, Hkv, M, W = 2, 1500, 8, 2, 64, 300
    q, kv = synth.attention_inputs(43, B, T, Hq, Hkv, 128)
    runs = []
    for _ in range(4):
        out = host.empty((B * T, Hq * 128), "bf16")
        ws = host.workspace(256)
        H.check(H.hymba_attention(dev(q, "bf16"), dev(kv, "bf16"), out, Hq * 128, B, T, Hq, Hkv, 128, M, W,
                                  H.HYMBA_BF16, ws), "attention")
        status_ok(ws)
        runs.append(to_np(out))
    for r in runs[1:]:
        np.testing.assert_array_equal(r, runs[0])
