"""fp64 CPU oracle for the forward (prefill) pass of Hymba's hybrid-head layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` do.  It shares no
code with the CUDA path (``hybrid_attention_ssm_hymba_b200``) and does not
import it; both are fed the same arrays by the seeded generator module.

Every function is the plain definition written out in float64 with numpy.  A
matrix product (``@``) is used as a library primitive; there is no blocking,
fusion or reordering beyond what the definitions state.  The attention is an
explicit masked softmax over each query row (no online rescaling) and the SSM
is the sequential recurrence, with the materialised alpha_ij matrix form kept
beside it as an independent checking mode.

Sources (web pages on Hymba, arXiv 2411.13676), cited by page and section:

* [R]  "Hymba: A Hybrid-head Architecture for Small Language Models" review,
       blog.outta.ai/m/421 -- sections "Design formulation" (X~, W_in_proj,
       attention head, alpha_ij, SSM head, total fusion formulation),
       "Combine global and local attention", "Cross-layer KV sharing",
       "Meta Tokens".
* [X]  metaphor-xennon.pages.dev "Hymba: hybrid attention-SSM heads" -- sections
       "混合头模块" (hybrid-head module diagram), "部分滑动窗口注意力" (partial SWA
       table), "可学习Meta-Tokens" (meta-token prepend), "层配置" (config dict),
       "PyTorch伪代码" (HymbaLayer pseudocode: RMSNorm per branch, 0.5-average).
* [S]  networkstorageforum.com summary, "Key Components of Hymba" (meta tokens
       as learned cache initialisation; blocks stacked with SWA and KV sharing).

Readings where the pages are silent or disagree (each also listed in the
design notes): attention scale 1/sqrt(head_dim); no positional encoding;
A = -exp(A_log) per channel (or per channel and state); [dt_low | B | C] =
x_proj(X_ssm) and dt = softplus(dt_low W_dt^T + b_dt); no conv1d and no D skip by
default (Mamba's causal depthwise conv + SiLU on X_ssm and its D skip are options);
RMSNorm over each branch's full width with eps and no separate gain by default (per-group
norm and difference fusion, from the intra-layer hybrid study, are options); the
branches of unequal width are combined as out_proj of their concatenation;
query i sees key j iff j <= i and (i - j <= W or j < M); meta rows are queries
under the same mask, run through the SSM from h = 0, and kept in the output;
the even layer of a pair produces K/V and the odd one consumes it; stacked
blocks are pre-norm residual around the mixer and a SwiGLU FFN.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute force, special cases that reduce to library
routines and the invariants the pages imply, and the generation step
(``layer_prefill_state``, ``layer_decode_step``) by ``tests/test_oracle_decode.py``
against the longer prefill it must reproduce.  No function is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

KV_OWN, KV_PRODUCE, KV_CONSUME = 0, 1, 2


def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# elementwise pieces

def softplus(z):
    """log(1 + e^z), evaluated without overflow.  Used for dt ([R] "Design
    formulation": Delta; the softplus discretisation is Mamba's, the reading
    stated above)."""
    z = f64(z)
    return np.logaddexp(0.0, z)


def silu(z):
    """z * sigmoid(z): the output gate G applied to the SSM head ([R] "Design
    formulation", Y_ssm = G . alpha(...) W_SSM X~ -- G = SiLU(W_G x~))."""
    z = f64(z)
    return z / (1.0 + np.exp(-z))


def rms_normalize(v, eps: float):
    """v / sqrt(mean(v^2) + eps) over the last axis: the per-branch norm(.) of
    [R] "Design formulation" (total fusion), an RMSNorm as in [X] "PyTorch伪代码"."""
    v = f64(v)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)


def rms_norm(v, eps: float, gain=None):
    """RMSNorm with a learnable per-feature gain (the pre-norms of the stacked blocks;
    gain None = unit gain): gain * v / sqrt(mean(v^2) + eps)."""
    y = rms_normalize(v, eps)
    return y if gain is None else y * f64(gain)


# ---------------------------------------------------------------------------
# meta tokens and projections

def meta_prepend(x, meta):
    """X~ = [Meta Tokens, X]: the same M learned rows in front of every sequence
    ([R] "Design formulation"; [X] "可学习Meta-Tokens")."""
    x = f64(x)
    if meta is None or len(meta) == 0:
        return x
    meta = f64(meta)
    B = x.shape[0]
    return np.concatenate([np.broadcast_to(meta, (B,) + meta.shape), x], axis=1)


def linear(x, w):
    """x W^T with W in [out, in] layout (library matrix product)."""
    return f64(x) @ f64(w).T


def split_in_proj(proj, s) -> Dict[str, np.ndarray]:
    """Split the fused projection W_in_proj = [W_Q, W_K, W_V, W_SSM, W_G]
    ([R] "Design formulation") into its five outputs (no K/V for a consumer)."""
    wa, wkv, di = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim, s.d_inner
    out, c = {}, 0
    out["q"] = proj[..., c:c + wa]; c += wa
    if s.kv_mode != KV_CONSUME:
        out["k"] = proj[..., c:c + wkv]; c += wkv
        out["v"] = proj[..., c:c + wkv]; c += wkv
    out["x_ssm"] = proj[..., c:c + di]; c += di
    out["g_raw"] = proj[..., c:c + di]; c += di
    assert c == proj.shape[-1]
    return out


# ---------------------------------------------------------------------------
# attention heads

def visible(i: int, j: int, n_meta: int, window: int) -> bool:
    """Causal, sliding-window attention with the meta tokens always visible
    ([R] "Combine global and local attention"; [R] "Meta Tokens"; [X]
    "部分滑动窗口注意力").  window < 0 means global causal attention."""
    if j > i:
        return False
    return window < 0 or (i - j) <= window or j < n_meta


def visibility_mask(T: int, n_meta: int, window: int, rows: Optional[np.ndarray] = None):
    """Boolean [len(rows), T] matrix of visible(i, j)."""
    i = np.arange(T) if rows is None else np.asarray(rows)
    j = np.arange(T)
    ii, jj = i[:, None], j[None, :]
    m = jj <= ii
    if window >= 0:
        m &= ((ii - jj) <= window) | (jj < n_meta)
    return m


def attention_probs(q, k, n_meta: int, window: int, rows: Optional[np.ndarray] = None):
    """Explicit masked softmax(Q K^T / sqrt(dh)) for one head: q [T or len(rows), dh],
    k [T, dh] -> [len(rows), T]  ([R] "Design formulation", attention head; the
    1/sqrt(dh) scale is the standard reading, the page prints none)."""
    q, k = f64(q), f64(k)
    T, dh = k.shape
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    s = (q @ k.T) / math.sqrt(dh)
    mask = visibility_mask(T, n_meta, window, rows)
    s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def attention(q, k, v, n_q_heads: int, n_kv_heads: int, n_meta: int, window: int,
              rows: Optional[np.ndarray] = None, row_block: int = 512):
    """Multi-head (GQA) attention for one sequence.

    q [T or len(rows), Hq*dh] (only the query rows listed in ``rows``, default
    all), k, v [T, Hkv*dh] -> [len(rows), Hq*dh].  Query head h reads K/V head
    h // (Hq / Hkv) (several query heads share one KV head, [X] "跨层KV缓存共享":
    KV sharing combined with GQA)."""
    q, k, v = f64(q), f64(k), f64(v)
    T = k.shape[0]
    dh = k.shape[1] // n_kv_heads
    group = n_q_heads // n_kv_heads
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), n_q_heads * dh))
    for h in range(n_q_heads):
        kh = k[:, (h // group) * dh:(h // group + 1) * dh]
        vh = v[:, (h // group) * dh:(h // group + 1) * dh]
        qh = q[:, h * dh:(h + 1) * dh]
        for r0 in range(0, len(rows), row_block):
            rr = rows[r0:r0 + row_block]
            p = attention_probs(qh[r0:r0 + row_block], kh, n_meta, window, rr)
            out[r0:r0 + row_block, h * dh:(h + 1) * dh] = p @ vh
    return out


# ---------------------------------------------------------------------------
# SSM heads

def ssm_decay_rate(a_log):
    """A = -exp(A_log): the continuous-time state matrix (diagonal), one value
    per channel (or per channel and state)."""
    return -np.exp(f64(a_log))


def selective_scan(x, dt, A, Bm, Cm, h0=None, return_state=False):
    """Sequential recurrence of the selective SSM ([R] "Design formulation"):

        h_t = exp(A dt_t) h_{t-1} + dt_t B_t x_t,   y_t = C_t . h_t,   h_{-1} = 0

    x, dt [T, Di]; A [Di] (or [Di, N]); Bm, Cm [T, N] -> y [T, Di].
    Leading batch axes are allowed on x, dt, Bm, Cm."""
    x, dt, A, Bm, Cm = f64(x), f64(dt), f64(A), f64(Bm), f64(Cm)
    lead = x.shape[:-2]
    T, Di = x.shape[-2:]
    N = Bm.shape[-1]
    A2 = A[:, None] if A.ndim == 1 else A                       # [Di, 1] or [Di, N]
    h = np.zeros(lead + (Di, N)) if h0 is None else f64(h0).copy()
    y = np.empty(lead + (T, Di))
    for t in range(T):
        d = dt[..., t, :, None]                                 # [..., Di, 1]
        a = np.exp(A2 * d)                                      # exp(A dt_t)
        h = a * h + (d * x[..., t, :, None]) * Bm[..., t, None, :]
        y[..., t, :] = np.einsum("...cn,...n->...c", h, Cm[..., t, :])
    return (y, h) if return_state else y


def ssm_alpha_matrix(dt, A, Bm, Cm):
    """The materialised mixing matrix of the SSM head ([R] "Design formulation"):

        alpha_{i,j} = C_i ( prod_{k=j+1..i} exp(A Delta_k) ) B_j Delta_j ,  j <= i

    returned per channel: [Di, T, T] (zero above the diagonal).  With A per
    state the product runs per state and C_i . (...) B_j sums over states.
    Brute force, O(T^3 N Di): small T only."""
    dt, A, Bm, Cm = f64(dt), f64(A), f64(Bm), f64(Cm)
    T, Di = dt.shape
    N = Bm.shape[1]
    A2 = np.broadcast_to(A[:, None] if A.ndim == 1 else A, (Di, N))
    alpha = np.zeros((Di, T, T))
    for i in range(T):
        for j in range(i + 1):
            prod = np.ones((Di, N))
            for kk in range(j + 1, i + 1):
                prod = prod * np.exp(A2 * dt[kk][:, None])
            alpha[:, i, j] = (prod * Bm[j][None, :] * Cm[i][None, :]).sum(axis=1) * dt[j]
    return alpha


def ssm_from_alpha(x, alpha):
    """y_i = sum_{j<=i} alpha_{i,j} x_j per channel: alpha [Di, T, T], x [T, Di]."""
    return np.einsum("cij,jc->ic", f64(alpha), f64(x))


def causal_conv1d(x, w_conv, b_conv):
    """Depthwise causal convolution along time, the short convolution of a Mamba head
    ([R] "Design formulation" names the SSM head a Mamba head; the pages print no
    convolution, so it is an option): out[t, c] = b[c] + sum_{k<K} w[c, k] x[t-(K-1)+k, c],
    rows before the first one read as zero.  x [..., T, Di], w_conv [Di, K], b_conv [Di]."""
    x, w = f64(x), f64(w_conv)
    K, T = w.shape[1], x.shape[-2]
    out = np.zeros_like(x) + f64(b_conv)
    for k in range(K):
        shift = K - 1 - k
        out[..., shift:, :] += w[:, k] * x[..., :T - shift, :]
    return out


def ssm_branch(x_ssm, g_raw, w_x, w_dt, b_dt, a_log, d_state: int, dt_rank: int, w_conv=None, b_conv=None,
               d_skip=None):
    """One sequence's SSM heads: x_proj -> (dt_low, B, C); dt = softplus(dt_low
    W_dt^T + b_dt); scan; gate.  x_ssm, g_raw [T, Di] -> Y_ssm [T, Di].
    Mamba options (not in the pages' formula): with w_conv the head's input is
    x = SiLU(conv(X_ssm) + b_conv) in place of X_ssm (for x_proj and the scan alike); with
    d_skip the output before the gate is y + D * x."""
    x = silu(causal_conv1d(x_ssm, w_conv, b_conv)) if w_conv is not None else f64(x_ssm)
    xdbc = linear(x, w_x)
    dt_low = xdbc[..., :dt_rank]
    Bm = xdbc[..., dt_rank:dt_rank + d_state]
    Cm = xdbc[..., dt_rank + d_state:dt_rank + 2 * d_state]
    dt = softplus(linear(dt_low, w_dt) + f64(b_dt))
    y = selective_scan(x, dt, ssm_decay_rate(a_log), Bm, Cm)
    if d_skip is not None:
        y = y + f64(d_skip) * x
    return silu(g_raw) * y


def _ssm_opts(p):
    return dict(w_conv=p.get("w_conv"), b_conv=p.get("b_conv"), d_skip=p.get("d_skip"))


# ---------------------------------------------------------------------------
# fusion, layer, stack

def rms_normalize_groups(v, eps: float, group: int = 0):
    """Group RMSNorm: each run of `group` consecutive features normalised on its own
    (group 0: the whole last axis, rms_normalize).  The intra-layer hybrid study
    summarised on the gist.science page finds group normalisation of the branch outputs
    effective; a group is read as one head's width."""
    v = f64(v)
    if not group or group == v.shape[-1]:
        return rms_normalize(v, eps)
    assert v.shape[-1] % group == 0
    g = v.reshape(v.shape[:-1] + (v.shape[-1] // group, group))
    return rms_normalize(g, eps).reshape(v.shape)


def branch_fusion(y_attn, y_ssm, beta1, beta2, eps: float, group: int = 0, difference: bool = False):
    """Z = [beta1 * norm(Y_attn) || beta2 * norm(Y_ssm)], the argument of W_out
    ([R] "Design formulation", total fusion formulation; the two branch widths
    differ, so the sum inside W_out(.) is taken as W_out applied to the
    concatenation, i.e. the sum of each branch mapped by its slice of W_out).
    Variants of the intra-layer hybrid study (gist.science page): norm per group of
    `group` features, and difference fusion, the SSM branch subtracted instead of added
    (its half of Z negated)."""
    sign = -1.0 if difference else 1.0
    return np.concatenate([f64(beta1) * rms_normalize_groups(y_attn, eps, group),
                           sign * f64(beta2) * rms_normalize_groups(y_ssm, eps, group)], axis=-1)


def _fusion_opts(s):
    return dict(group=getattr(s, "norm_group", 0), difference=bool(getattr(s, "fusion", 0)))


def layer_forward(x, meta, p: Dict[str, np.ndarray], s, kv_in: Optional[Tuple] = None,
                  return_parts: bool = False):
    """Forward pass of one hybrid-head layer.

    x [B, L, d] (meta given) or [B, T, d] (meta None: x already holds X~);
    p: weights in the generator's layouts; s: shape record with n_meta,
    n_q_heads, n_kv_heads, head_dim, window, d_inner, d_state, dt_rank,
    kv_mode, rms_eps.  kv_in = (K, V) [B, T, Hkv*dh] for a consuming layer.
    Returns out [B, T, d] (meta rows kept) and the layer's (K, V)."""
    xt = meta_prepend(x, meta)
    B, T, _ = xt.shape
    parts = split_in_proj(linear(xt, p["w_in"]), s)
    if s.kv_mode == KV_CONSUME:
        assert kv_in is not None, "a consuming layer needs the producer's K/V"
        k, v = f64(kv_in[0]), f64(kv_in[1])
    else:
        k, v = parts["k"], parts["v"]
    y_attn = np.stack([attention(parts["q"][b], k[b], v[b], s.n_q_heads, s.n_kv_heads,
                                 s.n_meta, s.window) for b in range(B)])
    y_ssm = np.stack([ssm_branch(parts["x_ssm"][b], parts["g_raw"][b], p["w_x"], p["w_dt"],
                                 p["b_dt"], p["a_log"], s.d_state, s.dt_rank, **_ssm_opts(p))
                      for b in range(B)])
    z = branch_fusion(y_attn, y_ssm, p["beta1"], p["beta2"], s.rms_eps, **_fusion_opts(s))
    out = linear(z, p["w_out"])
    if return_parts:
        return out, (k, v), dict(parts, y_attn=y_attn, y_ssm=y_ssm, z=z)
    return out, (k, v)


def layer_forward_rows(x, meta, p: Dict[str, np.ndarray], s, rows, kv_in: Optional[Tuple] = None):
    """Output rows ``rows`` of layer_forward for one sequence (x [1, L, d] or, with meta
    None, [1, T, d]): the projections and the SSM scan run over every row (each output row
    depends on all rows before it), the attention and out_proj only for the listed rows.
    kv_in = (K, V) [1, T, Hkv*dh] for a consuming layer.  Returns [len(rows), d]."""
    rows = np.asarray(rows)
    xt = meta_prepend(x, meta)
    parts = split_in_proj(linear(xt, p["w_in"]), s)
    if s.kv_mode == KV_CONSUME:
        assert kv_in is not None, "a consuming layer needs the producer's K/V"
        k, v = f64(kv_in[0]), f64(kv_in[1])
    else:
        k, v = parts["k"], parts["v"]
    y_attn = attention(parts["q"][0][rows], k[0], v[0], s.n_q_heads, s.n_kv_heads, s.n_meta, s.window,
                       rows=rows)
    y_ssm = ssm_branch(parts["x_ssm"][0], parts["g_raw"][0], p["w_x"], p["w_dt"], p["b_dt"], p["a_log"],
                       s.d_state, s.dt_rank, **_ssm_opts(p))[rows]
    return linear(branch_fusion(y_attn, y_ssm, p["beta1"], p["beta2"], s.rms_eps, **_fusion_opts(s)), p["w_out"])


# ---------------------------------------------------------------------------
# generation: one new token from the KV cache and the SSM state

def layer_prefill_state(x, meta, p: Dict[str, np.ndarray], s, kv_in: Optional[Tuple] = None):
    """layer_forward plus what generating the next token needs afterwards: the layer's
    K/V over all T rows (the attention heads' cache, [B, T, Hkv*dh] each) and the SSM
    heads' state after the last row, h_T [B, Di, N] -- the fixed-size state the SSM
    heads carry where attention keeps a growing cache ([R] "Efficiency and KV cache
    optimization").  Returns (out [B, T, d], (K, V), h_T)."""
    assert p.get("w_conv") is None, "the generation step carries no convolution state"
    out, (k, v), parts = layer_forward(x, meta, p, s, kv_in=kv_in, return_parts=True)
    hs = []
    for b in range(out.shape[0]):
        xdbc = linear(parts["x_ssm"][b], p["w_x"])
        dt = softplus(linear(xdbc[:, :s.dt_rank], p["w_dt"]) + f64(p["b_dt"]))
        _, h = selective_scan(parts["x_ssm"][b], dt, ssm_decay_rate(p["a_log"]),
                              xdbc[:, s.dt_rank:s.dt_rank + s.d_state],
                              xdbc[:, s.dt_rank + s.d_state:s.dt_rank + 2 * s.d_state], return_state=True)
        hs.append(h)
    return out, (k, v), np.stack(hs)


def layer_decode_step(x_t, p: Dict[str, np.ndarray], s, kv_cache: Tuple, h, pos: int):
    """One new token per sequence at row ``pos`` (the number of rows already in the
    cache, meta rows included): x_t [B, d] -> out_t [B, d].  The same definitions as
    layer_forward applied to row ``pos`` of a (pos + 1)-row sequence: the token's query
    attends over the cached keys and its own under the visibility rule (causal, window
    W, meta always visible); the SSM heads advance their state one step,
    h <- exp(A dt) h + dt x B, y = C . h ([R] "Design formulation").

    kv_cache = (K, V) [B, pos, Hkv*dh] for a layer with its own K/V (the new row is
    appended), or the producer's (K, V) [B, pos + 1, Hkv*dh] already holding the new row
    for a consuming layer.  h [B, Di, N].  Returns (out_t, (K, V) with pos + 1 rows,
    h_new)."""
    assert p.get("w_conv") is None, "the generation step carries no convolution state"
    xt = f64(x_t)[:, None, :]
    B = xt.shape[0]
    parts = split_in_proj(linear(xt, p["w_in"]), s)
    if s.kv_mode == KV_CONSUME:
        k, v = f64(kv_cache[0]), f64(kv_cache[1])
    else:
        k = np.concatenate([f64(kv_cache[0]), parts["k"]], axis=1)
        v = np.concatenate([f64(kv_cache[1]), parts["v"]], axis=1)
    assert k.shape[1] == pos + 1, "the cache must hold rows [0, pos]"
    y_attn = np.stack([attention(parts["q"][b], k[b], v[b], s.n_q_heads, s.n_kv_heads,
                                 s.n_meta, s.window, rows=np.array([pos])) for b in range(B)])
    A = ssm_decay_rate(p["a_log"])
    xdbc = linear(parts["x_ssm"], p["w_x"])
    dt = softplus(linear(xdbc[..., :s.dt_rank], p["w_dt"]) + f64(p["b_dt"]))
    ys, hs = [], []
    for b in range(B):
        y, hb = selective_scan(parts["x_ssm"][b], dt[b], A, xdbc[b, :, s.dt_rank:s.dt_rank + s.d_state],
                               xdbc[b, :, s.dt_rank + s.d_state:s.dt_rank + 2 * s.d_state], h0=h[b],
                               return_state=True)
        if p.get("d_skip") is not None:
            y = y + f64(p["d_skip"]) * parts["x_ssm"][b]
        ys.append(silu(parts["g_raw"][b]) * y)
        hs.append(hb)
    z = branch_fusion(y_attn, np.stack(ys), p["beta1"], p["beta2"], s.rms_eps, **_fusion_opts(s))
    return linear(z, p["w_out"])[:, 0], (k, v), np.stack(hs)


def swiglu_ffn(x, w_gate_up, w_down):
    """W_down( SiLU(x W_gate^T) * (x W_up^T) ); w_gate_up holds the gate rows
    then the up rows (FFN width from [X] "层配置": intermediate_size)."""
    F = w_gate_up.shape[0] // 2
    gu = linear(x, w_gate_up)
    return linear(silu(gu[..., :F]) * gu[..., F:], w_down)


def stack_forward(x, meta, params: Sequence[Dict[str, np.ndarray]], shapes: Sequence,
                  return_hidden: bool = False):
    """Stacked hybrid-head blocks ([S] "Key Components of Hymba": blocks stacked
    with sliding-window attention and cross-layer KV sharing; [R] "Cross-layer
    KV sharing": two consecutive layers share one KV cache).  Each block is
    h += mixer(RMSNorm_1(h)); h += SwiGLU(RMSNorm_2(h)), with the gains
    p["norm1"], p["norm2"] (unit gains when absent).
    Returns h [B, T, d] (and the list of per-block outputs if asked)."""
    h = meta_prepend(x, meta)
    kv = None
    hidden = []
    for p, s in zip(params, shapes):
        xn = rms_norm(h, s.rms_eps, p.get("norm1"))
        out, kv_l = layer_forward(xn, None, p, s, kv_in=kv if s.kv_mode == KV_CONSUME else None)
        if s.kv_mode != KV_CONSUME:
            kv = kv_l
        h = h + out
        if s.ffn_dim:
            h = h + swiglu_ffn(rms_norm(h, s.rms_eps, p.get("norm2")), p["w_gate_up"], p["w_down"])
        hidden.append(h)
    return (h, hidden) if return_hidden else h
