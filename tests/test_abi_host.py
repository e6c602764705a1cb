"""CPU-side checks of the C ABI: the library loads, exports every entry point
declared in include/hymba.h, and validates arguments without touching a GPU."""
import os
import re

import pytest

import hybrid_attention_ssm_hymba_b200 as H
from hybrid_attention_ssm_hymba_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hymba.h")).read()
    return sorted(set(re.findall(r"HYMBA_API\s+[\w\s\*]+?\b(hymba_\w+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    lib = H.load()
    declared = _declared()
    assert len(declared) >= 11
    assert set(declared) == set(H.ENTRY_POINTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings():
    for s in range(6):
        assert H.hymba_status_string(s)
    assert "timed out" in H.hymba_status_string(H.HYMBA_ERR_TIMEOUT)


@pytest.mark.parametrize("name", synth.WORKLOAD_ORDER)
def test_every_workload_is_supported(name):
    wl = synth.workload(name)
    cfgs = [H.make_cfg(s) for s in wl.layers]
    for c in cfgs:
        assert H.hymba_workspace_size(c) > 0
    assert H.hymba_stack_workspace_size(cfgs) > 0


def _cfg(**kw):
    return H.make_cfg(synth.workload("hymba350m_layer").first, **kw)


@pytest.mark.parametrize("kw,expect", [
    (dict(batch=0), H.HYMBA_ERR_INVALID_ARG),
    (dict(seq_len=0), H.HYMBA_ERR_INVALID_ARG),
    (dict(n_meta=-1), H.HYMBA_ERR_INVALID_ARG),
    (dict(window=-2), H.HYMBA_ERR_INVALID_ARG),
    (dict(n_q_heads=3, n_kv_heads=2), H.HYMBA_ERR_INVALID_ARG),
    (dict(kv_mode=3), H.HYMBA_ERR_INVALID_ARG),
    (dict(head_dim=64), H.HYMBA_ERR_UNSUPPORTED),
    (dict(d_state=24), H.HYMBA_ERR_UNSUPPORTED),
    (dict(n_meta=12), H.HYMBA_ERR_UNSUPPORTED),
    (dict(a_per_state=2), H.HYMBA_ERR_INVALID_ARG),
    (dict(dt_rank=40), H.HYMBA_ERR_UNSUPPORTED),
    (dict(dtype=7), H.HYMBA_ERR_INVALID_ARG),
    (dict(conv_width=5), H.HYMBA_ERR_INVALID_ARG),
    (dict(conv_width=-1), H.HYMBA_ERR_INVALID_ARG),
    (dict(fusion=2), H.HYMBA_ERR_INVALID_ARG),
    (dict(norm_group=96), H.HYMBA_ERR_UNSUPPORTED),
    (dict(norm_group=512), H.HYMBA_ERR_UNSUPPORTED),
])
def test_layer_validation_rejects_before_launch(kw, expect):
    """Bad configs return their status without any CUDA call (this runs on a CPU machine)."""
    c = _cfg(**kw)
    assert H.hymba_workspace_size(c) == 0
    w = H.make_weights({k: 1 << 20 for k in ("w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt",
                                             "beta1", "beta2")})
    st = H.hymba_layer_fwd(1 << 20, 1 << 20, w, c, None, None, 1 << 20, 1 << 20, ws_bytes=1 << 40,
                           stream=0)
    assert st == expect


def test_layer_rejects_missing_pointers_and_small_workspace():
    c = _cfg()
    full = {k: 1 << 20 for k in ("w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt", "beta1", "beta2")}
    need = H.hymba_workspace_size(c)
    assert H.hymba_layer_fwd(None, 1 << 20, H.make_weights(full), c, None, None, 1 << 20, 1 << 20,
                             ws_bytes=need, stream=0) == H.HYMBA_ERR_INVALID_ARG
    partial = dict(full, w_out=None)
    assert H.hymba_layer_fwd(1 << 20, 1 << 20, H.make_weights(partial), c, None, None, 1 << 20,
                             1 << 20, ws_bytes=need, stream=0) == H.HYMBA_ERR_INVALID_ARG
    assert H.hymba_layer_fwd(1 << 20, 1 << 20, H.make_weights(full), c, None, None, 1 << 20, 1 << 20,
                             ws_bytes=need - 1, stream=0) == H.HYMBA_ERR_WORKSPACE
    # a consuming layer needs kv_in, a producing one kv_out
    for mode in (H.HYMBA_KV_CONSUME, H.HYMBA_KV_PRODUCE):
        cm = _cfg(kv_mode=mode)
        assert H.hymba_layer_fwd(1 << 20, 1 << 20, H.make_weights(full), cm, None, None, 1 << 20,
                                 1 << 20, ws_bytes=1 << 40, stream=0) == H.HYMBA_ERR_INVALID_ARG
    # misaligned workspace
    assert H.hymba_layer_fwd(1 << 20, 1 << 20, H.make_weights(full), c, None, None, 1 << 20,
                             (1 << 20) + 8, ws_bytes=1 << 40, stream=0) == H.HYMBA_ERR_INVALID_ARG


def test_stack_validation():
    wl = synth.workload("hymba1p5b_stack24", n_layers=2)
    cfgs = [H.make_cfg(s) for s in wl.layers]
    full = {k: 1 << 20 for k in ("w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt", "beta1", "beta2",
                                 "w_gate_up", "w_down")}
    ws = [H.make_weights(full)] * 2
    # consumer first is invalid
    bad = [cfgs[1], cfgs[0]]
    assert H.hymba_stack_fwd(1 << 20, 1 << 20, ws, bad, 1 << 20, 1 << 20, ws_bytes=1 << 40,
                             stream=0) == H.HYMBA_ERR_INVALID_ARG
    # FFN weights required when ffn_dim > 0
    ws2 = [H.make_weights(dict(full, w_down=None))] * 2
    assert H.hymba_stack_fwd(1 << 20, 1 << 20, ws2, cfgs, 1 << 20, 1 << 20, ws_bytes=1 << 40,
                             stream=0) == H.HYMBA_ERR_INVALID_ARG
    need = H.hymba_stack_workspace_size(cfgs)
    assert H.hymba_stack_fwd(1 << 20, 1 << 20, ws, cfgs, 1 << 20, 1 << 20, ws_bytes=need - 1,
                             stream=0) == H.HYMBA_ERR_WORKSPACE


def test_stage_validation():
    assert H.load().hymba_gemm(None, 1, 1, 8, 16, 8, 1, 1, 256, None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_gemm(1, 1, 1, 8, 24, 8, 1, 1, 256, None) == H.HYMBA_ERR_UNSUPPORTED
    assert H.load().hymba_gemm(1, 1, 1, 8, 16, 8, 1, 1, 16, None) == H.HYMBA_ERR_WORKSPACE
    assert H.load().hymba_selective_scan(1, 1, 1, 1, 1, 1, 64, 1, 10, 64, 24, 0, 1, 1, 256,
                                         None) == H.HYMBA_ERR_UNSUPPORTED
    assert H.load().hymba_selective_scan(1, 1, 1, 1, 1, 1, 64, 1, 10, 64, 16, 2, 1, 1, 256,
                                         None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_attention(1, 1, 1, 256, 1, 10, 2, 1, 64, 0, -1, 1, 1, 256,
                                    None) == H.HYMBA_ERR_UNSUPPORTED
    assert H.load().hymba_attention(1, 1, 1, 256, 1, 10, 3, 2, 128, 0, -1, 1, 1, 256,
                                    None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_branch_norm(1, 1, 1, 4, 12, 16, 1e-6, 1, None) == H.HYMBA_ERR_UNSUPPORTED
    assert H.load().hymba_rmsnorm(1, 1, 4, 0, 1e-6, 1, None) == H.HYMBA_ERR_INVALID_ARG


def test_no_cpu_fallback_when_library_missing(tmp_path, monkeypatch):
    from hybrid_attention_ssm_hymba_b200 import _abi
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        _abi.load(str(tmp_path / "libhymba.so"))


def test_noalloc_rejects_oversized_config_before_touching_a_gpu():
    """The allocation-free layer entry point validates its size limit on the host."""
    cfg = _cfg()   # the full 350M-shaped layer needs ~300 MB of intermediates
    assert H.hymba_workspace_size(cfg) > H.HYMBA_NOALLOC_SCRATCH_BYTES
    w = H.make_weights({k: 16 for k in ("w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt", "beta1", "beta2")})
    assert H.hymba_layer_fwd_noalloc(16, 16, w, cfg, None, None, 16, stream=0) == H.HYMBA_ERR_WORKSPACE
    assert H.hymba_layer_fwd_noalloc(16, 16, w, _cfg(batch=0), None, None, 16, stream=0) == H.HYMBA_ERR_INVALID_ARG


def test_layer_fuses_dt_proj_only_where_the_scan_computes_dt():
    """bf16 with d_state 16 and dt_rank <= 64 (the 350M-shaped layer) runs its dt
    projection inside the scan; fp32, dt_rank 128 and invalid configs do not."""
    from hybrid_attention_ssm_hymba_b200 import synth
    assert H.hymba_layer_fuses_dt_proj(H.make_cfg(synth.workload("hymba350m_layer").first))
    assert not H.hymba_layer_fuses_dt_proj(H.make_cfg(synth.workload("hymba1p5b_stack24").first))
    assert not H.hymba_layer_fuses_dt_proj(H.make_cfg(synth.workload("tiny_fp32").first))
    bad = H.make_cfg(synth.workload("hymba350m_layer").first)
    bad.batch = 0
    assert not H.hymba_layer_fuses_dt_proj(bad)


def test_per_state_decay_layer_is_accepted():
    """a_per_state = 1 (A_log [d_inner, d_state]) is a supported layer configuration: it has a
    workspace size and does not fold the dt projection into the scan."""
    from hybrid_attention_ssm_hymba_b200 import synth
    import dataclasses
    c = H.make_cfg(dataclasses.replace(synth.workload("hymba350m_layer").first, a_per_state=1))
    assert H.hymba_workspace_size(c) > 0
    assert not H.hymba_layer_fuses_dt_proj(c)


def test_generation_and_prefix_entry_points_validate_on_the_host():
    """Bad arguments of the generation and meta-prefix calls return before any CUDA call."""
    c = _cfg()
    full = H.make_weights({k: 1 << 20 for k in ("w_in", "w_x", "w_dt", "w_out", "a_log", "b_dt", "beta1", "beta2")})
    P = 1 << 20
    need = H.hymba_decode_workspace_size(c)
    assert need >= H.hymba_workspace_size(c) > 0
    # cache smaller than the prompt; pos outside the cache; missing state
    assert H.load().hymba_layer_prefill(P, P, full, c, P, c.seq_len, P, P, P, need, None) == H.HYMBA_ERR_INVALID_ARG
    T = c.seq_len + c.n_meta
    assert H.load().hymba_layer_decode(P, full, c, P, T, T, P, P, P, need, None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_layer_decode(P, full, c, P, T, -1, P, P, P, need, None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_layer_decode(P, full, c, P, T + 1, T, None, P, P, need, None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_layer_decode(P, full, c, P, T + 1, T, P, P, P, need - 1, None) == H.HYMBA_ERR_WORKSPACE
    # more than 8 query heads per KV head, or a head_dim that is not a multiple of 32: unsupported
    assert H.hymba_decode_workspace_size(_cfg(n_q_heads=16, n_kv_heads=1)) == 0
    # meta prefix: needs meta rows; record and workspace checked
    assert H.hymba_meta_prefix_size(_cfg(n_meta=0)) == 0
    rec = H.hymba_meta_prefix_size(c)
    assert rec > 0 and rec % 256 == 0
    assert H.load().hymba_meta_prefix(P, full, c, None, P + 8, P, 1 << 40, None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_meta_prefix(P, full, _cfg(kv_mode=H.HYMBA_KV_CONSUME), None, P, P, 1 << 40,
                                      None) == H.HYMBA_ERR_INVALID_ARG
    assert H.load().hymba_layer_fwd_prefixed(P, P, full, c, None, None, P, P, 16, None) == H.HYMBA_ERR_WORKSPACE
