"""Failure detection without a GPU fault.

Every kernel of the library bounds its mbarrier waits: a wait that runs out records
HYMBA_ERR_TIMEOUT in the workspace's status word and the kernel returns, so the
context stays usable and the caller learns of it through hymba_workspace_status.
Here the failure is made on purpose, in the two forms that fault nothing:
  * on the host: the status word is written from the host, as a kernel would;
  * on the GPU: a wait that nothing ends, limited to a millisecond
    (hymba_check_wait_timeout), runs out and the kernel returns.
After each, the status is read and cleared and an ordinary layer call still works."""
import ctypes

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_hymba_b200 as H
from hybrid_attention_ssm_hymba_b200 import host, synth
from gpu_util import assert_close, dev, requires_cuda

import oracle as O


def test_wait_check_validates_arguments_on_the_host():
    """Argument checks run before any CUDA call (no GPU needed)."""
    fake = 1 << 20   # never dereferenced: the call returns before touching it
    lib = H.load()
    assert lib.hymba_check_wait_timeout(None, 256, 1000, None) == H.HYMBA_ERR_WORKSPACE
    assert lib.hymba_check_wait_timeout(ctypes.c_void_p(fake), 128, 1000, None) == H.HYMBA_ERR_WORKSPACE
    assert lib.hymba_check_wait_timeout(ctypes.c_void_p(fake), 256, 0, None) == H.HYMBA_ERR_INVALID_ARG
    assert lib.hymba_check_wait_timeout(ctypes.c_void_p(fake), 256, 2000000, None) == H.HYMBA_ERR_INVALID_ARG


def _small_layer_ok(ws):
    """A small bf16 layer on the same workspace, checked against the oracle."""
    wl = synth.workload("hymba350m_layer", batch=1, seq_len=130)
    s = wl.first
    x, meta = synth.layer_inputs(wl)
    p = synth.layer_params(wl, 0)
    cfg = H.make_cfg(s)
    assert ws.numel() >= H.hymba_workspace_size(cfg)
    out = host.empty((1, s.T, s.d_model), "bf16")
    H.check(H.hymba_layer_fwd(dev(x, "bf16"), dev(meta, "bf16"), H.make_weights(host.params_to_device(p, "bf16")),
                              cfg, None, None, out, ws), "layer after the timeout")
    assert H.hymba_workspace_status(ws) == H.HYMBA_OK
    ref, _ = O.layer_forward(x, meta, p, s)
    assert_close(out.float().cpu().numpy(), ref, "bf16", "layer after the timeout")


@pytest.mark.gpu
@requires_cuda
def test_status_word_written_from_the_host_is_reported_then_cleared():
    cfg = H.make_cfg(synth.workload("hymba350m_layer", batch=1, seq_len=130).first)
    ws = host.workspace(H.hymba_workspace_size(cfg))
    ws.view(torch.int32)[0] = H.HYMBA_ERR_TIMEOUT          # what a kernel whose wait ran out writes
    torch.cuda.synchronize()
    assert H.hymba_workspace_status(ws) == H.HYMBA_ERR_TIMEOUT
    assert int(ws.view(torch.int32)[0].item()) == 0          # read and cleared
    assert H.hymba_workspace_status(ws) == H.HYMBA_OK
    _small_layer_ok(ws)


@pytest.mark.gpu
@requires_cuda
@pytest.mark.parametrize("limit_us", [1000, 50])
def test_bounded_wait_runs_out_records_timeout_and_returns(limit_us):
    cfg = H.make_cfg(synth.workload("hymba350m_layer", batch=1, seq_len=130).first)
    ws = host.workspace(H.hymba_workspace_size(cfg))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    assert H.hymba_check_wait_timeout(ws, limit_us) == H.HYMBA_OK
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    assert ms >= 0.9 * limit_us / 1000.0, f"the wait gave up after {ms:.3f} ms, before its {limit_us} us limit"
    assert ms < 1000.0, f"the wait took {ms:.1f} ms"
    assert H.hymba_workspace_status(ws) == H.HYMBA_ERR_TIMEOUT
    assert H.hymba_workspace_status(ws) == H.HYMBA_OK
    _small_layer_ok(ws)
