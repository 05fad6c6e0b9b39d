"""Failure detection without a GPU fault.

Every wait of the forward on its own bulk copies is bounded.  With the wait
limit forced to zero a kernel gives up at its first wait, lets the copies
already issued land, records the failure and exits: in the call's own status
(the first 256 bytes of its workspace, read by mamba_check_status) and in the
library's sticky per-device fault word.  A full-pass CTA whose chunk summary
was never written records the failure and writes nothing, instead of starting
from a stale carry.  A launch the runtime rejects on the host returns
MM_ERR_CUDA.  In every case the context stays usable and the next (normal)
call is correct."""

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, gpu_fwd, np64, oracle_fwd, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu

MM_ERR_CUDA = 7
MM_ERR_TIMEOUT = 11


def _inputs(seed=71, L=200, D=64, B=2):
    inp = make_mixer_inputs_custom(B, L, D, act="bf16", seed=seed, h0_std=0.3)
    return inp, to_dev(inp)


def _outputs(inp):
    B, L, twoD = inp["xz"].shape
    D = twoD // 2
    return (torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((B, D, 16), float("nan"), device="cuda"),
            torch.zeros((B, D, 3), dtype=torch.bfloat16, device="cuda"))


def _workspace(inp):
    B, L, twoD = inp["xz"].shape
    # garbage contents: the status must not depend on the workspace being cleared
    return torch.randint(0, 255, (mm.workspace_size(B, L, twoD // 2),), dtype=torch.uint8, device="cuda")


def _check_parity(inp, y, h):
    ref = oracle_fwd(inp)
    assert_close(np64(y), ref["y"], "bf16", "y", stored_bf16=True)
    assert_close(np64(h), ref["h_last"], "bf16", "h_last")


def test_forced_copy_wait_timeout_is_reported_per_call_and_recoverable(monkeypatch):
    inp, dev = _inputs()
    ws = _workspace(inp)
    assert mm.fault_status(reset=True) == 0
    monkeypatch.setenv("MAMBA_MIXER_WAIT_LIMIT", "0")
    y, h, cs = _outputs(inp)
    gpu_fwd(dev, y=y, h_last=h, conv_state_out=cs, workspace=ws)
    assert mm.check_status(ws) == MM_ERR_TIMEOUT
    assert mm.fault_status() == MM_ERR_TIMEOUT
    assert mm.fault_status(reset=True) == MM_ERR_TIMEOUT
    assert mm.fault_status() == 0
    monkeypatch.delenv("MAMBA_MIXER_WAIT_LIMIT")
    # the next call on the same workspace replaces the status
    y, h, _ = gpu_fwd(dev, workspace=ws)
    assert mm.check_status(ws) == 0
    assert mm.fault_status() == 0
    _check_parity(inp, y, h)


def test_missing_chunk_summaries_stop_the_full_pass(monkeypatch):
    """Only the summary pass gives up: no summary of chunks 0..K-2 is written.
    The full pass's CTAs of chunks 1.. find the summaries missing, record it
    and write nothing -- no y computed from a stale carry -- while chunk 0,
    which needs no summary, completes."""
    monkeypatch.setenv("MAMBA_MIXER_CHUNKS", "4")
    inp, dev = _inputs(seed=72, L=512, D=64, B=1)
    ws = _workspace(inp)
    chunk_len = 128                       # 16 tiles of 32 tokens in 4 chunks
    monkeypatch.setenv("MAMBA_MIXER_SUMMARY_WAIT_LIMIT", "0")
    y, h, cs = _outputs(inp)
    gpu_fwd(dev, y=y, h_last=h, conv_state_out=cs, workspace=ws)
    assert mm.check_status(ws) == MM_ERR_TIMEOUT
    assert mm.fault_status(reset=True) == MM_ERR_TIMEOUT
    ref = oracle_fwd(inp)
    # chunk 0 is computed from h0 and is correct; every later token is untouched
    assert_close(np64(y[:, :chunk_len]), ref["y"][:, :chunk_len], "bf16", "y", stored_bf16=True)
    assert torch.isnan(y[:, chunk_len:].float()).all()
    assert torch.isnan(h).all()           # h_last belongs to the last chunk: not written
    monkeypatch.delenv("MAMBA_MIXER_SUMMARY_WAIT_LIMIT")
    y, h, _ = gpu_fwd(dev, workspace=ws)
    assert mm.check_status(ws) == 0
    _check_parity(inp, y, h)


def test_status_belongs_to_its_workspace(monkeypatch):
    """Two calls on two workspaces, queued back to back on one stream: the
    one that failed and the one that completed are told apart."""
    inp, dev = _inputs(seed=73)
    ws_a, ws_b = _workspace(inp), _workspace(inp)
    monkeypatch.setenv("MAMBA_MIXER_WAIT_LIMIT", "0")
    gpu_fwd(dev, workspace=ws_a)
    monkeypatch.delenv("MAMBA_MIXER_WAIT_LIMIT")
    y, h, _ = gpu_fwd(dev, workspace=ws_b)
    assert mm.check_status(ws_a) == MM_ERR_TIMEOUT
    assert mm.check_status(ws_b) == 0
    mm.fault_status(reset=True)
    _check_parity(inp, y, h)


def test_launch_rejected_on_the_host_returns_cuda_error(monkeypatch):
    """A launch configuration the runtime refuses (more shared memory than a
    CTA may have) is caught on the host: MM_ERR_CUDA, nothing reaches the
    GPU, and the next call runs normally."""
    inp, dev = _inputs(seed=74)
    monkeypatch.setenv("MAMBA_MIXER_TEST_LAUNCH_FAIL", "1")
    with pytest.raises(mm.MixerError) as exc:
        gpu_fwd(dev)
    assert exc.value.status == MM_ERR_CUDA
    monkeypatch.delenv("MAMBA_MIXER_TEST_LAUNCH_FAIL")
    ws = _workspace(inp)
    y, h, _ = gpu_fwd(dev, workspace=ws)
    assert mm.check_status(ws) == 0
    assert mm.fault_status() == 0
    _check_parity(inp, y, h)


def test_host_path_reports_a_failed_piece(monkeypatch):
    """mamba_mixer_fwd_host runs its pieces under one status epoch: a piece
    that gives up makes the call's status a failure."""
    inp = make_mixer_inputs_custom(1, 2048, 64, act="bf16", seed=75, h0_std=0.3)
    pin = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    params = {k: pin[k].cuda() if pin[k] is not None else None for k in ("conv_w", "conv_b", "dt_bias", "A", "Dskip")}
    ws = torch.empty(mm.host_workspace_size(1, 2048, 64), dtype=torch.uint8, device="cuda")

    def call():
        return mm.mixer_fwd_host(pin["xz"], params["conv_w"], params["conv_b"], pin["dt"], params["dt_bias"],
                                 params["A"], pin["Bm"], pin["Cm"], params["Dskip"], pin["h0"],
                                 pin["conv_state_in"], workspace=ws)

    monkeypatch.setenv("MAMBA_MIXER_WAIT_LIMIT", "0")
    call()
    assert mm.check_status(ws) == MM_ERR_TIMEOUT
    mm.fault_status(reset=True)
    monkeypatch.delenv("MAMBA_MIXER_WAIT_LIMIT")
    y, h, _ = call()
    assert mm.check_status(ws) == 0
    torch.cuda.synchronize()
    _check_parity(inp, y, h)
    assert np.isfinite(np64(y)).all()
