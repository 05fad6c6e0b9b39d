"""Failure detection without a GPU fault: every wait of the forward on its
own bulk copies is bounded.  With the wait limit forced to zero the kernel
gives up at its first wait, lets the copies already issued land, sets the
library's fault word and exits; the host reads the word, and the context
stays usable for the next (normal) call."""

import os

import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, gpu_fwd, np64, oracle_fwd, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu

MM_ERR_TIMEOUT = 11


def test_forced_copy_wait_timeout_is_reported_and_recoverable(monkeypatch):
    inp = make_mixer_inputs_custom(2, 200, 64, act="bf16", seed=71, h0_std=0.3)
    dev = to_dev(inp)
    assert mm.fault_status(reset=True) == 0
    monkeypatch.setenv("MAMBA_MIXER_WAIT_LIMIT", "0")
    gpu_fwd(dev)
    torch.cuda.synchronize()
    assert mm.fault_status() == MM_ERR_TIMEOUT
    assert mm.fault_status(reset=True) == MM_ERR_TIMEOUT
    assert mm.fault_status() == 0
    monkeypatch.delenv("MAMBA_MIXER_WAIT_LIMIT")
    y, h, _ = gpu_fwd(dev)
    torch.cuda.synchronize()
    assert mm.fault_status() == 0
    ref = oracle_fwd(inp)
    assert_close(np64(y), ref["y"], "bf16", "y", stored_bf16=True)
    assert_close(np64(h), ref["h_last"], "bf16", "h_last")
