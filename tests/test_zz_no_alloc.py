"""The forward entry point that allocates nothing (mamba_mixer_fwd_noalloc),
called through the C ABI, against the workspace-taking entry point
(mamba_mixer_fwd) on the same inputs: both run the same kernels on the same
launch plan, so their outputs must be the same bits, and the first case is
also checked against the fp64 oracle.

It exists for callers that cannot allocate device memory: host programs that
link only the C library and have no device allocator, and servers whose
device memory is fully planned before they start.  Its scratch is a fixed
array inside the library, shared by every call on a device, so the test runs
two different calls back to back: the second must not see anything the
first left in the scratch.  This file is named to be collected last.
"""

import ctypes

import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, np64, oracle_fwd, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_call(d, y, h, cs):
    Bsz, L, twoD = d["xz"].shape
    D = twoD // 2
    st = mm.lib().mamba_mixer_fwd_noalloc(
        _p(d["xz"]), _p(d["conv_w"]), _p(d["conv_b"]), _p(d["dt"]), _p(d["dt_bias"]), _p(d["A"]), _p(d["Bm"]),
        _p(d["Cm"]), _p(d["Dskip"]), _p(d.get("h0")), _p(d.get("conv_state_in")), _p(y), _p(h), _p(cs),
        Bsz, L, D, 16, 4, mm.MM_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, mm.status_string(st)


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        # one 1024-channel sequence: the launch plan splits time, so the scratch is used
        make_mixer_inputs_custom(1, 2048, 1024, act="bf16", seed=61, h0_std=0.3, conv_state_std=1.0),
        # a different shape and state: must not depend on what the first call left behind
        make_mixer_inputs_custom(2, 1500, 512, act="bf16", seed=62, h0_std=0.5, conv_state_std=1.0,
                                 A_mode="general"),
    ]
    for i, inp in enumerate(cases):
        Bsz, L, twoD = inp["xz"].shape
        assert mm.workspace_size(Bsz, L, twoD // 2) > 256       # a time-split plan: scratch beyond the status
        d = to_dev(inp)
        y_ref, h_ref, cs_ref = mm.mixer_fwd(d["xz"], d["conv_w"], d["conv_b"], d["dt"], d["dt_bias"], d["A"],
                                            d["Bm"], d["Cm"], d["Dskip"], d["h0"], d["conv_state_in"])
        y = torch.full_like(y_ref, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        cs = torch.zeros_like(cs_ref)
        _noalloc_call(d, y, h, cs)
        # the status of the call, kept in the library's own scratch
        assert mm.check_status(None) == 0
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
        assert torch.equal(h, h_ref)
        assert torch.equal(cs, cs_ref)
        if i == 0:
            ref = oracle_fwd(inp)
            assert_close(np64(y), ref["y"], "bf16", "y", stored_bf16=True)
            assert_close(np64(h), ref["h_last"], "bf16", "h_last")
