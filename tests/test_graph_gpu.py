"""The C-ABI calls captured in a CUDA graph and replayed.

A time-chunked forward is two launches, the second a programmatic dependent
of the first; under stream capture that becomes a programmatic edge of the
graph.  Replays must give the same bits as eager calls on the same inputs,
for the forward (chunked and not) and for the in-place decode step (state
and conv window advanced by each replay).
"""

import os

import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import decode_args, gpu_fwd, to_dev
from workloads import make_decode_inputs_custom, make_mixer_inputs_custom

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_plan():
    old = os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    yield
    os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    if old is not None:
        os.environ["MAMBA_MIXER_CHUNKS"] = old


@pytest.mark.parametrize("B,L,D", [(1, 2048, 1032), (3, 700, 520), (8, 256, 4096)])
def test_forward_graph_replay_matches_eager(B, L, D):
    dev = to_dev(make_mixer_inputs_custom(B, L, D, act="bf16", seed=91, h0_std=0.3, conv_state_std=1.0))
    y_e, h_e, cs_e = gpu_fwd(dev)
    torch.cuda.synchronize()

    ws = torch.empty(max(mm.workspace_size(B, L, D), 16), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(y_e)
    h = torch.empty_like(h_e)
    cs = torch.empty_like(cs_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                       # warm up outside capture on the capture stream
        gpu_fwd(dev, y=y, h_last=h, conv_state_out=cs, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gpu_fwd(dev, y=y, h_last=h, conv_state_out=cs, workspace=ws)
    for _ in range(2):
        y.zero_(); h.zero_(); cs.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_e)
        assert torch.equal(h, h_e)
        assert torch.equal(cs, cs_e)


def test_decode_graph_replay_advances_state_like_eager():
    inp = make_decode_inputs_custom(3, 16, 256, act="bf16", seed=92)
    dev = to_dev(inp)
    st_e, cs_e = dev["ssm_state"].clone(), dev["conv_state"].clone()
    for _ in range(3):
        y_e = mm.state_update(*decode_args(dev), st_e, cs_e)
    torch.cuda.synchronize()

    st, cs = dev["ssm_state"].clone(), dev["conv_state"].clone()
    y = torch.empty_like(y_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mm.state_update(*decode_args(dev), st, cs, y=y)
    # capture does not run the kernel: the state is still the initial one
    assert torch.equal(st, dev["ssm_state"])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(st, st_e)
    assert torch.equal(cs, cs_e)
    assert torch.equal(y, y_e)


def _replay_matches(call, outs_eager, outs):
    """Capture call() (writing `outs`) in a graph and check that each replay
    gives the same bits as the eager outputs."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                       # warm up outside capture on the capture stream
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(2):
        for o in outs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, outs_eager):
            assert torch.equal(o, e)


def test_ssd_graph_replay_matches_eager():
    """The Mamba-2 call (three launches; the call's epoch written by a kernel,
    not by a host copy) captured and replayed."""
    from workloads import make_ssd_inputs_custom

    d = to_dev(make_ssd_inputs_custom(2, 600, 4, groups=2, seed=93, h0_std=0.3))
    args = (d["x"], d["z"], d["dt"], d["dt_bias"], d["A"], d["Bm"], d["Cm"], d["Dskip"], d["h0"])
    y_e, h_e = mm.ssd_fwd(*args)
    torch.cuda.synchronize()
    ws = torch.empty(mm.ssd_workspace_size(2, 600, 4, groups=2), dtype=torch.uint8, device="cuda")
    y, h = torch.empty_like(y_e), torch.empty_like(h_e)
    _replay_matches(lambda: mm.ssd_fwd(*args, y=y, h_last=h, workspace=ws), (y_e, h_e), (y, h))
    assert mm.check_status(ws) == 0


def test_m3_graph_replay_matches_eager():
    """The Mamba-3 call (summary and full pass) captured and replayed."""
    from workloads import make_m3_inputs_custom

    d = to_dev(make_m3_inputs_custom(2, 700, 4, rank=2, groups=2, seed=94, h0_std=0.3, prev=True))
    keys = ("x", "z", "dt", "trap", "dt_bias", "A", "theta", "Bm", "Cm", "Dskip", "h0", "x_prev", "B_prev")
    args = tuple(d[k] for k in keys)
    y_e, h_e = mm.m3_fwd(*args)
    torch.cuda.synchronize()
    ws = torch.empty(mm.m3_workspace_size(2, 700, 4, 2, groups=2), dtype=torch.uint8, device="cuda")
    y, h = torch.empty_like(y_e), torch.empty_like(h_e)
    _replay_matches(lambda: mm.m3_fwd(*args, y=y, h_last=h, workspace=ws), (y_e, h_e), (y, h))
    assert mm.check_status(ws) == 0


def test_proj_matmul_graph_replay_matches_eager():
    """A projection product split in K (GEMM, then the sum of the partials)
    captured and replayed."""
    g = torch.Generator(device="cuda").manual_seed(95)
    A = torch.randn((256, 4096), device="cuda", generator=g).to(torch.bfloat16)
    W = (torch.randn((288, 4096), device="cuda", generator=g) / 64).to(torch.bfloat16)
    assert mm.proj_matmul_workspace_size(256, 288, 4096) > 256, "expected a split-K plan"
    o_e = mm.proj_matmul(A, W)
    torch.cuda.synchronize()
    ws = torch.empty(mm.proj_matmul_workspace_size(256, 288, 4096), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(o_e)
    _replay_matches(lambda: mm.proj_matmul(A, W, out=o, workspace=ws), (o_e,), (o,))
    assert mm.check_status(ws) == 0
