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
