"""Stream ordering of the time-chunked forward.

A chunked call is two launches: the summary pass, launched normally, and the
full pass, launched as a programmatic dependent of it.  The full pass reads
the inputs (and h0 / conv_state_in) without waiting on the summary grid, and
only its CTAs of chunks 1.. wait before reading the summaries.  These tests
chain calls with no host synchronisation between them, the way a model
would, and check the results against the fp64 oracle and against the same
chain run with a full synchronisation after every call:
  * each call's h0 / conv_state_in are the previous call's outputs;
  * each call's activations are written by a device kernel launched just
    before it on the same stream.
"""

import os

import numpy as np
import pytest
import torch

from gpu_util import assert_close, gpu_fwd, np64, oracle_fwd, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu

SEG = 1024      # tokens per call
NSEG = 3


@pytest.fixture(autouse=True)
def _four_chunks():
    old = os.environ.get("MAMBA_MIXER_CHUNKS")
    os.environ["MAMBA_MIXER_CHUNKS"] = "4"     # a summary and a full launch per call
    yield
    if old is None:
        os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    else:
        os.environ["MAMBA_MIXER_CHUNKS"] = old


def _chain(dev, sync_each: bool):
    """Run NSEG calls over consecutive SEG-token pieces of one sequence.  The
    activations of every call are produced on the stream right before it
    (an exact elementwise kernel: x + 0); the carried state is the previous
    call's output."""
    ys = []
    h, cs = dev["h0"], dev["conv_state_in"]
    for s in range(NSEG):
        sl = slice(s * SEG, (s + 1) * SEG)
        piece = dict(dev)
        for k in ("xz", "dt", "Bm", "Cm"):
            piece[k] = torch.add(dev[k][:, sl], 0)       # a fresh tensor, written by a kernel
        piece["h0"], piece["conv_state_in"] = h, cs
        y, h, cs = gpu_fwd(piece)
        ys.append(y)
        if sync_each:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    return torch.cat(ys, dim=1), h, cs


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_chained_calls_match_oracle_and_synchronised_chain(act):
    inp = make_mixer_inputs_custom(2, NSEG * SEG, 520, act=act, seed=81, h0_std=0.3, conv_state_std=1.0,
                                   conv_b_std=0.2)
    dev = to_dev(inp)
    y, h, cs = _chain(dev, sync_each=False)
    y_s, h_s, cs_s = _chain(dev, sync_each=True)
    assert torch.equal(y, y_s)
    assert torch.equal(h, h_s)
    assert torch.equal(cs, cs_s)

    ref = oracle_fwd(inp)
    assert_close(np64(y), ref["y"], act, "y", stored_bf16=True)
    assert_close(np64(h), ref["h_last"], act, "h_last")
    np.testing.assert_array_equal(np64(cs), ref["conv_state_out"])


def test_back_to_back_repeats_are_deterministic():
    """The same chunked call repeated with no synchronisation, its carried
    state fed back each time, gives the same bits as with a synchronisation
    between the calls."""
    inp = make_mixer_inputs_custom(1, 2000, 1032, act="bf16", seed=82, h0_std=0.3, conv_state_std=1.0)
    dev = to_dev(inp)

    def run(sync_each):
        h, cs = dev["h0"], dev["conv_state_in"]
        for _ in range(12):
            piece = dict(dev)
            piece["h0"], piece["conv_state_in"] = h, cs
            y, h, cs = gpu_fwd(piece)
            if sync_each:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return y, h, cs

    a = run(False)
    b = run(True)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_calls_on_a_side_stream_with_binding_allocations():
    """mixer_fwd and state_update on a side stream, with the outputs and the
    scratch workspace allocated by the binding (on the current stream and
    recorded on the side stream): the same bits as on the current stream."""
    import mamba_selective_scan_core_b200 as mm
    from gpu_util import decode_args
    from workloads import make_decode_inputs_custom

    dev = to_dev(make_mixer_inputs_custom(1, 2048, 1032, act="bf16", seed=96, h0_std=0.3, conv_state_std=1.0))
    assert mm.workspace_size(1, 2048, 1032) > 256        # a chunked plan: the binding allocates scratch
    ref = gpu_fwd(dev)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    out = gpu_fwd(dev, stream=side)
    side.synchronize()
    for a, b in zip(out, ref):
        assert torch.equal(a, b)

    dinp = to_dev(make_decode_inputs_custom(2, 8, 256, act="bf16", seed=97))
    st, cs = dinp["ssm_state"].clone(), dinp["conv_state"].clone()
    y_ref = mm.state_update(*decode_args(dinp), st, cs)
    torch.cuda.synchronize()
    st2, cs2 = dinp["ssm_state"].clone(), dinp["conv_state"].clone()
    side.wait_stream(torch.cuda.current_stream())
    y = mm.state_update(*decode_args(dinp), st2, cs2, stream=side)
    side.synchronize()
    assert torch.equal(y, y_ref)
    assert torch.equal(st2, st)
    assert torch.equal(cs2, cs)
