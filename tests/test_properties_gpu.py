"""Properties of the CUDA path that hold at any size: carrying (h_last,
conv_state_out) across calls equals one call (the state is all the history
the next token needs), and the decode step continues a prefill exactly as a
longer prefill would."""

import os

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, gpu_fwd, np64, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu


def _slice(dev, a, b, h0, cs):
    part = dict(dev)
    part.update(xz=dev["xz"][:, a:b].contiguous(), dt=dev["dt"][:, a:b].contiguous(),
                Bm=dev["Bm"][:, a:b].contiguous(), Cm=dev["Cm"][:, a:b].contiguous(), h0=h0, conv_state_in=cs)
    return part


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("D", [48, 8, 520])
def test_split_equals_unsplit_bitwise(act, D):
    # one time chunk per call, so both runs apply the same per-token arithmetic
    os.environ["MAMBA_MIXER_CHUNKS"] = "1"
    try:
        inp = make_mixer_inputs_custom(2, 300, D, act=act, seed=31, h0_std=0.3, conv_state_std=1.0)
        dev = to_dev(inp)
        y_full, h_full, cs_full = gpu_fwd(dev)
        cuts = [0, 1, 2, 5, 32, 33, 100, 300]
        h, cs = dev["h0"], dev["conv_state_in"]
        ys = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            y, h, cs = gpu_fwd(_slice(dev, a, b, h, cs))
            ys.append(y)
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(ys, dim=1), y_full)
        assert torch.equal(h, h_full)
        assert torch.equal(cs, cs_full)
    finally:
        os.environ.pop("MAMBA_MIXER_CHUNKS", None)


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("chunks", ["2", "3", "7"])
def test_time_chunks_match_one_chunk(act, chunks):
    """The two-pass time-chunked forward equals the single-chunk forward up to
    rounding (it is an exact re-association of the recurrence)."""
    inp = make_mixer_inputs_custom(2, 500, 24, act=act, seed=57, h0_std=0.4, conv_state_std=1.0, conv_b_std=0.1)
    dev = to_dev(inp)
    try:
        os.environ["MAMBA_MIXER_CHUNKS"] = "1"
        y1, h1, c1 = gpu_fwd(dev)
        os.environ["MAMBA_MIXER_CHUNKS"] = chunks
        yk, hk, ck = gpu_fwd(dev)
        torch.cuda.synchronize()
    finally:
        os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    assert_close(np64(yk), np64(y1), act, "y", stored_bf16=True)
    assert_close(np64(hk), np64(h1), act, "h_last")
    assert torch.equal(ck, c1)


def _decode_from_prefill(dev, t, h, cs):
    """Run the decode step for token t of every sequence (one layer)."""
    D = dev["dt"].shape[-1]
    x = dev["xz"][:, t, :D].unsqueeze(0).contiguous()
    z = dev["xz"][:, t, D:].unsqueeze(0).contiguous()
    dt = dev["dt"][:, t].unsqueeze(0).contiguous()
    Bm = dev["Bm"][:, t].unsqueeze(0).contiguous()
    Cm = dev["Cm"][:, t].unsqueeze(0).contiguous()
    ssm = h.unsqueeze(0).clone()
    csv = cs.unsqueeze(0).clone()
    y = mm.state_update(x, z, dt, dev["conv_w"][None], dev["conv_b"][None], dev["dt_bias"][None],
                        dev["Dskip"][None], dev["A"][None], Bm, Cm, ssm, csv)
    return y[0], ssm[0], csv[0]


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_decode_continues_prefill(act):
    """prefill(L-1) then one decode step == prefill(L) at its last token; and
    k decode steps from a prefix == the prefill of those k tokens."""
    B, L, D = 3, 40, 64
    inp = make_mixer_inputs_custom(B, L, D, act=act, seed=41, h0_std=0.3, conv_state_std=1.0, conv_b_std=0.1)
    dev = to_dev(inp)
    y_full, h_full, cs_full = gpu_fwd(dev)
    _, h, cs = gpu_fwd(_slice(dev, 0, L - 1, dev["h0"], dev["conv_state_in"]))
    y_last, h_last, cs_last = _decode_from_prefill(dev, L - 1, h, cs)
    torch.cuda.synchronize()
    assert_close(np64(y_last), np64(y_full[:, L - 1]), act, "y", stored_bf16=True)
    assert_close(np64(h_last), np64(h_full), act, "h")
    assert torch.equal(cs_last, cs_full)

    k0 = 25
    _, h, cs = gpu_fwd(_slice(dev, 0, k0, dev["h0"], dev["conv_state_in"]))
    ys = []
    for t in range(k0, L):
        yt, h, cs = _decode_from_prefill(dev, t, h, cs)
        ys.append(yt)
    torch.cuda.synchronize()
    assert_close(np64(torch.stack(ys, dim=1)), np64(y_full[:, k0:]), act, "y steps", stored_bf16=True)
    assert_close(np64(h), np64(h_full), act, "h steps")
    assert torch.equal(cs, cs_full)
