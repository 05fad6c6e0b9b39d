"""mamba_mixer_fwd_host: the forward on activations in host memory, which
cuts the sequence into pieces and overlaps their copies with the compute.

Checks, through the C ABI on the GPU:
  * with one time chunk per launch (MAMBA_MIXER_CHUNKS=1) it is bit-identical
    to one device-memory call -- the pieces only move where the state is
    carried, and a carried fp32 state / raw conv window is exact;
  * at the default launch plan it matches the fp64 oracle on ragged batched
    shapes with a carried state, in both dtypes;
  * pageable (not page-locked) host buffers give the same result;
  * an empty sequence passes the carried state through.
"""

import os

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, gpu_fwd, np64, oracle_fwd, to_dev
from workloads import make_mixer_inputs_custom

pytestmark = pytest.mark.gpu

HOST_KEYS = ("xz", "dt", "Bm", "Cm", "h0", "conv_state_in")
PARAM_KEYS = ("conv_w", "conv_b", "dt_bias", "A", "Dskip")


def host_fwd(inp, pin=True, stream=None):
    h = {k: (None if inp.get(k) is None else (inp[k].pin_memory() if pin else inp[k].clone())) for k in HOST_KEYS}
    d = {k: (None if inp.get(k) is None else inp[k].cuda()) for k in PARAM_KEYS}
    kw = {}
    if not pin:
        Bsz, L, twoD = inp["xz"].shape
        D = twoD // 2
        kw = dict(y=torch.empty((Bsz, L, D), dtype=inp["xz"].dtype),
                  h_last=torch.empty((Bsz, D, 16)),
                  conv_state_out=torch.empty((Bsz, D, 3), dtype=inp["xz"].dtype))
    out = mm.mixer_fwd_host(h["xz"], d["conv_w"], d["conv_b"], h["dt"], d["dt_bias"], d["A"], h["Bm"], h["Cm"],
                            d["Dskip"], h["h0"], h["conv_state_in"], stream=stream, **kw)
    (stream or torch.cuda.current_stream()).synchronize()
    return out


@pytest.fixture
def one_chunk():
    old = os.environ.get("MAMBA_MIXER_CHUNKS")
    os.environ["MAMBA_MIXER_CHUNKS"] = "1"
    yield
    if old is None:
        os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    else:
        os.environ["MAMBA_MIXER_CHUNKS"] = old


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_host_path_bitwise_equals_device_path(act, one_chunk):
    # 1300 tokens: pieces of 256, the last one ragged (20 tokens)
    inp = make_mixer_inputs_custom(2, 1300, 136, act=act, seed=71, h0_std=0.3, conv_state_std=1.0)
    y, h, cs = host_fwd(inp)
    yd, hd, csd = gpu_fwd(to_dev(inp))
    torch.cuda.synchronize()
    assert torch.equal(y, yd.cpu())
    assert torch.equal(h, hd.cpu())
    assert torch.equal(cs, csd.cpu())


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("B,L,D,A_mode", [(3, 700, 520, "structured"), (1, 2049, 64, "general")])
def test_host_path_matches_oracle(act, B, L, D, A_mode):
    inp = make_mixer_inputs_custom(B, L, D, act=act, seed=72, h0_std=0.2, conv_state_std=1.0, A_mode=A_mode)
    y, h, cs = host_fwd(inp)
    ref = oracle_fwd(inp)
    assert_close(np64(y), ref["y"], act, "y", stored_bf16=True)
    assert_close(np64(h), ref["h_last"], act, "h_last")
    np.testing.assert_array_equal(np64(cs), ref["conv_state_out"])


def test_host_path_pageable_buffers():
    inp = make_mixer_inputs_custom(2, 900, 128, act="bf16", seed=73, h0_std=0.2, conv_state_std=1.0)
    y, h, cs = host_fwd(inp, pin=True)
    y2, h2, cs2 = host_fwd(inp, pin=False)
    assert torch.equal(y, y2)
    assert torch.equal(h, h2)
    assert torch.equal(cs, cs2)


def test_host_path_on_a_side_stream():
    inp = make_mixer_inputs_custom(1, 600, 256, act="bf16", seed=74)
    y, h, cs = host_fwd(inp)
    s = torch.cuda.Stream()
    y2, h2, cs2 = host_fwd(inp, stream=s)
    assert torch.equal(y, y2)
    assert torch.equal(h, h2)


def test_host_path_empty_sequence_passes_state():
    inp = make_mixer_inputs_custom(2, 0, 64, act="bf16", seed=75, h0_std=0.5, conv_state_std=1.0)
    y, h, cs = host_fwd(inp)
    assert y.shape == (2, 0, 64)
    assert torch.equal(h, inp["h0"])
    assert torch.equal(cs, inp["conv_state_in"])


def test_host_path_jamba_prefill_workload_sampled():
    """The end-to-end leg's call at full size: the Jamba-shaped prefill
    (1 x 4096 x 8192, bf16) from pinned host memory, in its default piece
    plan, against the oracle on a deterministic channel sample."""
    from gpu_util import subset
    from workloads import CONFIGS, make_mixer_inputs, sample_channels

    cfg = CONFIGS["jamba_prefill"]
    inp = make_mixer_inputs(cfg)
    y, h, cs = host_fwd(inp)
    chans = sample_channels(cfg.d_inner, 256)
    ref = oracle_fwd(subset(inp, chans))
    S = torch.as_tensor(chans)
    assert_close(np64(y.index_select(-1, S)), ref["y"], "bf16", "y", stored_bf16=True)
    assert_close(np64(h.index_select(1, S)), ref["h_last"], "bf16", "h_last")
    np.testing.assert_array_equal(np64(cs.index_select(1, S)), ref["conv_state_out"])
