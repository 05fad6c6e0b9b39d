"""The fused RMSNorm of B_t and C_t (mamba_mixer_fwd_normed and
mamba_state_update_normed) against the fp64 oracle, which normalises B and C
over their d_state entries (oracle_rmsnorm_rows) and then runs the plain
recurrence.  The pages place RMSNorm inside the Mamba layer, on its internal
activations; B_t and C_t are the reading this library takes."""

import os

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
import oracle
from gpu_util import THREADS, assert_close, decode_args, gpu_fwd, np64, to_dev
from workloads import CONFIGS, make_decode_inputs, make_decode_inputs_custom, make_mixer_inputs, \
    make_mixer_inputs_custom, make_norm_weights

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(autouse=True)
def _tuning_env():
    old = os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    yield
    os.environ.pop("MAMBA_MIXER_CHUNKS", None)
    if old is not None:
        os.environ["MAMBA_MIXER_CHUNKS"] = old


def check_normed_fwd(inp, act, wb, wc):
    dev = to_dev(inp)
    y, h, cs = gpu_fwd(dev, b_norm_w=wb.cuda() if wb is not None else None,
                       c_norm_w=wc.cuda() if wc is not None else None, norm_eps=EPS)
    torch.cuda.synchronize()
    ref = oracle.mixer_fwd_normed(inp["xz"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["dt_bias"], inp["A"],
                                  inp["Bm"], inp["Cm"], inp["Dskip"], inp.get("h0"), inp.get("conv_state_in"),
                                  b_norm_w=wb, c_norm_w=wc, norm_eps=EPS, threads=THREADS)
    assert_close(np64(y), ref["y"], act, "y", stored_bf16=True)
    assert_close(np64(h), ref["h_last"], act, "h_last")
    np.testing.assert_array_equal(np64(cs), ref["conv_state_out"])


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("B,L,D", [(1, 1, 8), (2, 37, 40), (1, 257, 136), (2, 64, 520)])
@pytest.mark.parametrize("A_mode", ["structured", "general"])
def test_normed_small_shapes(act, B, L, D, A_mode):
    inp = make_mixer_inputs_custom(B, L, D, act=act, seed=2000 + L + D + B, h0_std=0.5, conv_state_std=1.0,
                                   conv_b_std=0.2, A_mode=A_mode, dt_std=0.5)
    wb, wc = make_norm_weights(seed=L + D)
    check_normed_fwd(inp, act, wb, wc)


@pytest.mark.parametrize("which", ["B", "C"])
def test_normed_one_input_only(which):
    inp = make_mixer_inputs_custom(2, 100, 64, act="bf16", seed=2101, h0_std=0.5)
    wb, wc = make_norm_weights(seed=7)
    check_normed_fwd(inp, "bf16", wb if which == "B" else None, wc if which == "C" else None)


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("chunks", [2, 5])
def test_normed_time_chunked(act, chunks):
    """The summary pass normalises B the same way as the full pass."""
    os.environ["MAMBA_MIXER_CHUNKS"] = str(chunks)
    inp = make_mixer_inputs_custom(2, 333, 40, act=act, seed=2200 + chunks, h0_std=0.5, conv_state_std=1.0)
    wb, wc = make_norm_weights(seed=chunks)
    check_normed_fwd(inp, act, wb, wc)


def test_normed_jamba_prefill_full():
    """The Jamba-shaped prefill with both norms, every channel and token."""
    inp = make_mixer_inputs(CONFIGS["jamba_prefill"])
    wb, wc = make_norm_weights(seed=11)
    check_normed_fwd(inp, "bf16", wb, wc)


def check_normed_decode(inp, act, wb, wc):
    dev = to_dev(inp)
    ssm, cs = dev["ssm_state"].clone(), dev["conv_state"].clone()
    y = mm.state_update(*decode_args(dev), ssm, cs, b_norm_w=wb.cuda(), c_norm_w=wc.cuda(), norm_eps=EPS)
    torch.cuda.synchronize()
    ref = oracle.state_update_normed(*decode_args(inp), inp["ssm_state"], inp["conv_state"], b_norm_w=wb,
                                     c_norm_w=wc, norm_eps=EPS, threads=THREADS)
    assert_close(np64(y), ref["y"], act, "y", stored_bf16=True)
    assert_close(np64(ssm), ref["ssm_state"], act, "ssm_state")
    np.testing.assert_array_equal(np64(cs), ref["conv_state"])


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("NL,B,D", [(1, 1, 8), (3, 5, 256)])
def test_normed_decode_small(act, NL, B, D):
    inp = make_decode_inputs_custom(NL, B, D, act=act, seed=NL * 31 + B + D, conv_b_std=0.2)
    wb, wc = make_norm_weights(layers=NL, seed=NL + B)
    check_normed_decode(inp, act, wb, wc)


def test_normed_decode_workload_full():
    inp = make_decode_inputs(CONFIGS["decode_28x128"])
    wb, wc = make_norm_weights(layers=28, seed=12)
    check_normed_decode(inp, "bf16", wb, wc)


def test_normed_decode_continues_normed_prefill():
    """A normed prefill of L tokens followed by one normed decode step equals
    the normed prefill of L+1 tokens at the last token."""
    full = make_mixer_inputs_custom(1, 65, 64, act="f32", seed=2300, h0_std=0.3, conv_state_std=1.0)
    wb, wc = make_norm_weights(seed=13)
    pre = {k: (v[:, :64].contiguous() if k in ("xz", "dt", "Bm", "Cm") else v) for k, v in full.items()}
    dev = to_dev(pre)
    _, h, cs = gpu_fwd(dev, b_norm_w=wb.cuda(), c_norm_w=wc.cuda(), norm_eps=EPS)
    D = 64
    t = 64
    dec = {"x": full["xz"][:, t:t + 1, :D].reshape(1, 1, D), "z": full["xz"][:, t:t + 1, D:].reshape(1, 1, D),
           "dt": full["dt"][:, t:t + 1].reshape(1, 1, D), "conv_w": full["conv_w"][None], "conv_b": full["conv_b"][None],
           "dt_bias": full["dt_bias"][None], "Dskip": full["Dskip"][None], "A": full["A"][None],
           "Bm": full["Bm"][:, t:t + 1].reshape(1, 1, 16), "Cm": full["Cm"][:, t:t + 1].reshape(1, 1, 16)}
    ddev = to_dev(dec)
    ssm = h.reshape(1, 1, D, 16).clone()
    csd = cs.reshape(1, 1, D, 3).clone()
    y1 = mm.state_update(*decode_args(ddev), ssm, csd, b_norm_w=wb[None].cuda(), c_norm_w=wc[None].cuda(),
                         norm_eps=EPS)
    torch.cuda.synchronize()
    ref = oracle.mixer_fwd_normed(full["xz"], full["conv_w"], full["conv_b"], full["dt"], full["dt_bias"],
                                  full["A"], full["Bm"], full["Cm"], full["Dskip"], full["h0"],
                                  full["conv_state_in"], b_norm_w=wb, c_norm_w=wc, norm_eps=EPS)
    assert_close(np64(y1).reshape(1, 1, D), ref["y"][:, t:t + 1], "f32", "y")
    assert_close(np64(ssm).reshape(1, D, 16), ref["h_last"], "f32", "h_last")
