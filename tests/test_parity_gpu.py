"""CUDA path vs the fp64 oracle, element by element, on seeded inputs.

Small cases cover several tiles, ragged tails, every lanes-per-channel
layout, both activation dtypes, structured and general A, and the optional
inputs.  The five workloads run at full size in the launch configuration the
benchmark uses: the Jamba-shaped prefill and the 28-layer decode are compared
in full (every channel, every row); the 4 x 32768 and 256K-token workloads on
deterministic samples of 1024 and 256 channels, which the oracle computes
exactly (channels are independent given the shared B/C).
"""

import os

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
from gpu_util import assert_close, gpu_fwd, np64, oracle_fwd, subset, to_dev, decode_args, THREADS
import oracle
from ws_layout import ws_bytes
from workloads import CONFIGS, make_decode_inputs, make_decode_inputs_custom, make_mixer_inputs, \
    make_mixer_inputs_custom, sample_channels

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _tuning_env():
    names = ("MAMBA_MIXER_CHUNKS",)
    old = {n: os.environ.pop(n, None) for n in names}
    yield
    for n in names:
        os.environ.pop(n, None)
        if old[n] is not None:
            os.environ[n] = old[n]


def check_fwd(inp, act, chans=None, **kw):
    dev = to_dev(inp)
    y, hl, cs = gpu_fwd(dev, **kw)
    torch.cuda.synchronize()
    if chans is None:
        ref = oracle_fwd(inp)
        got_y, got_h, got_cs = np64(y), np64(hl), np64(cs)
    else:
        ref = oracle_fwd(subset(inp, chans))
        S = torch.as_tensor(chans)
        got_y = np64(y.index_select(-1, S.to(y.device)))
        got_h = np64(hl.index_select(1, S.to(hl.device)))
        got_cs = np64(cs.index_select(1, S.to(cs.device)))
    assert_close(got_y, ref["y"], act, "y", stored_bf16=True)
    assert_close(got_h, ref["h_last"], act, "h_last")
    # the carried window is raw input values: exact
    np.testing.assert_array_equal(got_cs, ref["conv_state_out"])
    return y, hl, cs


# ------------------------------------------------------------------ small shapes
SMALL = []
for act in ("bf16", "f32"):
    for (B, L, D) in [(1, 1, 8), (2, 2, 16), (1, 3, 24), (3, 5, 8), (1, 33, 64), (2, 100, 40), (1, 257, 136),
                      (2, 64, 520)]:
        SMALL.append((act, B, L, D))


@pytest.mark.parametrize("act,B,L,D", SMALL)
@pytest.mark.parametrize("A_mode", ["structured", "general"])
def test_small_shapes(act, B, L, D, A_mode):
    inp = make_mixer_inputs_custom(B, L, D, act=act, seed=1000 + L * 7 + D + B, h0_std=0.5, conv_state_std=1.0,
                                   conv_b_std=0.2, A_mode=A_mode, dt_std=0.5)
    check_fwd(inp, act)


CHUNKED = [(act, k, A_mode) for act in ("bf16", "f32") for k in (1, 2, 5, 11) for A_mode in ("structured", "general")]


@pytest.mark.parametrize("act,chunks,A_mode", CHUNKED)
def test_time_chunked(act, chunks, A_mode):
    """The two-pass time-chunked forward (summary pass + seeded full pass),
    ragged last chunk included."""
    os.environ["MAMBA_MIXER_CHUNKS"] = str(chunks)
    inp = make_mixer_inputs_custom(2, 333, 40, act=act, seed=900 + chunks * 10, h0_std=0.5,
                                   conv_state_std=1.0, conv_b_std=0.2, A_mode=A_mode, dt_std=0.5)
    check_fwd(inp, act)


@pytest.mark.parametrize("A_mode", ["structured", "general"])
def test_wide_ctas_partial_last_block(A_mode):
    """d_inner 504 (63 channel octets) in 256-channel CTAs, the second of each
    pair 248 channels wide; 8 sequences x 12 time chunks need more than one
    CTA per SM, so the two-stage ring compiled for the 256-channel width runs
    (summary and full pass), with inactive threads in every second CTA."""
    os.environ["MAMBA_MIXER_CHUNKS"] = "12"
    inp = make_mixer_inputs_custom(8, 1100, 504, act="bf16", seed=4242, h0_std=0.5, conv_state_std=1.0,
                                   conv_b_std=0.2, A_mode=A_mode, dt_std=0.5)
    check_fwd(inp, "bf16")


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_optional_inputs_absent(act):
    inp = make_mixer_inputs_custom(2, 70, 32, act=act, seed=77)
    inp["conv_b"] = None
    inp["Dskip"] = None
    assert inp["h0"] is None and inp["conv_state_in"] is None
    check_fwd(inp, act)


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_large_step_sizes(act):
    # dt up to ~N(0, 3): softplus far into its tails, strong decay
    inp = make_mixer_inputs_custom(1, 96, 16, act=act, seed=5, dt_std=3.0, h0_std=1.0, A_mode="general")
    check_fwd(inp, act)


def test_seqlen_zero_passes_state_through():
    inp = make_mixer_inputs_custom(2, 0, 16, act="bf16", seed=3, h0_std=1.0, conv_state_std=1.0)
    dev = to_dev(inp)
    y, hl, cs = gpu_fwd(dev)
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 16)
    assert torch.equal(hl, dev["h0"])
    assert torch.equal(cs, dev["conv_state_in"])


def test_batch_zero_is_noop():
    inp = make_mixer_inputs_custom(0, 5, 16, act="bf16", seed=3)
    y, hl, cs = gpu_fwd(to_dev(inp))
    assert y.numel() == 0 and hl.numel() == 0


# ------------------------------------------------------------------ workloads
def test_tiny_f32_workload():
    cfg = CONFIGS["tiny_f32"]
    check_fwd(make_mixer_inputs(cfg), "f32")


def test_jamba_prefill_workload_full():
    """Every channel and token of the Jamba-shaped prefill against the oracle."""
    cfg = CONFIGS["jamba_prefill"]
    inp = make_mixer_inputs(cfg)
    check_fwd(inp, "bf16")


def test_jamba_prefill_general_A_full():
    """The Jamba-shaped prefill with per-state A rows (as trained weights
    have): the general path at full size, in the launch plan the bench's
    general_a leg times, every channel against the oracle."""
    cfg = CONFIGS["jamba_prefill"]
    inp = make_mixer_inputs(cfg, A_mode="general")
    check_fwd(inp, "bf16")


def test_batched_prefill_workload_sampled():
    cfg = CONFIGS["batched_prefill"]
    inp = make_mixer_inputs(cfg)
    check_fwd(inp, "bf16", chans=sample_channels(cfg.d_inner, 1024))


@pytest.mark.parametrize("B,chunks", [(2, 4), (3, 3)])
def test_multi_sequence_chunk_plans_sampled(B, chunks):
    """Two and three Jamba-shaped sequences at full size, with the launch
    plans the planner picks for them (4 and 3 time chunks: the carried state
    crosses chunk boundaries inside every sequence of the batch)."""
    assert mm.workspace_size(B, 4096, 8192) == ws_bytes(B, chunks, 8192)
    inp = make_mixer_inputs_custom(B, 4096, 8192, act="bf16", seed=80 + B, h0_std=0.1, conv_state_std=1.0)
    check_fwd(inp, "bf16", chans=sample_channels(8192, 64))


@pytest.mark.parametrize("act", ["bf16", "f32"])
def test_narrow_sequence_sixteen_chunks(act):
    """64 channels x 4096 tokens: the default plan takes the maximum 16 time
    chunks (a 15-step carry chain), checked against the oracle in full."""
    assert mm.workspace_size(1, 4096, 64) == ws_bytes(1, 16, 64)
    inp = make_mixer_inputs_custom(1, 4096, 64, act=act, seed=91, h0_std=0.3, conv_state_std=1.0)
    check_fwd(inp, act)


def _run_carried(dev, n, D):
    L = dev["xz"].shape[1]
    step = L // n
    y = torch.empty((1, L, D), dtype=torch.bfloat16, device="cuda")
    bufs = [(torch.empty((1, D, 16), device="cuda"), torch.empty((1, D, 3), dtype=torch.bfloat16, device="cuda"))
            for _ in range(2)]
    h, cs = None, None
    for i in range(n):
        sl = slice(i * step, (i + 1) * step)
        part = dict(dev)
        part.update(xz=dev["xz"][:, sl].contiguous(), dt=dev["dt"][:, sl].contiguous(),
                    Bm=dev["Bm"][:, sl].contiguous(), Cm=dev["Cm"][:, sl].contiguous(), h0=h, conv_state_in=cs)
        hout, csout = bufs[i % 2]
        yi, h, cs = gpu_fwd(part, h_last=hout, conv_state_out=csout)
        y[:, sl] = yi
        del part
    return y, h.clone(), cs.clone()


def test_long_256k_carried_chunks_sampled():
    """256K tokens as 8 carried 32768-token calls (the launch plan the
    benchmark uses) against the unsplit oracle; and, with one time chunk per
    call, bit-identical to a single unsplit call."""
    cfg = CONFIGS["long_256k"]
    inp = make_mixer_inputs(cfg)
    dev = to_dev(inp)
    L, D, n = cfg.seqlen, cfg.d_inner, cfg.chunks
    y, h, cs = _run_carried(dev, n, D)
    torch.cuda.synchronize()
    chans = sample_channels(D, 256)
    ref = oracle_fwd(subset(inp, chans))
    S = torch.as_tensor(chans, device="cuda")
    assert_close(np64(y.index_select(-1, S)), ref["y"], "bf16", "y", stored_bf16=True)
    assert_close(np64(h.index_select(1, S)), ref["h_last"], "bf16", "h_last")
    np.testing.assert_array_equal(np64(cs.index_select(1, S)), ref["conv_state_out"])
    del y
    os.environ["MAMBA_MIXER_CHUNKS"] = "1"
    y8, h8, cs8 = _run_carried(dev, n, D)
    y1, h1, cs1 = gpu_fwd(dev)
    torch.cuda.synchronize()
    assert torch.equal(y8, y1)
    assert torch.equal(h8, h1)
    assert torch.equal(cs8, cs1)


# ------------------------------------------------------------------ decode
def check_decode(inp, act, rows=None):
    dev = to_dev(inp)
    ssm = dev["ssm_state"].clone()
    cs = dev["conv_state"].clone()
    y = mm.state_update(*decode_args(dev), ssm, cs)
    torch.cuda.synchronize()
    NL, B, D = inp["x"].shape
    if rows is None:
        ref = oracle.state_update(*decode_args(inp), inp["ssm_state"], inp["conv_state"], threads=THREADS)
        assert_close(np64(y), ref["y"], act, "y", stored_bf16=True)
        assert_close(np64(ssm), ref["ssm_state"], act, "ssm_state")
        np.testing.assert_array_equal(np64(cs), ref["conv_state"])
    else:
        # rows: (layer, batch) pairs, all channels of each
        for (l, b) in rows:
            one = {k: (v[l:l + 1, b:b + 1] if k in ("x", "z", "dt", "Bm", "Cm", "ssm_state", "conv_state")
                       else v[l:l + 1]) for k, v in inp.items() if v is not None}
            one["conv_b"] = inp["conv_b"][l:l + 1] if inp["conv_b"] is not None else None
            ref = oracle.state_update(*decode_args(one), one["ssm_state"], one["conv_state"], threads=THREADS)
            assert_close(np64(y[l:l + 1, b:b + 1]), ref["y"], act, f"y[{l},{b}]", stored_bf16=True)
            assert_close(np64(ssm[l:l + 1, b:b + 1]), ref["ssm_state"], act, f"ssm[{l},{b}]")
            np.testing.assert_array_equal(np64(cs[l:l + 1, b:b + 1]), ref["conv_state"])
    return y, ssm, cs


@pytest.mark.parametrize("act", ["bf16", "f32"])
@pytest.mark.parametrize("NL,B,D", [(1, 1, 8), (2, 3, 40), (3, 5, 256)])
@pytest.mark.parametrize("A_mode", ["structured", "general"])
def test_decode_small(act, NL, B, D, A_mode):
    inp = make_decode_inputs_custom(NL, B, D, act=act, seed=NL * 100 + B * 10 + D, A_mode=A_mode, conv_b_std=0.2)
    check_decode(inp, act)


def test_decode_workload_full():
    """All 28 x 128 (layer, batch) rows, every channel, against the oracle."""
    cfg = CONFIGS["decode_28x128"]
    inp = make_decode_inputs(cfg)
    check_decode(inp, "bf16")
