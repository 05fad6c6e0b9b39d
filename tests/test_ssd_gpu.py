"""The Mamba-2 form of the scan (mamba_ssd_fwd: scalar decay per head, grouped
B/C, chunked products on the tensor cores) against the fp64 oracle
(oracle_ssd_fwd, the plain per-channel recurrence).

Tolerance: the problem statement's bound for bf16 inputs with fp32 state,
max |err| <= 2e-2 rms(ref) per output tensor, y's own rounding to bf16
excluded as for the other forwards.  The operands the kernels compute (the
weighted x, the decayed C.B matrix, the carried state) enter the products as
bf16 hi + lo parts, about 16 bits; a single bf16 rounding of them (a relative
2^-9 per term) broke this bound, and the margins table shows how far inside
it the split keeps the results."""

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
import oracle
from gpu_util import THREADS, assert_close, np64, to_dev
from workloads import SSD_CONFIGS, make_ssd_inputs, make_ssd_inputs_custom

pytestmark = pytest.mark.gpu

MM_ERR_TIMEOUT = 11


def gpu_ssd(d, **kw):
    return mm.ssd_fwd(d["x"], d.get("z"), d["dt"], d.get("dt_bias"), d["A"], d["Bm"], d["Cm"], d.get("Dskip"),
                      d.get("h0"), **kw)


def oracle_ssd(inp, threads=THREADS):
    return oracle.ssd_fwd(inp["x"], inp.get("z"), inp["dt"], inp.get("dt_bias"), inp["A"], inp["Bm"], inp["Cm"],
                          inp.get("Dskip"), inp.get("h0"), headdim=64, threads=threads)


def heads_subset(inp, heads):
    """Inputs restricted to some heads (heads are independent given their
    group's B/C; with one group every head reads the same B/C)."""
    hs = torch.as_tensor(np.asarray(heads), dtype=torch.long)
    chans = (hs[:, None] * 64 + torch.arange(64)[None, :]).reshape(-1)
    out = dict(inp)
    out["x"] = inp["x"].index_select(-1, chans)
    out["z"] = inp["z"].index_select(-1, chans) if inp.get("z") is not None else None
    out["dt"] = inp["dt"].index_select(-1, hs)
    for k in ("dt_bias", "A", "Dskip"):
        out[k] = inp[k].index_select(0, hs) if inp.get(k) is not None else None
    out["h0"] = inp["h0"].index_select(1, hs) if inp.get("h0") is not None else None
    return out


def check(inp, y, h, heads=None):
    ref_in = heads_subset(inp, heads) if heads is not None else inp
    ref = oracle_ssd(ref_in)
    gy, gh = np64(y), np64(h)
    if heads is not None:
        chans = (np.asarray(heads)[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
        gy, gh = gy[..., chans], gh[:, np.asarray(heads)]
    assert_close(gy, ref["y"], "bf16", "y", stored_bf16=True)
    assert_close(gh, ref["h_last"], "bf16", "h_last")


@pytest.mark.parametrize("B,L,H,G", [(1, 1, 1, 1), (1, 5, 2, 1), (1, 127, 2, 2), (2, 128, 2, 1), (1, 129, 3, 3),
                                     (2, 300, 4, 2), (1, 1000, 2, 1), (3, 515, 8, 4)])
def test_ssd_small(B, L, H, G):
    inp = make_ssd_inputs_custom(B, L, H, groups=G, seed=B * 1000 + L + H * 7 + G, h0_std=0.3)
    y, h = gpu_ssd(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, h)


@pytest.mark.parametrize("gate,h0,skip,bias", [(False, False, False, False), (True, False, True, False),
                                               (False, True, False, True)])
def test_ssd_optional_inputs(gate, h0, skip, bias):
    inp = make_ssd_inputs_custom(2, 333, 4, seed=17, h0_std=0.2 if h0 else 0.0, gate=gate)
    if not skip:
        inp["Dskip"] = None
    if not bias:
        inp["dt_bias"] = None
    y, h = gpu_ssd(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, h)


def test_ssd_large_steps():
    """Large step sizes (dt ~ N(0, 2)): chunks whose decays underflow to zero
    within a few tokens, and softplus's linear tail."""
    inp = make_ssd_inputs_custom(1, 640, 4, seed=23, h0_std=0.5, dt_std=2.0)
    y, h = gpu_ssd(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, h)


def test_ssd_empty_sequence():
    """seqlen 0: no token, h_last = h0 (or zeros without h0)."""
    inp = make_ssd_inputs_custom(2, 0, 3, seed=29, h0_std=0.4)
    d = to_dev(inp)
    _, h = gpu_ssd(d)
    torch.cuda.synchronize()
    assert torch.equal(h, d["h0"])
    _, h = gpu_ssd(dict(d, h0=None))
    torch.cuda.synchronize()
    assert torch.count_nonzero(h).item() == 0


def test_ssd_split_equals_unsplit():
    """A sequence run as two calls with h_last carried into h0: split on a
    chunk boundary it is the same arithmetic (bit-exact); a ragged split
    regroups the chunks and matches the oracle."""
    inp = make_ssd_inputs_custom(2, 700, 4, seed=31, h0_std=0.3)
    d = to_dev(inp)
    y, h = gpu_ssd(d)

    def part(lo, hi, h0):
        c = dict(d)
        for k in ("x", "z", "dt", "Bm", "Cm"):
            c[k] = d[k][:, lo:hi].contiguous()
        c["h0"] = h0
        return gpu_ssd(c)

    y1, h1 = part(0, 256, d["h0"])
    y2, h2 = part(256, 700, h1)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], dim=1), y)
    assert torch.equal(h2, h)
    y1, h1 = part(0, 301, d["h0"])
    y2, h2 = part(301, 700, h1)
    torch.cuda.synchronize()
    check(inp, torch.cat([y1, y2], dim=1), h2)


def test_ssd_repeatable_and_status():
    """Two calls on the same inputs agree bit for bit, and the call's status
    reads complete."""
    inp = make_ssd_inputs_custom(1, 500, 4, seed=37)
    d = to_dev(inp)
    ws = torch.randint(0, 255, (mm.ssd_workspace_size(1, 500, 4),), dtype=torch.uint8, device="cuda")
    y1, h1 = gpu_ssd(d, workspace=ws)
    assert mm.check_status(ws) == 0
    y2, h2 = gpu_ssd(d, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


def test_ssd_forced_wait_timeout_is_reported(monkeypatch):
    """With the wait limit forced to zero the chunk kernels give up at their
    first wait, record it in the call's status and the device fault word,
    and the next call is correct."""
    inp = make_ssd_inputs_custom(1, 300, 2, seed=41)
    d = to_dev(inp)
    ws = torch.randint(0, 255, (mm.ssd_workspace_size(1, 300, 2),), dtype=torch.uint8, device="cuda")
    assert mm.fault_status(reset=True) == 0
    monkeypatch.setenv("MAMBA_MIXER_WAIT_LIMIT", "0")
    gpu_ssd(d, workspace=ws)
    assert mm.check_status(ws) == MM_ERR_TIMEOUT
    assert mm.fault_status(reset=True) == MM_ERR_TIMEOUT
    monkeypatch.delenv("MAMBA_MIXER_WAIT_LIMIT")
    y, h = gpu_ssd(d, workspace=ws)
    assert mm.check_status(ws) == 0
    assert mm.fault_status() == 0
    check(inp, y, h)


def test_ssd_mamba2_prefill_full_size():
    """The Mamba-2 workload at full size (4096 tokens, 128 heads of 64, d_state
    128): every channel against the oracle."""
    cfg = SSD_CONFIGS["mamba2_prefill"]
    inp = make_ssd_inputs(cfg)
    y, h = gpu_ssd(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, h)


def test_ssd_mamba2_batched_sampled_heads():
    """4 x 8192 tokens with an initial state: 12 of the 128 heads (the first,
    the last and an even stride) against the oracle."""
    cfg = SSD_CONFIGS["mamba2_batched"]
    inp = make_ssd_inputs(cfg)
    y, h = gpu_ssd(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, h, heads=[0, 1, 13, 29, 41, 57, 64, 77, 90, 103, 126, 127])


def test_ssd_token_by_token_continues_prefill():
    """Decode use: a prefill of 61 tokens, then three one-token calls, each
    starting from the previous call's h_last, matches the oracle's single run
    of all 64 tokens."""
    inp = make_ssd_inputs_custom(2, 64, 4, groups=2, seed=43, h0_std=0.2)
    d = to_dev(inp)

    def part(lo, hi, h0):
        c = dict(d)
        for k in ("x", "z", "dt", "Bm", "Cm"):
            c[k] = d[k][:, lo:hi].contiguous()
        c["h0"] = h0
        return gpu_ssd(c)

    ys = []
    y, h = part(0, 61, d["h0"])
    ys.append(y)
    for t in range(61, 64):
        y, h = part(t, t + 1, h)
        ys.append(y)
    torch.cuda.synchronize()
    check(inp, torch.cat(ys, dim=1), h)


# ---------------------------------------------------------------- one-token step (decode)
def gpu_ssd_decode(d, state=None):
    """mamba_ssd_state_update on the first token of one-token inputs d, in place
    on `state` (a copy of d's h0, or zeros, when not given).  Returns y
    [B,1,H*P] and the state."""
    B, _, C = d["x"].shape
    H = d["A"].shape[0]
    if state is None:
        state = d["h0"].clone() if d.get("h0") is not None else torch.zeros((B, H, 64, 128), device="cuda")
    tok = {k: (d[k][:, 0].contiguous() if d.get(k) is not None else None) for k in ("x", "z", "dt", "Bm", "Cm")}
    y = mm.ssd_state_update(tok["x"], tok["z"], tok["dt"], d.get("dt_bias"), d["A"], tok["Bm"], tok["Cm"],
                            d.get("Dskip"), state)
    return y[:, None], state


@pytest.mark.parametrize("B,H,G,gate,skip,bias,h0", [(1, 1, 1, True, True, True, True),
                                                     (2, 4, 2, True, True, True, True),
                                                     (3, 6, 3, False, False, True, True),
                                                     (2, 8, 1, True, False, False, True),
                                                     (5, 2, 2, True, True, True, False)])
def test_ssd_decode_small(B, H, G, gate, skip, bias, h0):
    """One token against the oracle's one-token run from the same state."""
    inp = make_ssd_inputs_custom(B, 1, H, groups=G, seed=300 + B * 11 + H, h0_std=0.3 if h0 else 0.0, gate=gate)
    if not skip:
        inp["Dskip"] = None
    if not bias:
        inp["dt_bias"] = None
    y, state = gpu_ssd_decode(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, state)


def test_ssd_decode_large_steps():
    """Large and small step sizes (softplus on both tails, decays near 0 and 1)."""
    inp = make_ssd_inputs_custom(2, 1, 4, seed=77, h0_std=0.5, dt_std=4.0)
    y, state = gpu_ssd_decode(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, state)


def test_ssd_decode_continues_prefill():
    """Decode use: a prefill of 61 tokens, then three decode steps in place on
    its h_last, match the oracle's single run of all 64 tokens."""
    inp = make_ssd_inputs_custom(2, 64, 4, groups=2, seed=45, h0_std=0.2)
    d = to_dev(inp)
    c = dict(d)
    for k in ("x", "z", "dt", "Bm", "Cm"):
        c[k] = d[k][:, :61].contiguous()
    y0, state = gpu_ssd(c)
    ys = [y0]
    for t in range(61, 64):
        c = dict(d)
        for k in ("x", "z", "dt", "Bm", "Cm"):
            c[k] = d[k][:, t:t + 1].contiguous()
        y, state = gpu_ssd_decode(c, state)
        ys.append(y)
    torch.cuda.synchronize()
    check(inp, torch.cat(ys, dim=1), state)


def test_ssd_decode_matches_one_token_prefill():
    """The decode step and the chunked prefill of one token agree (the two
    paths sum in different orders; both within the tolerance of the oracle,
    and close to each other)."""
    inp = make_ssd_inputs_custom(2, 1, 4, groups=1, seed=51, h0_std=0.3)
    d = to_dev(inp)
    yp, hp = gpu_ssd(d)
    yd, hd = gpu_ssd_decode(d)
    torch.cuda.synchronize()
    check(inp, yd, hd)
    assert torch.allclose(hd, hp, rtol=1e-4, atol=1e-4)


def test_ssd_decode_full_size():
    """The decode workload at full size (128 sequences x 128 heads of 64,
    d_state 128: a 512 MB state), as the bench times it: every head of every
    sequence against the oracle."""
    cfg = SSD_CONFIGS["mamba2_decode"]
    inp = make_ssd_inputs(cfg)
    y, state = gpu_ssd_decode(to_dev(inp))
    torch.cuda.synchronize()
    check(inp, y, state)


def test_ssd_decode_graph_replay():
    """Captured in a CUDA graph, two replays from the same state give the
    bits of two eager calls."""
    inp = make_ssd_inputs_custom(2, 1, 4, seed=53, h0_std=0.3)
    d = to_dev(inp)
    s_eager = d["h0"].clone()
    ye1, _ = gpu_ssd_decode(d, s_eager)
    ye2, _ = gpu_ssd_decode(d, s_eager)
    s_graph = d["h0"].clone()
    tok = {k: d[k][:, 0].contiguous() for k in ("x", "z", "dt", "Bm", "Cm")}
    yg = torch.empty_like(ye1[:, 0])
    mm.ssd_state_update(tok["x"], tok["z"], tok["dt"], d["dt_bias"], d["A"], tok["Bm"], tok["Cm"], d["Dskip"],
                        s_graph.clone(), y=yg)      # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mm.ssd_state_update(tok["x"], tok["z"], tok["dt"], d["dt_bias"], d["A"], tok["Bm"], tok["Cm"], d["Dskip"],
                            s_graph, y=yg)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg, ye1[:, 0])
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg, ye2[:, 0])
    assert torch.equal(s_graph, s_eager)

