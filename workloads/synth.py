"""Seeded synthetic inputs for the Mamba mixer core and its decode step.

Shapes and value distributions follow the five workloads the mixer is measured
on: a tiny fp32 case, a Jamba-shaped single-layer prefill (hidden 4096 x
expand 2 = d_inner 8192, d_state 16, conv width 4), a batched prefill with an
initial state, a 256K-token prefill run as 8 carried chunks, and a one-token
decode across 28 stacked Mamba layers at batch 128.

Recipe (the same for every workload unless the workload says otherwise):
  x, z            ~ N(0, 1)                       (act dtype)
  dt (pre-bias)   ~ 0.1 * N(0, 1)                 (act dtype)
  B_t, C_t        ~ N(0, 1), one group shared by all channels (act dtype)
  conv_w          ~ U(-0.5, 0.5)                  (fp32)
  conv_b          = 0                             (fp32)
  dt_bias         = inverse-softplus(v), v log-uniform in [1e-3, 1e-1] (fp32)
  A[d, n]         = -(n + 1)                      (fp32)
  D (skip)        = 1 (tiny case) or ~ N(1, 0.1)  (fp32)
  h0              = absent, or 0.1 * N(0, 1)      (fp32)
  decode states   ssm ~ 0.1 * N(0, 1) fp32, conv window ~ N(0, 1) act dtype

Every tensor draws from its own counter-keyed stream: block ``i`` of tensor
``k`` in a workload with seed ``s`` uses ``numpy.random.SeedSequence([s, k,
i])``, so the values do not depend on how many threads fill them.  Values are
drawn in fp32 (fp64 for the inverse-softplus input) and rounded to the
activation dtype with round-to-nearest-even; every consumer sees exactly those
rounded values.

This module holds no step of the mixer itself.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_BLOCK = 1 << 22  # elements per independently seeded block

# fixed stream ids, one per tensor
_T_XZ, _T_DT, _T_B, _T_C, _T_CONVW, _T_DTB, _T_D, _T_H0, _T_SSM, _T_CONVS, _T_X, _T_Z, _T_CONVB, _T_A = range(14)
_T_BNORM, _T_CNORM, _T_WX, _T_WDT, _T_DTNORM = 14, 15, 16, 17, 18
_T_SSD_X, _T_SSD_Z, _T_SSD_DT, _T_SSD_B, _T_SSD_C, _T_SSD_DTB, _T_SSD_A, _T_SSD_D, _T_SSD_H0 = range(19, 28)
_T_M3_TRAP, _T_M3_THETA, _T_M3_XP, _T_M3_BP = range(28, 32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill_blocks(n: int, seed: int, tid: int, draw) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nblk = (n + _BLOCK - 1) // _BLOCK

    def work(i):
        lo = i * _BLOCK
        hi = min(n, lo + _BLOCK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, i])))
        out[lo:hi] = draw(rng, hi - lo)

    if nblk <= 1:
        for i in range(nblk):
            work(i)
    else:
        with ThreadPoolExecutor(max_workers=min(_threads(), nblk)) as ex:
            list(ex.map(work, range(nblk)))
    return out


def _normal(shape, seed, tid, std=1.0, mean=0.0) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1

    def draw(rng, m):
        v = rng.standard_normal(m, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        if mean != 0.0:
            v += np.float32(mean)
        return v

    return _fill_blocks(n, seed, tid, draw).reshape(shape)


def _uniform(shape, seed, tid, lo, hi) -> np.ndarray:
    n = int(np.prod(shape))

    def draw(rng, m):
        return rng.uniform(lo, hi, m).astype(np.float32)

    return _fill_blocks(n, seed, tid, draw).reshape(shape)


def _dt_bias(shape, seed, tid) -> np.ndarray:
    """dt_bias such that softplus(dt_bias) is log-uniform in [1e-3, 1e-1]."""
    n = int(np.prod(shape))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, 0])))
    v = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), n))  # fp64
    return np.log(np.expm1(v)).astype(np.float32).reshape(shape)


def _act(arr: np.ndarray, act: str) -> torch.Tensor:
    t = torch.from_numpy(arr)
    if act == "bf16":
        return t.to(torch.bfloat16)
    if act == "f32":
        return t.to(torch.float32)
    raise ValueError(f"unknown activation dtype {act!r}")


def _structured_A(lead_shape, N) -> np.ndarray:
    a = -np.arange(1, N + 1, dtype=np.float32)
    return np.broadcast_to(a, tuple(lead_shape) + (N,)).copy()


def _general_A(shape, seed, tid) -> np.ndarray:
    # A = -exp(U(ln 0.5, ln 16)): the negative real diagonal a trained layer has,
    # with no relation between the entries of a row.
    u = _uniform(shape, seed, tid, math.log(0.5), math.log(16.0))
    return (-np.exp(u.astype(np.float64))).astype(np.float32)


@dataclass(frozen=True)
class MixerConfig:
    name: str
    batch: int
    seqlen: int
    d_inner: int
    d_state: int = 16
    d_conv: int = 4
    act: str = "bf16"
    seed: int = 0
    h0_std: float = 0.0          # 0 -> no initial state (zeros)
    dskip: str = "normal"        # "ones" or "normal" (N(1, 0.1))
    chunks: int = 1              # sequential carried calls the sequence is split into
    desc: str = ""

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    layers: int
    batch: int
    d_inner: int
    d_state: int = 16
    d_conv: int = 4
    act: str = "bf16"
    seed: int = 0
    desc: str = ""


CONFIGS = {
    "tiny_f32": MixerConfig(
        "tiny_f32", batch=1, seqlen=256, d_inner=64, act="f32", seed=0, dskip="ones",
        desc="tiny selective-scan forward, fp32 everywhere"),
    "jamba_prefill": MixerConfig(
        "jamba_prefill", batch=1, seqlen=4096, d_inner=8192, seed=1,
        desc="Jamba-shaped single Mamba layer prefill, bf16 activations, fp32 state"),
    "batched_prefill": MixerConfig(
        "batched_prefill", batch=4, seqlen=32768, d_inner=8192, seed=2, h0_std=0.1,
        desc="batched prefill with an initial state h0 ~ 0.1 N(0,1)"),
    "long_256k": MixerConfig(
        "long_256k", batch=1, seqlen=262144, d_inner=8192, seed=3, chunks=8,
        desc="256K-token prefill as 8 sequential 32768-token calls with carried state"),
    "decode_28x128": DecodeConfig(
        "decode_28x128", layers=28, batch=128, d_inner=8192, seed=4,
        desc="one-token state update across 28 stacked Mamba layers, batch 128"),
}


@dataclass(frozen=True)
class SsdConfig:
    """A prefill of the Mamba-2 form: H heads of P channels (d_inner = H P),
    one scalar decay per head and token, B_t/C_t of d_state entries per group."""
    name: str
    batch: int
    seqlen: int
    heads: int
    headdim: int = 64
    d_state: int = 128
    groups: int = 1
    seed: int = 0
    h0_std: float = 0.0
    gate: bool = True
    desc: str = ""

    @property
    def d_inner(self) -> int:
        return self.heads * self.headdim

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


SSD_CONFIGS = {
    "mamba2_prefill": SsdConfig(
        "mamba2_prefill", batch=1, seqlen=4096, heads=128, seed=5,
        desc="Mamba-2 form at the Jamba width: d_inner 8192 as 128 heads of 64, d_state 128, one B/C group"),
    "mamba2_batched": SsdConfig(
        "mamba2_batched", batch=4, seqlen=8192, heads=128, seed=6, h0_std=0.1,
        desc="Mamba-2 form, 4 x 8192 tokens with an initial state"),
    "mamba2_decode": SsdConfig(
        "mamba2_decode", batch=128, seqlen=1, heads=128, seed=8, h0_std=0.3,
        desc="Mamba-2 form, one decode token for 128 sequences at the Jamba width: a 512 MB fp32 state"),
}


def make_ssd_inputs_custom(batch, seqlen, heads, headdim=64, d_state=128, groups=1, seed=0, h0_std=0.0,
                           gate=True, dt_std=0.1):
    """Seeded inputs of the Mamba-2 form as CPU torch tensors.

    x, z [B,L,H*P] ~ N(0,1) (bf16; x is the layer's input after its
    convolution; z None without the gate), dt [B,L,H] ~ dt_std N(0,1) (bf16),
    Bm/Cm [B,L,G,N] ~ N(0,1) (bf16), per head dt_bias = inverse-softplus of a
    log-uniform [1e-3, 1e-1] step, A = -exp(U(ln 1, ln 16)), D ~ N(1, 0.1)
    (fp32), h0 [B,H,P,N] ~ h0_std N(0,1) fp32 or None."""
    B, L, H, P, N, G = batch, seqlen, heads, headdim, d_state, groups
    s = seed
    out = {}
    out["x"] = _act(_normal((B, L, H * P), s, _T_SSD_X), "bf16")
    out["z"] = _act(_normal((B, L, H * P), s, _T_SSD_Z), "bf16") if gate else None
    out["dt"] = _act(_normal((B, L, H), s, _T_SSD_DT, std=dt_std), "bf16")
    out["Bm"] = _act(_normal((B, L, G, N), s, _T_SSD_B), "bf16")
    out["Cm"] = _act(_normal((B, L, G, N), s, _T_SSD_C), "bf16")
    out["dt_bias"] = torch.from_numpy(_dt_bias((H,), s, _T_SSD_DTB))
    u = _uniform((H,), s, _T_SSD_A, 0.0, math.log(16.0))
    out["A"] = torch.from_numpy((-np.exp(u.astype(np.float64))).astype(np.float32))
    out["Dskip"] = torch.from_numpy(_normal((H,), s, _T_SSD_D, std=0.1, mean=1.0))
    out["h0"] = torch.from_numpy(_normal((B, H, P, N), s, _T_SSD_H0, std=h0_std)) if h0_std > 0 else None
    return out


def make_ssd_inputs(cfg: SsdConfig, **overrides):
    kw = dict(batch=cfg.batch, seqlen=cfg.seqlen, heads=cfg.heads, headdim=cfg.headdim, d_state=cfg.d_state,
              groups=cfg.groups, seed=cfg.seed, h0_std=cfg.h0_std, gate=cfg.gate)
    kw.update(overrides)
    return make_ssd_inputs_custom(**kw)


def make_mixer_inputs_custom(batch, seqlen, d_inner, d_state=16, d_conv=4, act="bf16", seed=0,
                             h0_std=0.0, dskip="normal", conv_state_std=0.0, conv_b_std=0.0,
                             A_mode="structured", dt_std=0.1):
    """Seeded mixer-forward inputs as CPU torch tensors.

    Returns a dict with xz [B,L,2D], dt [B,L,D], Bm/Cm [B,L,N] (act dtype),
    conv_w [D,W], conv_b [D], dt_bias [D], A [D,N], Dskip [D] (fp32), and
    h0 [B,D,N] fp32 / conv_state_in [B,D,W-1] act, each None when absent.
    """
    B, L, D, N, W = batch, seqlen, d_inner, d_state, d_conv
    s = seed
    out = {}
    out["xz"] = _act(_normal((B, L, 2 * D), s, _T_XZ), act)
    out["dt"] = _act(_normal((B, L, D), s, _T_DT, std=dt_std), act)
    out["Bm"] = _act(_normal((B, L, N), s, _T_B), act)
    out["Cm"] = _act(_normal((B, L, N), s, _T_C), act)
    out["conv_w"] = torch.from_numpy(_uniform((D, W), s, _T_CONVW, -0.5, 0.5))
    if conv_b_std > 0:
        out["conv_b"] = torch.from_numpy(_normal((D,), s, _T_CONVB, std=conv_b_std))
    else:
        out["conv_b"] = torch.zeros(D, dtype=torch.float32)
    out["dt_bias"] = torch.from_numpy(_dt_bias((D,), s, _T_DTB))
    if A_mode == "structured":
        out["A"] = torch.from_numpy(_structured_A((D,), N))
    elif A_mode == "general":
        out["A"] = torch.from_numpy(_general_A((D, N), s, _T_A))
    else:
        raise ValueError(A_mode)
    if dskip == "ones":
        out["Dskip"] = torch.ones(D, dtype=torch.float32)
    else:
        out["Dskip"] = torch.from_numpy(_normal((D,), s, _T_D, std=0.1, mean=1.0))
    out["h0"] = torch.from_numpy(_normal((B, D, N), s, _T_H0, std=h0_std)) if h0_std > 0 else None
    if conv_state_std > 0:
        out["conv_state_in"] = _act(_normal((B, D, W - 1), s, _T_CONVS, std=conv_state_std), act)
    else:
        out["conv_state_in"] = None
    return out


def make_mixer_inputs(cfg: MixerConfig, **overrides):
    kw = dict(batch=cfg.batch, seqlen=cfg.seqlen, d_inner=cfg.d_inner, d_state=cfg.d_state,
              d_conv=cfg.d_conv, act=cfg.act, seed=cfg.seed, h0_std=cfg.h0_std, dskip=cfg.dskip)
    kw.update(overrides)
    return make_mixer_inputs_custom(**kw)


def make_decode_inputs_custom(layers, batch, d_inner, d_state=16, d_conv=4, act="bf16", seed=0,
                              A_mode="structured", conv_b_std=0.0):
    """Seeded decode-step inputs as CPU torch tensors.

    x, z, dt [NL,B,D] and Bm/Cm [NL,B,N] in the act dtype; per-layer parameters
    conv_w [NL,D,W], conv_b/dt_bias/Dskip [NL,D], A [NL,D,N] in fp32; the carried
    state ssm_state [NL,B,D,N] fp32 and conv_state [NL,B,D,W-1] act dtype.
    """
    NL, B, D, N, W = layers, batch, d_inner, d_state, d_conv
    s = seed
    out = {}
    out["x"] = _act(_normal((NL, B, D), s, _T_X), act)
    out["z"] = _act(_normal((NL, B, D), s, _T_Z), act)
    out["dt"] = _act(_normal((NL, B, D), s, _T_DT, std=0.1), act)
    out["Bm"] = _act(_normal((NL, B, N), s, _T_B), act)
    out["Cm"] = _act(_normal((NL, B, N), s, _T_C), act)
    out["conv_w"] = torch.from_numpy(_uniform((NL, D, W), s, _T_CONVW, -0.5, 0.5))
    if conv_b_std > 0:
        out["conv_b"] = torch.from_numpy(_normal((NL, D), s, _T_CONVB, std=conv_b_std))
    else:
        out["conv_b"] = torch.zeros(NL, D, dtype=torch.float32)
    out["dt_bias"] = torch.from_numpy(_dt_bias((NL, D), s, _T_DTB))
    if A_mode == "structured":
        out["A"] = torch.from_numpy(_structured_A((NL, D), N))
    else:
        out["A"] = torch.from_numpy(_general_A((NL, D, N), s, _T_A))
    out["Dskip"] = torch.from_numpy(_normal((NL, D), s, _T_D, std=0.1, mean=1.0))
    out["ssm_state"] = torch.from_numpy(_normal((NL, B, D, N), s, _T_SSM, std=0.1))
    out["conv_state"] = _act(_normal((NL, B, D, W - 1), s, _T_CONVS), act)
    return out


def make_decode_inputs(cfg: DecodeConfig, **overrides):
    kw = dict(layers=cfg.layers, batch=cfg.batch, d_inner=cfg.d_inner, d_state=cfg.d_state,
              d_conv=cfg.d_conv, act=cfg.act, seed=cfg.seed)
    kw.update(overrides)
    return make_decode_inputs_custom(**kw)


def sample_channels(d_inner: int, count: int = 256) -> np.ndarray:
    """A deterministic channel subset for checks at full size: the first and
    last 8 channels plus an even stride through the rest."""
    if d_inner <= count:
        return np.arange(d_inner)
    if count <= 32:
        return np.unique(np.linspace(0, d_inner - 1, count).round().astype(np.int64))
    edge = list(range(8)) + list(range(d_inner - 8, d_inner))
    stride = max(1, d_inner // (count - 16))
    mid = [d for d in range(3, d_inner, stride) if 8 <= d < d_inner - 8][: count - 16]
    sel = sorted(set(edge + mid))
    return np.array(sel, dtype=np.int64)


def subset_channels(inp: dict, chans) -> dict:
    """Mixer-forward inputs restricted to the channels ``chans`` (a copy).
    Channels are independent given the shared B/C, so a computation on the
    subset equals the full computation restricted to those channels."""
    S = torch.as_tensor(np.asarray(chans), dtype=torch.long)
    D = inp["dt"].shape[-1]
    xz = inp["xz"]
    out = dict(inp)
    out["xz"] = torch.cat([xz[..., :D].index_select(-1, S), xz[..., D:].index_select(-1, S)], dim=-1)
    out["dt"] = inp["dt"].index_select(-1, S)
    for k in ("conv_w", "conv_b", "dt_bias", "A", "Dskip"):
        out[k] = inp[k].index_select(0, S) if inp.get(k) is not None else None
    for k in ("h0", "conv_state_in"):
        out[k] = inp[k].index_select(1, S) if inp.get(k) is not None else None
    return out


def make_norm_weights(d_state: int = 16, layers=None, seed: int = 0):
    """Per-state weights of the RMSNorm of B and C: U(0.5, 1.5) fp32, shape
    [d_state] (forward) or [layers, d_state] (decode).  Returns (b_norm_w,
    c_norm_w)."""
    shape = (d_state,) if layers is None else (layers, d_state)
    wb = _uniform(shape, seed, _T_BNORM, 0.5, 1.5)
    wc = _uniform(shape, seed, _T_CNORM, 0.5, 1.5)
    return torch.from_numpy(wb), torch.from_numpy(wc)


def make_projection_weights(d_inner: int, dt_rank: int = 256, d_state: int = 16, seed: int = 0):
    """Weights of the projections either side of the scan, bf16 (RNE):
    W_x [dt_rank + 2 d_state, d_inner] ~ N(0, 1/d_inner) (so x_proj keeps the
    scale of u), W_dt [d_inner, dt_rank] ~ N(0, 0.01/dt_rank) (so dt keeps the
    workloads' 0.1 N(0, 1) scale for unit-rms dt_low), and the RMSNorm weight
    of dt_low [dt_rank] ~ U(0.5, 1.5) fp32.  Returns (W_x, W_dt, dt_norm_w)."""
    wx = _normal((dt_rank + 2 * d_state, d_inner), seed, _T_WX, std=1.0 / math.sqrt(d_inner))
    wdt = _normal((d_inner, dt_rank), seed, _T_WDT, std=0.1 / math.sqrt(dt_rank))
    wn = _uniform((dt_rank,), seed, _T_DTNORM, 0.5, 1.5)
    return _act(wx, "bf16"), _act(wdt, "bf16"), torch.from_numpy(wn)



@dataclass(frozen=True)
class M3Config:
    """A prefill of the Mamba-3 form: H heads of P channels, each channel's
    d_state entries as d_state/2 complex numbers, R inputs and outputs
    sharing a state (R = 1: single input)."""
    name: str
    batch: int
    seqlen: int
    heads: int
    headdim: int = 64
    d_state: int = 16
    groups: int = 1
    rank: int = 1
    seed: int = 0
    h0_std: float = 0.0
    prev: bool = False
    gate: bool = True
    desc: str = ""

    @property
    def d_inner(self) -> int:
        return self.heads * self.headdim

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


M3_CONFIGS = {
    "mamba3_prefill": M3Config(
        "mamba3_prefill", batch=1, seqlen=4096, heads=128, seed=7,
        desc="Mamba-3 form at the Jamba width: 128 heads of 64, d_state 16 (8 complex pairs), one input"),
    "mamba3_mimo": M3Config(
        "mamba3_mimo", batch=1, seqlen=4096, heads=128, rank=4, seed=8, h0_std=0.1, prev=True,
        desc="Mamba-3 form with 4 inputs and outputs per state, an initial state and a previous token"),
    "mamba3_decode": M3Config(
        "mamba3_decode", batch=512, seqlen=1, heads=128, seed=9, h0_std=0.3, prev=True,
        desc="Mamba-3 form, one decode token for 512 sequences at the Jamba width (a 268 MB fp32 state), "
             "the previous token given"),
}


def make_m3_inputs_custom(batch, seqlen, heads, headdim=64, d_state=16, groups=1, rank=1, seed=0, h0_std=0.0,
                          prev=False, gate=True, trap=True, dt_std=0.1):
    """Seeded inputs of the Mamba-3 form as CPU torch tensors.

    x, z [B,L,R,H*P] ~ N(0,1) (bf16; z None without the gate), dt [B,L,H] ~
    dt_std N(0,1) (bf16), trap [B,L,H] ~ U(0,1) (bf16; None: 1/2),
    Bm/Cm [B,L,R,G,N] ~ N(0,1) (bf16); per head dt_bias = inverse-softplus of
    a log-uniform [1e-3, 1e-1] step, A = -exp(U(ln 1, ln 16)), D ~ N(1, 0.1),
    rotation frequencies theta [H, N/2] ~ U(-2, 2) (fp32); h0 [B,H,P,N] ~
    h0_std N(0,1) fp32 or None; x_prev [B,R,H*P] and B_prev [B,R,G,N] ~ N(0,1)
    (bf16) when prev."""
    B, L, H, P, N, G, R = batch, seqlen, heads, headdim, d_state, groups, rank
    s = seed
    out = {}
    out["x"] = _act(_normal((B, L, R, H * P), s, _T_SSD_X), "bf16")
    out["z"] = _act(_normal((B, L, R, H * P), s, _T_SSD_Z), "bf16") if gate else None
    out["dt"] = _act(_normal((B, L, H), s, _T_SSD_DT, std=dt_std), "bf16")
    out["trap"] = _act(_uniform((B, L, H), s, _T_M3_TRAP, 0.0, 1.0), "bf16") if trap else None
    out["Bm"] = _act(_normal((B, L, R, G, N), s, _T_SSD_B), "bf16")
    out["Cm"] = _act(_normal((B, L, R, G, N), s, _T_SSD_C), "bf16")
    out["dt_bias"] = torch.from_numpy(_dt_bias((H,), s, _T_SSD_DTB))
    u = _uniform((H,), s, _T_SSD_A, 0.0, math.log(16.0))
    out["A"] = torch.from_numpy((-np.exp(u.astype(np.float64))).astype(np.float32))
    out["theta"] = torch.from_numpy(_uniform((H, N // 2), s, _T_M3_THETA, -2.0, 2.0))
    out["Dskip"] = torch.from_numpy(_normal((H,), s, _T_SSD_D, std=0.1, mean=1.0))
    out["h0"] = torch.from_numpy(_normal((B, H, P, N), s, _T_SSD_H0, std=h0_std)) if h0_std > 0 else None
    out["x_prev"] = _act(_normal((B, R, H * P), s, _T_M3_XP), "bf16") if prev else None
    out["B_prev"] = _act(_normal((B, R, G, N), s, _T_M3_BP), "bf16") if prev else None
    return out


def make_m3_inputs(cfg: M3Config, **overrides):
    kw = dict(batch=cfg.batch, seqlen=cfg.seqlen, heads=cfg.heads, headdim=cfg.headdim, d_state=cfg.d_state,
              groups=cfg.groups, rank=cfg.rank, seed=cfg.seed, h0_std=cfg.h0_std, prev=cfg.prev, gate=cfg.gate)
    kw.update(overrides)
    return make_m3_inputs_custom(**kw)
