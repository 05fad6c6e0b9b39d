"""The C-ABI library on the host, without a GPU: it loads, exports every
function the public header declares, and rejects bad arguments with the
documented status before touching the device.  Pointers here are fake
addresses, so every call that takes them runs in a child process that sees no
CUDA device (abi_nodevice): arguments that pass validation stop at the device
check with MM_ERR_DEVICE and nothing is launched, whether or not the machine
running the tests has a GPU."""

import ctypes
import os
import re

import pytest

import mamba_selective_scan_core_b200 as mm
from abi_nodevice import NoDeviceLib
from ws_layout import ws_bytes
from mamba_selective_scan_core_b200 import build as mmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mamba_mixer.h")

OK, ENULL, ESHAPE, EALIGN, EDTYPE, EALIAS, EUNSUP, ECUDA, EDEVICE, EWORKSPACE, ESCRATCH, ETIMEOUT, EARG = range(13)


@pytest.fixture(scope="module")
def L():
    """The library's entry points, called in a process with no visible device."""
    mmbuild.build()
    mm.lib()
    worker = NoDeviceLib()
    yield worker
    worker.close()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mamba_\w+)\s*\(", src)))


def test_header_declares_expected_api():
    assert set(declared_functions()) == set(mm.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    mmbuild.build()
    lib = mm.lib()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from {mm.library_path()}"


def test_checked_build_exports_the_same_symbols():
    """The checked build (index checks in the forward and decode kernels)
    is the same C ABI: every declared function, C linkage."""
    path = mmbuild.build_checked()
    out = os.popen(f"nm -D --defined-only {path}").read()
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in names, f"{name} missing from {path}"


def test_exported_symbols_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {mm.library_path()}").read()
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in names


def test_version_and_strings():
    mmbuild.build()
    assert mm.abi_version() == 8
    for code in range(14):
        s = mm.status_string(code)
        assert s and s != "unknown status"
    assert mm.status_string(99) == "unknown status"
    # the plan on a machine without a GPU is a B200's (148 SMs).  One
    # 8192-channel sequence (128 warps of channel pairs) is split into 9 time
    # chunks of 480 tokens: 8 carried chunk boundaries
    assert mm.workspace_size(1, 4096, 8192) == ws_bytes(1, 9, 8192)
    # two such sequences: 4 chunks; three: 3 chunks
    assert mm.workspace_size(2, 4096, 8192) == ws_bytes(2, 4, 8192)
    assert mm.workspace_size(3, 4096, 8192) == ws_bytes(3, 3, 8192)
    # four: one chunk (their 512 warps fill the SMs well enough that a summary
    # pass over half the tokens would cost more than it gains)
    assert mm.workspace_size(4, 32768, 8192) == 256
    # enough sequences need no time chunks: only the status header
    assert mm.workspace_size(8, 4096, 8192) == 256
    assert mm.workspace_size(1, 0, 8192) == 256
    assert mm.workspace_size(1, 4096, 8192, act=5) == 0


# ---------------------------------------------------------------- mixer_fwd validation
BASE = 0x7F0000000000   # a fake, 16-byte-aligned device address region
WS_ADDR = BASE + (1 << 40)   # a fake workspace address, clear of every buffer


def fwd_args(B=1, Lq=64, D=64, N=16, W=4, act=1, **over):
    es = 4 if act == 0 else 2
    sizes = dict(xz=B * Lq * 2 * D * es, conv_w=D * W * 4, conv_b=D * 4, dt=B * Lq * D * es, dt_bias=D * 4,
                 A=D * N * 4, Bm=B * Lq * N * es, Cm=B * Lq * N * es, Dskip=D * 4, h0=B * D * N * 4,
                 cs_in=B * D * (W - 1) * es, y=B * Lq * D * es, h_last=B * D * N * 4,
                 cs_out=B * D * (W - 1) * es)
    ptrs = {}
    addr = BASE
    for k, v in sizes.items():
        ptrs[k] = addr
        addr += (v + 4095) // 4096 * 4096 + 4096
    ptrs.update(over)
    order = ["xz", "conv_w", "conv_b", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "h0", "cs_in",
             "y", "h_last", "cs_out"]
    # a fake workspace of the size the plan needs, far from the buffers
    ws_need = mm.workspace_size(max(B, 1), max(Lq, 0), D) if B >= 0 and Lq >= 0 and D > 0 and D % 8 == 0 else 256
    return [ptrs[k] for k in order] + [B, Lq, D, N, W, act, WS_ADDR, max(ws_need, 256), None]


def call_fwd(L, **kw):
    return L.mamba_mixer_fwd(*fwd_args(**kw))


def test_fwd_workspace_rules(L):
    # B1 L4096 D64 has 2 warps of channels: the plan splits time and needs scratch
    need = mm.workspace_size(1, 4096, 64)
    assert need > 256
    args = fwd_args(B=1, Lq=4096, D=64)
    ws_addr = BASE + (1 << 36)
    ok = list(args)
    ok[-3], ok[-2] = ws_addr, need
    assert L.mamba_mixer_fwd(*ok) == EDEVICE
    missing = list(args)
    missing[-3], missing[-2] = None, need
    assert L.mamba_mixer_fwd(*missing) == 9
    small = list(args)
    small[-3], small[-2] = ws_addr, need - 4
    assert L.mamba_mixer_fwd(*small) == 9
    mis = list(args)
    mis[-3], mis[-2] = ws_addr + 4, need
    assert L.mamba_mixer_fwd(*mis) == EALIGN
    alias = list(args)
    alias[-3], alias[-2] = args[11], need          # workspace over y
    assert L.mamba_mixer_fwd(*alias) == EALIAS


def test_fwd_valid_arguments_reach_the_device_check(L):
    # everything valid: validation passes and the call stops at the device check
    st = call_fwd(L)
    assert st == EDEVICE


def test_fwd_batch_zero_is_a_noop(L):
    assert call_fwd(L, B=0) == OK


@pytest.mark.parametrize("act", [2, -1])
def test_fwd_bad_dtype(L, act):
    assert call_fwd(L, act=act) == EDTYPE


@pytest.mark.parametrize("kw", [dict(B=-1), dict(Lq=-1), dict(D=0), dict(D=-8), dict(N=0), dict(W=0)])
def test_fwd_bad_shape(L, kw):
    assert call_fwd(L, **kw) == ESHAPE


@pytest.mark.parametrize("kw", [dict(N=8), dict(N=32), dict(W=3), dict(W=2), dict(D=12), dict(D=65)])
def test_fwd_unsupported(L, kw):
    assert call_fwd(L, **kw) == EUNSUP


def test_fwd_overflowing_sizes(L):
    assert call_fwd(L, B=1 << 20, Lq=1 << 40) == ESHAPE


def test_fwd_sequence_length_bound(L):
    # one sequence's xz rows (seqlen x 2 d_inner elements) must span less than
    # 2^40 bytes, the bulk copy engine's stride limit: 2^25 tokens at d_inner
    # 8192 in bf16 is exactly 2^40
    assert call_fwd(L, Lq=1 << 25, D=8192) == ESHAPE
    assert mm.workspace_size(1, 1 << 25, 8192) == 0
    assert call_fwd(L, Lq=(1 << 25) - 32, D=8192) != ESHAPE
    assert mm.workspace_size(1, (1 << 25) - 32, 8192) > 0
    assert call_fwd(L, Lq=(1 << 30) + 1, D=8) == ESHAPE
    # the host-memory forward bounds each piece (about an eighth of the sequence) instead
    assert mm.host_workspace_size(1, 1 << 25, 8192) > 0
    assert mm.host_workspace_size(1, 1 << 29, 8192) == 0


@pytest.mark.parametrize("name", ["xz", "conv_w", "dt", "dt_bias", "A", "Bm", "Cm", "y", "h_last", "cs_out"])
def test_fwd_required_null(L, name):
    assert call_fwd(L, **{name: None}) == ENULL


@pytest.mark.parametrize("name", ["conv_b", "Dskip", "h0", "cs_in"])
def test_fwd_optional_null_passes_validation(L, name):
    assert call_fwd(L, **{name: None}) == EDEVICE


def test_fwd_seqlen_zero_needs_no_token_buffers(L):
    assert call_fwd(L, Lq=0, xz=None, dt=None, Bm=None, Cm=None, y=None) == EDEVICE


@pytest.mark.parametrize("name", ["xz", "conv_w", "conv_b", "dt", "A", "Bm", "h0", "cs_in", "y", "h_last", "cs_out"])
def test_fwd_misaligned(L, name):
    args = fwd_args()
    base = dict(zip(["xz", "conv_w", "conv_b", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "h0", "cs_in",
                     "y", "h_last", "cs_out"], args[:14]))
    assert call_fwd(L, **{name: base[name] + 8}) == EALIGN


@pytest.mark.parametrize("out,inp", [("y", "xz"), ("y", "dt"), ("h_last", "h0"), ("cs_out", "cs_in"),
                                     ("y", "Bm"), ("h_last", "A"), ("y", "h_last"), ("cs_out", "y")])
def test_fwd_alias(L, out, inp):
    args = fwd_args()
    names = ["xz", "conv_w", "conv_b", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "h0", "cs_in",
             "y", "h_last", "cs_out"]
    base = dict(zip(names, args[:14]))
    assert call_fwd(L, **{out: base[inp]}) == EALIAS


def test_fwd_partial_overlap_is_alias(L):
    args = fwd_args()
    names = ["xz", "conv_w", "conv_b", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "h0", "cs_in",
             "y", "h_last", "cs_out"]
    base = dict(zip(names, args[:14]))
    # y starting 16 bytes before the end of dt
    dt_bytes = 1 * 64 * 64 * 2
    assert call_fwd(L, y=base["dt"] + dt_bytes - 16) == EALIAS


# ---------------------------------------------------------------- fused RMSNorm of B and C
def normed_args(wb=None, wc=None, eps=1e-6, **kw):
    a = fwd_args(**kw)
    return a[:-3] + [wb, wc, eps] + a[-3:]


NORM_W = BASE + (1 << 39)    # fake weight rows, clear of every buffer


def test_normed_fwd_validation(L):
    # valid: stops at the device check; no weight at all is the plain forward
    assert L.mamba_mixer_fwd_normed(*normed_args(NORM_W, NORM_W + 256)) == EDEVICE
    assert L.mamba_mixer_fwd_normed(*normed_args(None, None, eps=0.0)) == EDEVICE
    # eps must be positive and finite once a weight is given
    for eps in (0.0, -1.0, float("inf"), float("nan")):
        assert L.mamba_mixer_fwd_normed(*normed_args(NORM_W, None, eps=eps)) == EARG
        assert L.mamba_mixer_fwd_normed(*normed_args(None, NORM_W, eps=eps)) == EARG
    assert L.mamba_mixer_fwd_normed(*normed_args(NORM_W + 4, None)) == EALIGN
    # a weight under an output
    y_addr = fwd_args()[11]
    assert L.mamba_mixer_fwd_normed(*normed_args(y_addr, None)) == EALIAS
    # the same argument checks as the plain forward come first
    assert L.mamba_mixer_fwd_normed(*normed_args(NORM_W, None, xz=None)) == ENULL


def test_normed_decode_validation(L):
    def args(wb, wc, eps=1e-6, **kw):
        a = upd_args(**kw)
        return a[:-1] + [wb, wc, eps, a[-1]]

    assert L.mamba_state_update_normed(*args(NORM_W, NORM_W + 4096)) == EDEVICE
    assert L.mamba_state_update_normed(*args(NORM_W, None, eps=0.0)) == EARG
    assert L.mamba_state_update_normed(*args(NORM_W + 8, None)) == EALIGN
    assert L.mamba_state_update_normed(*args(upd_args()[12], None)) == EALIAS     # weight under y


# ---------------------------------------------------------------- projections
def test_proj_matmul_validation(L):
    A, W, O, WS = BASE, BASE + (1 << 33), BASE + (1 << 34), BASE + (1 << 35)
    need = mm.proj_matmul_workspace_size(4096, 288, 8192)
    # x_proj's shape splits K four ways on 148 SMs: fp32 partials after the status
    assert need == 256 + 4 * 4096 * 288 * 4
    assert mm.proj_matmul_workspace_size(256, 8192, 256) == 256
    assert L.mamba_proj_matmul(A, W, O, 4096, 288, 8192, 1, WS, need, None) == EDEVICE
    assert L.mamba_proj_matmul(A, W, O, 4096, 288, 8192, 1, WS, need - 16, None) == EWORKSPACE
    assert L.mamba_proj_matmul(A, W, O, 64, 64, 64, 3, WS, 256, None) == EDTYPE
    assert L.mamba_proj_matmul(A, W, O, 64, 64, 60, 0, WS, 256, None) == EUNSUP
    assert L.mamba_proj_matmul(A, W, O, 64, 60, 64, 0, WS, 256, None) == EUNSUP
    assert L.mamba_proj_matmul(A, W, O, -1, 64, 64, 0, WS, 256, None) == ESHAPE
    assert L.mamba_proj_matmul(A, W, O, 0, 64, 64, 0, None, 0, None) == OK
    assert L.mamba_proj_matmul(None, W, O, 64, 64, 64, 0, WS, 256, None) == ENULL
    assert L.mamba_proj_matmul(A + 8, W, O, 64, 64, 64, 0, WS, 256, None) == EALIGN
    assert L.mamba_proj_matmul(A, W, A, 64, 64, 64, 0, WS, 256, None) == EALIAS
    assert L.mamba_proj_matmul(A, W, O, 64, 64, 64, 0, O, 256, None) == EALIAS


def test_projected_validation(L):
    a = fwd_args(B=1, Lq=64, D=64)
    xz, conv_w, conv_b, dt_bias, A, Dskip = a[0], a[1], a[2], a[4], a[5], a[8]
    y, h, cs = a[11], a[12], a[13]
    WX, WDT, WS, NW = BASE + (1 << 33), BASE + (1 << 34), BASE + (1 << 35), BASE + (1 << 36)
    need = mm.projected_workspace_size(1, 64, 64, 32)
    assert need > 256

    def call(act=1, R=32, D=64, eps=1e-6, wd=None, ws=WS, ws_bytes=None, **over):
        return L.mamba_mixer_fwd_projected(over.get("xz", xz), conv_w, conv_b, WX, WDT, dt_bias, A, Dskip, None, None,
                                           wd, None, None, eps, y, h, cs, 1, 64, D, 16, R, 4, act, ws,
                                           need if ws_bytes is None else ws_bytes, None)

    assert call() == EDEVICE
    assert call(wd=NW) == EDEVICE
    assert call(act=0) == EUNSUP
    assert call(R=30) == EUNSUP
    assert call(D=72) == EUNSUP
    assert call(wd=NW, eps=0.0) == EARG
    assert call(ws_bytes=need - 16) == EWORKSPACE
    assert call(ws=xz) == EALIAS           # the workspace over an input
    assert call(xz=None) == ENULL


# ---------------------------------------------------------------- Mamba-2 form
def ssd_args(B=2, Lq=300, H=4, P=64, N=128, G=2, ws_bytes=None, **over):
    """mamba_ssd_fwd arguments on fake addresses, each buffer 2^32 apart."""
    names = ["x", "z", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "h0", "y", "h_last"]
    addr = {n: BASE + (i << 32) for i, n in enumerate(names)}
    addr.update(over)
    ws = over.get("ws", WS_ADDR)
    need = mm.ssd_workspace_size(max(B, 1), Lq, H, P, N, G) if ws_bytes is None else ws_bytes
    return [addr[n] for n in names] + [B, Lq, H, P, N, G, ws, need, None]


def test_ssd_workspace_size_rules():
    # header, fp32 chunk states, entering states as two bf16 parts, fp32 chunk
    # decays: 4096 tokens are 32 chunks of 128; 128 heads of 64 x 128 states
    states = 32 * 128 * 64 * 128
    assert mm.ssd_workspace_size(1, 4096, 128) == 256 + states * 4 + states * 4 + 128 * 32 * 4
    assert mm.ssd_workspace_size(1, 0, 128) == 256
    assert mm.ssd_workspace_size(1, 4096, 128, headdim=32) == 0
    assert mm.ssd_workspace_size(1, 4096, 128, d_state=64) == 0
    assert mm.ssd_workspace_size(1, 4096, 6, groups=4) == 0
    assert mm.ssd_workspace_size(0, 4096, 128) == 0


def test_ssd_validation(L):
    assert L.mamba_ssd_fwd(*ssd_args()) == EDEVICE
    assert L.mamba_ssd_fwd(*ssd_args(z=None, dt_bias=None, Dskip=None, h0=None)) == EDEVICE
    assert L.mamba_ssd_fwd(*ssd_args(P=32)) == EUNSUP
    assert L.mamba_ssd_fwd(*ssd_args(N=64)) == EUNSUP
    assert L.mamba_ssd_fwd(*ssd_args(H=6, G=4)) == ESHAPE
    assert L.mamba_ssd_fwd(*ssd_args(G=0)) == ESHAPE
    assert L.mamba_ssd_fwd(*ssd_args(Lq=-1, ws_bytes=0)) == ESHAPE
    assert L.mamba_ssd_fwd(*ssd_args(B=0, ws_bytes=0)) == OK
    for name in ("x", "dt", "A", "Bm", "Cm", "y", "h_last"):
        assert L.mamba_ssd_fwd(*ssd_args(**{name: None})) == ENULL, name
    # no token: only A and h_last are needed
    assert L.mamba_ssd_fwd(*ssd_args(Lq=0, x=None, dt=None, Bm=None, Cm=None, y=None)) == EDEVICE
    for name in ("x", "Bm", "h0", "y", "dt_bias"):
        assert L.mamba_ssd_fwd(*ssd_args(**{name: BASE + (1 << 40) + 8})) == EALIGN, name
    assert L.mamba_ssd_fwd(*ssd_args(y=BASE)) == EALIAS                      # y over x
    assert L.mamba_ssd_fwd(*ssd_args(h_last=BASE + (8 << 32))) == EALIAS     # h_last over h0
    assert L.mamba_ssd_fwd(*ssd_args(h_last=BASE + (9 << 32) + 64)) == EALIAS   # h_last over y
    assert L.mamba_ssd_fwd(*ssd_args(ws=BASE + (5 << 32))) == EALIAS         # workspace over B
    need = mm.ssd_workspace_size(2, 300, 4, 64, 128, 2)
    assert L.mamba_ssd_fwd(*ssd_args(ws_bytes=need - 16)) == EWORKSPACE
    assert L.mamba_ssd_fwd(*ssd_args(ws=None)) == EWORKSPACE
    assert L.mamba_ssd_fwd(*ssd_args(ws=WS_ADDR + 8)) == EALIGN


def ssd_decode_args(B=2, H=4, P=64, N=128, G=2, **over):
    """mamba_ssd_state_update arguments on fake addresses, each buffer 2^32 apart."""
    names = ["x", "z", "dt", "dt_bias", "A", "Bm", "Cm", "Dskip", "state", "y"]
    addr = {n: BASE + (i << 32) for i, n in enumerate(names)}
    addr.update(over)
    return [addr[n] for n in names] + [B, H, P, N, G, None]


def test_ssd_decode_validation(L):
    assert L.mamba_ssd_state_update(*ssd_decode_args()) == EDEVICE
    assert L.mamba_ssd_state_update(*ssd_decode_args(z=None, dt_bias=None, Dskip=None)) == EDEVICE
    assert L.mamba_ssd_state_update(*ssd_decode_args(P=32)) == EUNSUP
    assert L.mamba_ssd_state_update(*ssd_decode_args(N=64)) == EUNSUP
    assert L.mamba_ssd_state_update(*ssd_decode_args(H=6, G=4)) == ESHAPE
    assert L.mamba_ssd_state_update(*ssd_decode_args(G=0)) == ESHAPE
    assert L.mamba_ssd_state_update(*ssd_decode_args(B=-1)) == ESHAPE
    assert L.mamba_ssd_state_update(*ssd_decode_args(B=70000)) == ESHAPE
    assert L.mamba_ssd_state_update(*ssd_decode_args(B=0)) == OK
    for name in ("x", "dt", "A", "Bm", "Cm", "state", "y"):
        assert L.mamba_ssd_state_update(*ssd_decode_args(**{name: None})) == ENULL, name
    for name in ("x", "z", "Cm", "state", "y", "Dskip"):
        assert L.mamba_ssd_state_update(*ssd_decode_args(**{name: BASE + (1 << 40) + 8})) == EALIGN, name
    assert L.mamba_ssd_state_update(*ssd_decode_args(y=BASE)) == EALIAS                  # y over x
    assert L.mamba_ssd_state_update(*ssd_decode_args(state=BASE + (5 << 32))) == EALIAS  # state over B
    assert L.mamba_ssd_state_update(*ssd_decode_args(y=BASE + (8 << 32) + 64)) == EALIAS # y over state


# ---------------------------------------------------------------- Mamba-3 form
def m3_args(B=2, Lq=300, R=2, H=4, P=64, N=16, G=2, ws_bytes=None, **over):
    """mamba_m3_fwd arguments on fake addresses, each buffer 2^32 apart."""
    names = ["x", "z", "dt", "trap", "dt_bias", "A", "theta", "Bm", "Cm", "Dskip", "h0", "x_prev", "B_prev",
             "y", "h_last"]
    addr = {n: BASE + (i << 32) for i, n in enumerate(names)}
    addr.update(over)
    ws = over.get("ws", WS_ADDR)
    need = mm.m3_workspace_size(max(B, 1), Lq, H, R, P, N, G) if ws_bytes is None else ws_bytes
    return [addr[n] for n in names] + [B, Lq, R, H, P, N, G, ws, need, None]


def test_m3_workspace_size_rules():
    # 4096 tokens of one sequence with 128 heads: 64 CTAs of 128 channels a
    # chunk; 8 CTAs on each of 148 SMs want 19 chunks, of 7 tiles (224
    # tokens), so 19 chunks and 18 chunk end states (fp32, 16 per channel) and
    # 18 products per head
    assert mm.m3_workspace_size(1, 4096, 128) == 256 + 18 * 8192 * 16 * 4 + 18 * 128 * 16 * 4
    assert mm.m3_workspace_size(1, 0, 128) == 256
    assert mm.m3_workspace_size(1, 4096, 128, rank=3) == 0
    assert mm.m3_workspace_size(1, 4096, 128, d_state=32) == 0
    assert mm.m3_workspace_size(1, 4096, 3) == 0


def test_m3_validation(L):
    assert L.mamba_m3_fwd(*m3_args()) == EDEVICE
    assert L.mamba_m3_fwd(*m3_args(z=None, trap=None, dt_bias=None, Dskip=None, h0=None, x_prev=None,
                                   B_prev=None)) == EDEVICE
    assert L.mamba_m3_fwd(*m3_args(P=32)) == EUNSUP
    assert L.mamba_m3_fwd(*m3_args(N=32)) == EUNSUP
    assert L.mamba_m3_fwd(*m3_args(R=3)) == EUNSUP
    assert L.mamba_m3_fwd(*m3_args(H=3, G=1)) == EUNSUP
    assert L.mamba_m3_fwd(*m3_args(H=6, G=4)) == ESHAPE
    assert L.mamba_m3_fwd(*m3_args(Lq=-1, ws_bytes=0)) == ESHAPE
    assert L.mamba_m3_fwd(*m3_args(B=0, ws_bytes=0)) == OK
    for name in ("x", "dt", "A", "theta", "Bm", "Cm", "y", "h_last"):
        assert L.mamba_m3_fwd(*m3_args(**{name: None})) == ENULL, name
    assert L.mamba_m3_fwd(*m3_args(x_prev=None)) == ENULL       # x_prev and B_prev together
    assert L.mamba_m3_fwd(*m3_args(Lq=0, x=None, dt=None, Bm=None, Cm=None, y=None)) == EDEVICE
    for name in ("x", "trap", "theta", "B_prev", "y"):
        assert L.mamba_m3_fwd(*m3_args(**{name: BASE + (1 << 40) + 8})) == EALIGN, name
    assert L.mamba_m3_fwd(*m3_args(y=BASE)) == EALIAS                        # y over x
    assert L.mamba_m3_fwd(*m3_args(h_last=BASE + (10 << 32))) == EALIAS      # h_last over h0
    assert L.mamba_m3_fwd(*m3_args(ws=BASE + (7 << 32))) == EALIAS           # workspace over B
    need = mm.m3_workspace_size(2, 300, 4, 2, 64, 16, 2)
    assert L.mamba_m3_fwd(*m3_args(ws_bytes=need - 16)) == EWORKSPACE


# ---------------------------------------------------------------- state_update validation
def upd_args(NL=2, B=3, D=64, N=16, W=4, act=1, **over):
    es = 4 if act == 0 else 2
    rows = NL * B * D
    sizes = dict(x=rows * es, z=rows * es, dt=rows * es, conv_w=NL * D * W * 4, conv_b=NL * D * 4,
                 dt_bias=NL * D * 4, Dskip=NL * D * 4, A=NL * D * N * 4, Bm=NL * B * N * es,
                 Cm=NL * B * N * es, ssm=rows * N * 4, cs=rows * (W - 1) * es, y=rows * es)
    ptrs = {}
    addr = BASE
    for k, v in sizes.items():
        ptrs[k] = addr
        addr += (v + 4095) // 4096 * 4096 + 4096
    ptrs.update(over)
    order = ["x", "z", "dt", "conv_w", "conv_b", "dt_bias", "Dskip", "A", "Bm", "Cm", "ssm", "cs", "y"]
    return [ptrs[k] for k in order] + [NL, B, D, N, W, act, None]


def call_upd(L, **kw):
    return L.mamba_state_update(*upd_args(**kw))


def test_update_valid_reaches_device_check(L):
    assert call_upd(L) == EDEVICE


def test_update_empty_is_noop(L):
    assert call_upd(L, NL=0) == OK
    assert call_upd(L, B=0) == OK


@pytest.mark.parametrize("name", ["x", "z", "dt", "conv_w", "dt_bias", "A", "Bm", "Cm", "ssm", "cs", "y"])
def test_update_required_null(L, name):
    assert call_upd(L, **{name: None}) == ENULL


@pytest.mark.parametrize("kw,code", [(dict(act=3), EDTYPE), (dict(N=4), EUNSUP), (dict(W=5), EUNSUP),
                                     (dict(D=20), EUNSUP), (dict(NL=-1), ESHAPE)])
def test_update_bad_sizes(L, kw, code):
    assert call_upd(L, **kw) == code


def test_update_alias(L):
    args = upd_args()
    assert call_upd(L, y=args[0]) == EALIAS          # y over x
    assert call_upd(L, cs=args[10]) == EALIAS        # conv_state over ssm_state
    assert call_upd(L, ssm=args[7]) == EALIAS        # state over A


def test_update_misaligned(L):
    args = upd_args()
    assert call_upd(L, ssm=args[10] + 4) == EALIGN


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    # the binding never falls back: a missing library is an ImportError
    monkeypatch.setattr(mm, "_lib", None)
    monkeypatch.setattr(mm, "library_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        mm.lib()


def test_noalloc_rejects_sizes_beyond_its_scratch(L, monkeypatch):
    # 16 forced time chunks over 65536 channels need 15 * 65536 * 68 bytes of
    # scratch, more than the built-in 8 MiB: rejected before any launch
    monkeypatch.setenv("MAMBA_MIXER_CHUNKS", "16")
    L.setenv("MAMBA_MIXER_CHUNKS", "16")
    try:
        args = fwd_args(B=8, Lq=4096, D=8192)
        assert mm.workspace_size(8, 4096, 8192) > 8 << 20
        noalloc = args[:-3] + [args[-1]]          # same arguments without workspace and its size
        assert L.mamba_mixer_fwd_noalloc(*noalloc) == ESCRATCH
    finally:
        L.setenv("MAMBA_MIXER_CHUNKS", None)


def test_noalloc_validates_like_the_forward(L):
    args = fwd_args()
    noalloc = args[:-3] + [args[-1]]
    bad = list(noalloc)
    bad[0] = None                             # xz
    assert L.mamba_mixer_fwd_noalloc(*bad) == ENULL
    assert L.mamba_mixer_fwd_noalloc(*noalloc) == EDEVICE


def test_noalloc_argument_checks_come_before_the_scratch_limit(L, monkeypatch):
    # sizes beyond the built-in scratch, but an argument mamba_mixer_fwd would
    # reject: the forward's own error wins
    L.setenv("MAMBA_MIXER_CHUNKS", "16")
    try:
        args = fwd_args(B=8, Lq=4096, D=8192)
        noalloc = args[:-3] + [args[-1]]
        for idx, value, code in ((0, None, ENULL), (3, args[3] + 8, EALIGN), (11, args[0], EALIAS)):
            bad = list(noalloc)
            bad[idx] = value
            assert L.mamba_mixer_fwd_noalloc(*bad) == code
    finally:
        L.setenv("MAMBA_MIXER_CHUNKS", None)


def test_check_status_arguments(L):
    # a misaligned workspace is rejected before any device access
    assert L.mamba_check_status(BASE + 8, None) == EALIGN
    # with no device, reading the status (or the noalloc scratch's) fails cleanly
    assert L.mamba_check_status(BASE, None) == ECUDA
    assert L.mamba_check_status(None, None) in (ECUDA, EDEVICE)


# ---------------------------------------------------------------- host-memory forward
def host_args(B=1, Lq=64, D=64, ws=None, ws_bytes=0, **over):
    """mamba_mixer_fwd_host arguments over fake addresses (the same layout as
    fwd_args, reused for host and device buffers alike)."""
    a = fwd_args(B=B, Lq=Lq, D=D, **over)
    return a[:-3] + [ws, ws_bytes, None, None, None]


def test_host_workspace_size_rules():
    need = mm.host_workspace_size(1, 4096, 8192)
    # two staging slots of one 512-token piece (xz, dt, B, C, y in bf16) plus
    # two carried states and the piece forward's scratch
    piece_bytes = 512 * (2 * 8192 + 8192 + 16 + 16 + 8192) * 2
    assert need >= 2 * piece_bytes + 2 * 8192 * (16 * 4 + 3 * 2)
    assert need < 2 * piece_bytes + (16 << 20)
    assert mm.host_workspace_size(1, 0, 64) > 0           # an empty sequence still carries its state
    assert mm.host_workspace_size(1, 4096, 60) == 0       # d_inner % 8 != 0
    assert mm.host_workspace_size(0, 4096, 64) == 0
    assert mm.host_workspace_size(1, 4096, 64, act=7) == 0


def test_host_fwd_validates_before_any_copy(L):
    need = mm.host_workspace_size(2, 1000, 64)
    ws = BASE + (1 << 36)
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=ws, ws_bytes=need, xz=None)) == ENULL
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=ws, ws_bytes=need, act=5)) == EDTYPE
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=ws, ws_bytes=need - 1)) == EWORKSPACE
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=None, ws_bytes=0)) == EWORKSPACE
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=ws + 8, ws_bytes=need)) == EALIGN
    # device parameters must be aligned; host activations need not be
    assert L.mamba_mixer_fwd_host(*host_args(B=2, Lq=1000, ws=ws, ws_bytes=need, A=BASE + 4)) == EALIGN
    args = host_args(B=2, Lq=1000, ws=ws, ws_bytes=need)
    args[0] += 2                                          # unaligned host xz: still accepted
    assert L.mamba_mixer_fwd_host(*args) == EDEVICE
    # a host output overlapping a host input
    args = host_args(B=2, Lq=1000, ws=ws, ws_bytes=need)
    args[11] = args[0]                                    # y over xz
    assert L.mamba_mixer_fwd_host(*args) == EALIAS
    assert L.mamba_mixer_fwd_host(*host_args(B=0, Lq=1000, ws=None, ws_bytes=0)) == OK


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mamba_mixer.h"

int main(void) {
    /* host-only entry points: no device is needed */
    if (mamba_mixer_abi_version() != MAMBA_MIXER_ABI_VERSION) return 1;
    size_t ws = mamba_mixer_workspace_size(1, 4096, 8192, 16, 4, MM_BF16);
    if (ws < (size_t)8 * 8192 * 17 * 4) return 2;
    if (strcmp(mamba_status_string(MM_OK), "ok") != 0) return 3;
    /* a rejected call: NULL required pointers, caught before any launch */
    mm_status st = mamba_mixer_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                   NULL, NULL, NULL, 1, 64, 64, 16, 4, MM_BF16, NULL, 0, NULL);
    if (st != MM_ERR_NULL) return 4;
    printf("%zu\n", ws);
    return 0;
}
"""


def test_plain_c_program_uses_the_abi(L, tmp_path):
    """The boundary is a C ABI: a C11 program (no C++, no torch) includes the
    header, links the library and calls its host-only entry points."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(mm.library_path())
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmamba_mixer", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == str(ws_bytes(1, 9, 8192))


def m3_decode_args(B=2, R=2, H=4, P=64, N=16, G=2, **over):
    """mamba_m3_state_update arguments on fake addresses, each buffer 2^32 apart."""
    names = ["x", "z", "dt", "trap", "dt_bias", "A", "theta", "Bm", "Cm", "Dskip", "state", "x_prev", "B_prev", "y"]
    addr = {n: BASE + (i << 32) for i, n in enumerate(names)}
    addr.update(over)
    return [addr[n] for n in names] + [B, R, H, P, N, G, None]


def test_m3_decode_validation(L):
    assert L.mamba_m3_state_update(*m3_decode_args()) == EDEVICE
    assert L.mamba_m3_state_update(*m3_decode_args(z=None, trap=None, dt_bias=None, Dskip=None, x_prev=None,
                                                   B_prev=None)) == EDEVICE
    assert L.mamba_m3_state_update(*m3_decode_args(P=32)) == EUNSUP
    assert L.mamba_m3_state_update(*m3_decode_args(N=32)) == EUNSUP
    assert L.mamba_m3_state_update(*m3_decode_args(R=3)) == EUNSUP
    assert L.mamba_m3_state_update(*m3_decode_args(H=3, G=1)) == EUNSUP
    assert L.mamba_m3_state_update(*m3_decode_args(H=6, G=4)) == ESHAPE
    assert L.mamba_m3_state_update(*m3_decode_args(B=-1)) == ESHAPE
    assert L.mamba_m3_state_update(*m3_decode_args(B=0)) == OK
    for name in ("x", "dt", "A", "theta", "Bm", "Cm", "state", "y"):
        assert L.mamba_m3_state_update(*m3_decode_args(**{name: None})) == ENULL, name
    assert L.mamba_m3_state_update(*m3_decode_args(x_prev=None)) == ENULL      # x_prev and B_prev together
    for name in ("x", "trap", "theta", "state", "B_prev", "y"):
        assert L.mamba_m3_state_update(*m3_decode_args(**{name: BASE + (1 << 40) + 8})) == EALIGN, name
    assert L.mamba_m3_state_update(*m3_decode_args(y=BASE)) == EALIAS                   # y over x
    assert L.mamba_m3_state_update(*m3_decode_args(state=BASE + (7 << 32))) == EALIAS   # state over B
    assert L.mamba_m3_state_update(*m3_decode_args(y=BASE + (10 << 32) + 64)) == EALIAS # y over state
