"""Python binding of the B200 Mamba mixer core library (libmamba_mixer.so).

Argument marshalling only: tensors are checked (device, dtype, shape,
contiguity), output tensors are allocated with torch when not given, and the
data pointers plus the current CUDA stream go through ctypes to the C ABI of
``include/mamba_mixer.h``.  Every step of the computation runs in the
library's kernels; there is no fallback path.  If the compiled library is
missing, loading fails with an error that says how to build it.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "MM_F32", "MM_BF16", "MixerError", "lib", "library_path", "mixer_fwd", "mixer_fwd_noalloc", "mixer_fwd_host",
    "state_update", "workspace_size", "host_workspace_size", "status_string", "abi_version", "fault_status",
    "check_status", "proj_matmul", "proj_matmul_workspace_size", "mixer_fwd_projected",
    "projected_workspace_size", "ssd_fwd", "ssd_workspace_size", "ssd_state_update", "m3_fwd", "m3_state_update", "m3_workspace_size", "EXPORTED_SYMBOLS",
]

MM_F32 = 0
MM_BF16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libmamba_mixer.so"
_lib = None

EXPORTED_SYMBOLS = (
    "mamba_mixer_fwd",
    "mamba_mixer_fwd_noalloc",
    "mamba_mixer_fwd_host",
    "mamba_mixer_workspace_size",
    "mamba_mixer_host_workspace_size",
    "mamba_state_update",
    "mamba_status_string",
    "mamba_mixer_abi_version",
    "mamba_mixer_fault_status",
    "mamba_check_status",
    "mamba_mixer_fwd_normed",
    "mamba_state_update_normed",
    "mamba_proj_matmul",
    "mamba_proj_matmul_workspace_size",
    "mamba_mixer_fwd_projected",
    "mamba_mixer_projected_workspace_size",
    "mamba_mixer_projected_layout",
    "mamba_ssd_fwd",
    "mamba_ssd_workspace_size",
    "mamba_ssd_state_update",
    "mamba_m3_fwd",
    "mamba_m3_workspace_size",
    "mamba_m3_state_update",
)


class MixerError(RuntimeError):
    """A non-zero mm_status returned by the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (mm_status {status})")


def library_path() -> str:
    """The library this process loads: libmamba_mixer.so, or its checked build
    libmamba_mixer_checked.so when MAMBA_MIXER_CHECKED=1 is set before the
    first call (index checks in the forward and decode kernels; an access
    outside its buffer is skipped and reported as MM_ERR_BOUNDS)."""
    if os.environ.get("MAMBA_MIXER_CHECKED") == "1":
        return os.path.join(_HERE, "libmamba_mixer_checked.so")
    return os.path.join(_HERE, _LIB_NAME)


def _declare(L):
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    L.mamba_mixer_fwd.restype = ctypes.c_int
    L.mamba_mixer_fwd.argtypes = [P] * 14 + [I64] * 5 + [ctypes.c_int, P, ctypes.c_size_t, P]
    L.mamba_mixer_fwd_noalloc.restype = ctypes.c_int
    L.mamba_mixer_fwd_noalloc.argtypes = [P] * 14 + [I64] * 5 + [ctypes.c_int, P]
    L.mamba_mixer_fwd_host.restype = ctypes.c_int
    L.mamba_mixer_fwd_host.argtypes = [P] * 14 + [I64] * 5 + [ctypes.c_int, P, ctypes.c_size_t, P, P, P]
    L.mamba_mixer_workspace_size.restype = ctypes.c_size_t
    L.mamba_mixer_workspace_size.argtypes = [I64] * 5 + [ctypes.c_int]
    L.mamba_mixer_host_workspace_size.restype = ctypes.c_size_t
    L.mamba_mixer_host_workspace_size.argtypes = [I64] * 5 + [ctypes.c_int]
    L.mamba_state_update.restype = ctypes.c_int
    L.mamba_state_update.argtypes = [P] * 13 + [I64] * 5 + [ctypes.c_int, P]
    L.mamba_status_string.restype = ctypes.c_char_p
    L.mamba_status_string.argtypes = [ctypes.c_int]
    L.mamba_mixer_abi_version.restype = ctypes.c_int
    L.mamba_mixer_abi_version.argtypes = []
    L.mamba_mixer_fault_status.restype = ctypes.c_int
    L.mamba_mixer_fault_status.argtypes = [ctypes.c_int]
    L.mamba_check_status.restype = ctypes.c_int
    L.mamba_check_status.argtypes = [P, P]
    L.mamba_mixer_fwd_normed.restype = ctypes.c_int
    L.mamba_mixer_fwd_normed.argtypes = [P] * 14 + [I64] * 5 + [ctypes.c_int, P, P, ctypes.c_float, P,
                                                                 ctypes.c_size_t, P]
    L.mamba_state_update_normed.restype = ctypes.c_int
    L.mamba_state_update_normed.argtypes = [P] * 13 + [I64] * 5 + [ctypes.c_int, P, P, ctypes.c_float, P]
    L.mamba_proj_matmul.restype = ctypes.c_int
    L.mamba_proj_matmul.argtypes = [P, P, P, I64, I64, I64, ctypes.c_int, P, ctypes.c_size_t, P]
    L.mamba_proj_matmul_workspace_size.restype = ctypes.c_size_t
    L.mamba_proj_matmul_workspace_size.argtypes = [I64, I64, I64]
    L.mamba_mixer_fwd_projected.restype = ctypes.c_int
    L.mamba_mixer_fwd_projected.argtypes = [P] * 13 + [ctypes.c_float] + [P] * 3 + [I64] * 6 + [
        ctypes.c_int, P, ctypes.c_size_t, P]
    L.mamba_mixer_projected_workspace_size.restype = ctypes.c_size_t
    L.mamba_mixer_projected_workspace_size.argtypes = [I64] * 6 + [ctypes.c_int]
    L.mamba_mixer_projected_layout.restype = ctypes.c_int
    L.mamba_mixer_projected_layout.argtypes = [I64] * 6 + [P]
    L.mamba_ssd_fwd.restype = ctypes.c_int
    L.mamba_ssd_fwd.argtypes = [P] * 11 + [I64] * 6 + [P, ctypes.c_size_t, P]
    L.mamba_ssd_workspace_size.restype = ctypes.c_size_t
    L.mamba_ssd_workspace_size.argtypes = [I64] * 6
    L.mamba_ssd_state_update.restype = ctypes.c_int
    L.mamba_ssd_state_update.argtypes = [P] * 10 + [I64] * 5 + [P]
    L.mamba_m3_fwd.restype = ctypes.c_int
    L.mamba_m3_fwd.argtypes = [P] * 15 + [I64] * 7 + [P, ctypes.c_size_t, P]
    L.mamba_m3_workspace_size.restype = ctypes.c_size_t
    L.mamba_m3_workspace_size.argtypes = [I64] * 7
    L.mamba_m3_state_update.restype = ctypes.c_int
    L.mamba_m3_state_update.argtypes = [P] * 14 + [I64] * 6 + [P]
    return L


def lib():
    """The loaded C library (ctypes.CDLL).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build the CUDA library first "
                "(python -m mamba_selective_scan_core_b200.build, or __graft_entry__.build())")
        _lib = _declare(ctypes.CDLL(path))
    return _lib


def status_string(status: int) -> str:
    return lib().mamba_status_string(int(status)).decode()


def abi_version() -> int:
    return int(lib().mamba_mixer_abi_version())


def fault_status(reset: bool = False) -> int:
    """0 if no kernel gave up waiting for its bulk copies on the current
    device, else MM_ERR_TIMEOUT (11) -- or MM_ERR_BOUNDS (13) when a kernel of
    the checked build skipped an access outside its buffer; clears the word
    when reset is set."""
    return int(lib().mamba_mixer_fault_status(1 if reset else 0))


def check_status(workspace=None, stream=None) -> int:
    """Status of the last forward that ran on `workspace` (a CUDA uint8
    tensor given to mixer_fwd or mixer_fwd_host; None = the fixed scratch of
    mixer_fwd_noalloc): 0 if it completed, MM_ERR_TIMEOUT (11) if one of its
    kernels gave up a bounded wait, MM_ERR_BOUNDS (13) if the checked build
    skipped an access outside its buffer.  Waits for `stream` (default: current)."""
    import torch

    dev = workspace.device if workspace is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(lib().mamba_check_status(_ptr(workspace), _stream_handle(stream)))


def _act_code(dtype):
    import torch

    if dtype == torch.bfloat16:
        return MM_BF16
    if dtype == torch.float32:
        return MM_F32
    raise TypeError(f"activation dtype must be bfloat16 or float32, got {dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, dtype, shape, device):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_handle(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _keep_alive_on(tensors, streams):
    """Tell torch's caching allocator that device tensors this module
    allocated are used by work queued on `streams` (besides the stream current
    at allocation), so their memory is not handed out again before that work
    has finished."""
    for t in tensors:
        for s in streams:
            if s is not None:
                t.record_stream(s)


def workspace_size(batch, seqlen, d_inner, d_state=16, d_conv=4, act=MM_BF16) -> int:
    return int(lib().mamba_mixer_workspace_size(batch, seqlen, d_inner, d_state, d_conv, act))


def mixer_fwd(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, conv_state_in=None, *,
              y=None, h_last=None, conv_state_out=None, workspace=None, stream=None,
              b_norm_w=None, c_norm_w=None, norm_eps=1e-6):
    """Selective-scan forward.  Shapes: xz [B,L,2D], dt [B,L,D], Bm/Cm [B,L,N]
    (act dtype: bf16 or fp32); conv_w [D,W], conv_b/dt_bias/Dskip [D], A [D,N],
    h0 [B,D,N] (fp32); conv_state_in [B,D,W-1] (act).  conv_b, Dskip, h0 and
    conv_state_in may be None.  b_norm_w / c_norm_w ([N] fp32) switch on the
    fused RMSNorm of B / C (mamba_mixer_fwd_normed).  Returns (y [B,L,D],
    h_last [B,D,N], conv_state_out [B,D,W-1]), allocating any output not
    given."""
    import torch

    act = _act_code(xz.dtype)
    Bsz, L, twoD = xz.shape
    D = twoD // 2
    N = A.shape[-1]
    W = conv_w.shape[-1]
    dev = xz.device
    f32 = torch.float32
    made = []
    _check(xz, "xz", xz.dtype, (Bsz, L, 2 * D), dev)
    _check(conv_w, "conv_w", f32, (D, W), dev)
    _check(conv_b, "conv_b", f32, (D,), dev)
    _check(dt, "dt", xz.dtype, (Bsz, L, D), dev)
    _check(dt_bias, "dt_bias", f32, (D,), dev)
    _check(A, "A", f32, (D, N), dev)
    _check(Bm, "Bm", xz.dtype, (Bsz, L, N), dev)
    _check(Cm, "Cm", xz.dtype, (Bsz, L, N), dev)
    _check(Dskip, "Dskip", f32, (D,), dev)
    _check(h0, "h0", f32, (Bsz, D, N), dev)
    _check(conv_state_in, "conv_state_in", xz.dtype, (Bsz, D, W - 1), dev)
    _check(b_norm_w, "b_norm_w", f32, (N,), dev)
    _check(c_norm_w, "c_norm_w", f32, (N,), dev)
    normed = b_norm_w is not None or c_norm_w is not None
    if y is None:
        y = torch.empty((Bsz, L, D), dtype=xz.dtype, device=dev)
        made.append(y)
    if h_last is None:
        h_last = torch.empty((Bsz, D, N), dtype=f32, device=dev)
        made.append(h_last)
    if conv_state_out is None:
        conv_state_out = torch.empty((Bsz, D, W - 1), dtype=xz.dtype, device=dev)
        made.append(conv_state_out)
    _check(y, "y", xz.dtype, (Bsz, L, D), dev)
    _check(h_last, "h_last", f32, (Bsz, D, N), dev)
    _check(conv_state_out, "conv_state_out", xz.dtype, (Bsz, D, W - 1), dev)
    ws_bytes = workspace_size(Bsz, L, D, N, W, act)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        made.append(workspace)
    args = (_ptr(xz), _ptr(conv_w), _ptr(conv_b), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(Bm), _ptr(Cm),
            _ptr(Dskip), _ptr(h0), _ptr(conv_state_in), _ptr(y), _ptr(h_last), _ptr(conv_state_out),
            Bsz, L, D, N, W, act)
    tail = (_ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    with torch.cuda.device(dev):
        if normed:
            st = lib().mamba_mixer_fwd_normed(*args, _ptr(b_norm_w), _ptr(c_norm_w), float(norm_eps), *tail)
        else:
            st = lib().mamba_mixer_fwd(*args, *tail)
    if st != 0:
        raise MixerError(st, "mamba_mixer_fwd_normed" if normed else "mamba_mixer_fwd")
    _keep_alive_on(made, (stream,))
    return y, h_last, conv_state_out


def host_workspace_size(batch, seqlen, d_inner, d_state=16, d_conv=4, act=MM_BF16) -> int:
    return int(lib().mamba_mixer_host_workspace_size(batch, seqlen, d_inner, d_state, d_conv, act))


def _check_host(t, name, dtype, shape):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_side_streams = {}


def _copy_streams(dev):
    """Two side streams per device for the host path's copies (created once)."""
    import torch

    key = torch.device(dev).index
    if key not in _side_streams:
        with torch.cuda.device(dev):
            _side_streams[key] = (torch.cuda.Stream(), torch.cuda.Stream())
    return _side_streams[key]


def mixer_fwd_host(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, conv_state_in=None, *,
                   y=None, h_last=None, conv_state_out=None, workspace=None, stream=None):
    """mixer_fwd on activations in host memory (mamba_mixer_fwd_host): xz, dt,
    Bm, Cm, h0, conv_state_in and the outputs are CPU tensors (page-locked for
    the copies to overlap the compute; outputs are allocated pinned when not
    given); conv_w, conv_b, dt_bias, A, Dskip are CUDA tensors on the device
    that runs it.  Copies go on two side streams, the forward on `stream`
    (default: the current stream), which waits for the copies back: the
    outputs are valid once `stream` is synchronised."""
    import torch

    act = _act_code(xz.dtype)
    Bsz, L, twoD = xz.shape
    D = twoD // 2
    N = A.shape[-1]
    W = conv_w.shape[-1]
    dev = conv_w.device
    f32 = torch.float32
    for t, name, dtype, shape in ((xz, "xz", xz.dtype, (Bsz, L, 2 * D)), (dt, "dt", xz.dtype, (Bsz, L, D)),
                                  (Bm, "Bm", xz.dtype, (Bsz, L, N)), (Cm, "Cm", xz.dtype, (Bsz, L, N)),
                                  (h0, "h0", f32, (Bsz, D, N)),
                                  (conv_state_in, "conv_state_in", xz.dtype, (Bsz, D, W - 1))):
        _check_host(t, name, dtype, shape)
    _check(conv_w, "conv_w", f32, (D, W), dev)
    _check(conv_b, "conv_b", f32, (D,), dev)
    _check(dt_bias, "dt_bias", f32, (D,), dev)
    _check(A, "A", f32, (D, N), dev)
    _check(Dskip, "Dskip", f32, (D,), dev)
    if y is None:
        y = torch.empty((Bsz, L, D), dtype=xz.dtype).pin_memory()
    if h_last is None:
        h_last = torch.empty((Bsz, D, N), dtype=f32).pin_memory()
    if conv_state_out is None:
        conv_state_out = torch.empty((Bsz, D, W - 1), dtype=xz.dtype).pin_memory()
    _check_host(y, "y", xz.dtype, (Bsz, L, D))
    _check_host(h_last, "h_last", f32, (Bsz, D, N))
    _check_host(conv_state_out, "conv_state_out", xz.dtype, (Bsz, D, W - 1))
    ws_bytes = host_workspace_size(Bsz, L, D, N, W, act)
    made = []
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        made.append(workspace)
    s_in, s_out = _copy_streams(dev)
    with torch.cuda.device(dev):
        st = lib().mamba_mixer_fwd_host(
            _ptr(xz), _ptr(conv_w), _ptr(conv_b), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(Bm), _ptr(Cm),
            _ptr(Dskip), _ptr(h0), _ptr(conv_state_in), _ptr(y), _ptr(h_last), _ptr(conv_state_out),
            Bsz, L, D, N, W, act, _ptr(workspace), ws_bytes, _stream_handle(stream),
            ctypes.c_void_p(s_in.cuda_stream), ctypes.c_void_p(s_out.cuda_stream))
    if st != 0:
        raise MixerError(st, "mamba_mixer_fwd_host")
    _keep_alive_on(made, (stream, s_in, s_out))
    return y, h_last, conv_state_out


def mixer_fwd_noalloc(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, conv_state_in=None, *,
                      y, h_last, conv_state_out, stream=None):
    """mixer_fwd through the entry point that takes no workspace and allocates
    nothing (its scratch is a fixed array inside the library).  The caller
    passes the output tensors; calls that overlap on the GPU race on the
    shared scratch, so serialise them."""
    import torch

    act = _act_code(xz.dtype)
    Bsz, L, twoD = xz.shape
    D = twoD // 2
    N = A.shape[-1]
    W = conv_w.shape[-1]
    dev = xz.device
    f32 = torch.float32
    for t, name, dtype, shape in (
            (xz, "xz", xz.dtype, (Bsz, L, 2 * D)), (conv_w, "conv_w", f32, (D, W)), (conv_b, "conv_b", f32, (D,)),
            (dt, "dt", xz.dtype, (Bsz, L, D)), (dt_bias, "dt_bias", f32, (D,)), (A, "A", f32, (D, N)),
            (Bm, "Bm", xz.dtype, (Bsz, L, N)), (Cm, "Cm", xz.dtype, (Bsz, L, N)), (Dskip, "Dskip", f32, (D,)),
            (h0, "h0", f32, (Bsz, D, N)), (conv_state_in, "conv_state_in", xz.dtype, (Bsz, D, W - 1)),
            (y, "y", xz.dtype, (Bsz, L, D)), (h_last, "h_last", f32, (Bsz, D, N)),
            (conv_state_out, "conv_state_out", xz.dtype, (Bsz, D, W - 1))):
        _check(t, name, dtype, shape, dev)
    with torch.cuda.device(dev):
        st = lib().mamba_mixer_fwd_noalloc(
            _ptr(xz), _ptr(conv_w), _ptr(conv_b), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(Bm), _ptr(Cm),
            _ptr(Dskip), _ptr(h0), _ptr(conv_state_in), _ptr(y), _ptr(h_last), _ptr(conv_state_out),
            Bsz, L, D, N, W, act, _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_mixer_fwd_noalloc")
    return y, h_last, conv_state_out


def state_update(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state, *,
                 y=None, stream=None, b_norm_w=None, c_norm_w=None, norm_eps=1e-6):
    """One-token decode step for NL stacked layers, in place on ssm_state
    [NL,B,D,N] (fp32) and conv_state [NL,B,D,W-1] (act).  x/z/dt [NL,B,D] and
    Bm/Cm [NL,B,N] in the act dtype; conv_w [NL,D,W], conv_b/dt_bias/Dskip
    [NL,D], A [NL,D,N] in fp32 (conv_b, Dskip may be None).  b_norm_w /
    c_norm_w ([NL,N] fp32) switch on the fused RMSNorm of B / C
    (mamba_state_update_normed).  Returns y [NL,B,D]."""
    import torch

    act = _act_code(x.dtype)
    NL, Bsz, D = x.shape
    N = A.shape[-1]
    W = conv_w.shape[-1]
    dev = x.device
    f32 = torch.float32
    for t, name in ((x, "x"), (z, "z"), (dt, "dt")):
        _check(t, name, x.dtype, (NL, Bsz, D), dev)
    _check(conv_w, "conv_w", f32, (NL, D, W), dev)
    for t, name in ((conv_b, "conv_b"), (dt_bias, "dt_bias"), (Dskip, "Dskip")):
        _check(t, name, f32, (NL, D), dev)
    _check(A, "A", f32, (NL, D, N), dev)
    _check(Bm, "Bm", x.dtype, (NL, Bsz, N), dev)
    _check(Cm, "Cm", x.dtype, (NL, Bsz, N), dev)
    _check(ssm_state, "ssm_state", f32, (NL, Bsz, D, N), dev)
    _check(conv_state, "conv_state", x.dtype, (NL, Bsz, D, W - 1), dev)
    _check(b_norm_w, "b_norm_w", f32, (NL, N), dev)
    _check(c_norm_w, "c_norm_w", f32, (NL, N), dev)
    normed = b_norm_w is not None or c_norm_w is not None
    made = []
    if y is None:
        y = torch.empty((NL, Bsz, D), dtype=x.dtype, device=dev)
        made.append(y)
    _check(y, "y", x.dtype, (NL, Bsz, D), dev)
    args = (_ptr(x), _ptr(z), _ptr(dt), _ptr(conv_w), _ptr(conv_b), _ptr(dt_bias), _ptr(Dskip), _ptr(A),
            _ptr(Bm), _ptr(Cm), _ptr(ssm_state), _ptr(conv_state), _ptr(y), NL, Bsz, D, N, W, act)
    with torch.cuda.device(dev):
        if normed:
            st = lib().mamba_state_update_normed(*args, _ptr(b_norm_w), _ptr(c_norm_w), float(norm_eps),
                                                 _stream_handle(stream))
        else:
            st = lib().mamba_state_update(*args, _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_state_update_normed" if normed else "mamba_state_update")
    _keep_alive_on(made, (stream,))
    return y


def proj_matmul_workspace_size(M, N, K) -> int:
    return int(lib().mamba_proj_matmul_workspace_size(M, N, K))


def proj_matmul(A, W, *, out=None, out_dtype=None, workspace=None, stream=None):
    """out = A @ W^T on the tensor cores (mamba_proj_matmul): A [M, K] and W
    [N, K] bf16 CUDA tensors, out [M, N] fp32 (default) or bf16."""
    import torch

    M, K = A.shape
    N = W.shape[0]
    dev = A.device
    _check(A, "A", torch.bfloat16, (M, K), dev)
    _check(W, "W", torch.bfloat16, (N, K), dev)
    dtype = out_dtype or (out.dtype if out is not None else torch.float32)
    if out is None:
        out = torch.empty((M, N), dtype=dtype, device=dev)
    _check(out, "out", dtype, (M, N), dev)
    code = MM_BF16 if dtype == torch.bfloat16 else MM_F32
    ws_bytes = proj_matmul_workspace_size(M, N, K)
    made = []
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        made.append(workspace)
    with torch.cuda.device(dev):
        st = lib().mamba_proj_matmul(_ptr(A), _ptr(W), _ptr(out), M, N, K, code, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_proj_matmul")
    _keep_alive_on(made, (stream,))
    return out


def projected_workspace_size(batch, seqlen, d_inner, dt_rank, d_state=16, d_conv=4, act=MM_BF16) -> int:
    return int(lib().mamba_mixer_projected_workspace_size(batch, seqlen, d_inner, d_state, dt_rank, d_conv, act))


def projected_intermediates(workspace, batch, seqlen, d_inner, dt_rank, d_state=16, d_conv=4):
    """Views of the intermediates a mixer_fwd_projected call left in its
    workspace (u, dt_low, Bm, Cm, dt; bf16), by mamba_mixer_projected_layout."""
    import torch

    offs = (ctypes.c_size_t * 5)()
    st = lib().mamba_mixer_projected_layout(batch, seqlen, d_inner, d_state, dt_rank, d_conv, offs)
    if st != 0:
        raise MixerError(st, "mamba_mixer_projected_layout")
    shapes = ((batch, seqlen, d_inner), (batch, seqlen, dt_rank), (batch, seqlen, d_state), (batch, seqlen, d_state),
              (batch, seqlen, d_inner))
    out = []
    for off, shp in zip(offs, shapes):
        n = 1
        for v in shp:
            n *= v
        out.append(workspace[off:off + 2 * n].view(torch.bfloat16).view(shp))
    return dict(zip(("u", "dt_low", "Bm", "Cm", "dt"), out))


def mixer_fwd_projected(xz, conv_w, conv_b, W_x, W_dt, dt_bias, A, Dskip, h0=None, conv_state_in=None, *,
                        dt_norm_w=None, b_norm_w=None, c_norm_w=None, norm_eps=1e-6, y=None, h_last=None,
                        conv_state_out=None, workspace=None, stream=None):
    """The mixer with its producers (mamba_mixer_fwd_projected): u = SiLU(conv
    x), x_proj (W_x [R + 2N, D] bf16) split into dt_low | B | C with optional
    RMSNorms (dt_norm_w [R], b_norm_w / c_norm_w [N] fp32), dt_proj (W_dt
    [D, R] bf16), then the selective scan.  bf16 activations only.  Returns
    (y, h_last, conv_state_out)."""
    import torch

    Bsz, L, twoD = xz.shape
    D = twoD // 2
    N = A.shape[-1]
    W = conv_w.shape[-1]
    R = W_dt.shape[-1]
    dev = xz.device
    f32, bf = torch.float32, torch.bfloat16
    _check(xz, "xz", bf, (Bsz, L, 2 * D), dev)
    _check(conv_w, "conv_w", f32, (D, W), dev)
    _check(conv_b, "conv_b", f32, (D,), dev)
    _check(W_x, "W_x", bf, (R + 2 * N, D), dev)
    _check(W_dt, "W_dt", bf, (D, R), dev)
    _check(dt_bias, "dt_bias", f32, (D,), dev)
    _check(A, "A", f32, (D, N), dev)
    _check(Dskip, "Dskip", f32, (D,), dev)
    _check(h0, "h0", f32, (Bsz, D, N), dev)
    _check(conv_state_in, "conv_state_in", bf, (Bsz, D, W - 1), dev)
    _check(dt_norm_w, "dt_norm_w", f32, (R,), dev)
    _check(b_norm_w, "b_norm_w", f32, (N,), dev)
    _check(c_norm_w, "c_norm_w", f32, (N,), dev)
    made = []
    if y is None:
        y = torch.empty((Bsz, L, D), dtype=bf, device=dev)
        made.append(y)
    if h_last is None:
        h_last = torch.empty((Bsz, D, N), dtype=f32, device=dev)
        made.append(h_last)
    if conv_state_out is None:
        conv_state_out = torch.empty((Bsz, D, W - 1), dtype=bf, device=dev)
        made.append(conv_state_out)
    ws_bytes = projected_workspace_size(Bsz, L, D, R, N, W)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        made.append(workspace)
    with torch.cuda.device(dev):
        st = lib().mamba_mixer_fwd_projected(
            _ptr(xz), _ptr(conv_w), _ptr(conv_b), _ptr(W_x), _ptr(W_dt), _ptr(dt_bias), _ptr(A), _ptr(Dskip),
            _ptr(h0), _ptr(conv_state_in), _ptr(dt_norm_w), _ptr(b_norm_w), _ptr(c_norm_w), float(norm_eps),
            _ptr(y), _ptr(h_last), _ptr(conv_state_out), Bsz, L, D, N, R, W, MM_BF16, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_mixer_fwd_projected")
    _keep_alive_on(made, (stream,))
    return y, h_last, conv_state_out



def ssd_workspace_size(batch, seqlen, heads, headdim=64, d_state=128, groups=1) -> int:
    return int(lib().mamba_ssd_workspace_size(batch, seqlen, heads, headdim, d_state, groups))


def ssd_fwd(x, z, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, *, headdim=64, y=None, h_last=None, workspace=None,
            stream=None):
    """The Mamba-2 form of the scan (mamba_ssd_fwd): x, z [B,L,H*P] bf16 (z may
    be None: no gate), dt [B,L,H] bf16, dt_bias/A/Dskip [H] fp32 (dt_bias and
    Dskip may be None), Bm/Cm [B,L,G,N] bf16, h0 [B,H,P,N] fp32 or None, P =
    headdim.  Returns (y [B,L,H*P] bf16, h_last [B,H,P,N] fp32), allocating any
    output not given."""
    import torch

    bf, f32 = torch.bfloat16, torch.float32
    Bsz, L, HP = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[2], Bm.shape[3]
    if HP != H * P:
        raise ValueError(f"x has {HP} channels, expected heads x headdim = {H * P}")
    dev = x.device
    made = []
    _check(x, "x", bf, (Bsz, L, H * P), dev)
    _check(z, "z", bf, (Bsz, L, H * P), dev)
    _check(dt, "dt", bf, (Bsz, L, H), dev)
    _check(dt_bias, "dt_bias", f32, (H,), dev)
    _check(A, "A", f32, (H,), dev)
    _check(Bm, "Bm", bf, (Bsz, L, G, N), dev)
    _check(Cm, "Cm", bf, (Bsz, L, G, N), dev)
    _check(Dskip, "Dskip", f32, (H,), dev)
    _check(h0, "h0", f32, (Bsz, H, P, N), dev)
    if y is None:
        y = torch.empty((Bsz, L, H * P), dtype=bf, device=dev)
        made.append(y)
    if h_last is None:
        h_last = torch.empty((Bsz, H, P, N), dtype=f32, device=dev)
        made.append(h_last)
    _check(y, "y", bf, (Bsz, L, H * P), dev)
    _check(h_last, "h_last", f32, (Bsz, H, P, N), dev)
    ws_bytes = ssd_workspace_size(Bsz, L, H, P, N, G)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        made.append(workspace)
    with torch.cuda.device(dev):
        st = lib().mamba_ssd_fwd(_ptr(x), _ptr(z), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(Bm), _ptr(Cm),
                                 _ptr(Dskip), _ptr(h0), _ptr(y), _ptr(h_last), Bsz, L, H, P, N, G,
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_ssd_fwd")
    _keep_alive_on(made, (stream,))
    return y, h_last


def ssd_state_update(x, z, dt, dt_bias, A, Bm, Cm, Dskip, state, *, headdim=64, y=None, stream=None):
    """One token of the Mamba-2 form (mamba_ssd_state_update), in place on
    state [B,H,P,N] fp32: x, z [B,H*P] bf16 (z may be None: no gate), dt [B,H]
    bf16, dt_bias/A/Dskip [H] fp32 (dt_bias and Dskip may be None), Bm/Cm
    [B,G,N] bf16, P = headdim.  Returns y [B,H*P] bf16, allocated if not given."""
    import torch

    bf, f32 = torch.bfloat16, torch.float32
    Bsz, HP = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[1], Bm.shape[2]
    if HP != H * P:
        raise ValueError(f"x has {HP} channels, expected heads x headdim = {H * P}")
    dev = x.device
    made = []
    _check(x, "x", bf, (Bsz, H * P), dev)
    _check(z, "z", bf, (Bsz, H * P), dev)
    _check(dt, "dt", bf, (Bsz, H), dev)
    _check(dt_bias, "dt_bias", f32, (H,), dev)
    _check(A, "A", f32, (H,), dev)
    _check(Bm, "Bm", bf, (Bsz, G, N), dev)
    _check(Cm, "Cm", bf, (Bsz, G, N), dev)
    _check(Dskip, "Dskip", f32, (H,), dev)
    _check(state, "state", f32, (Bsz, H, P, N), dev)
    if y is None:
        y = torch.empty((Bsz, H * P), dtype=bf, device=dev)
        made.append(y)
    _check(y, "y", bf, (Bsz, H * P), dev)
    with torch.cuda.device(dev):
        st = lib().mamba_ssd_state_update(_ptr(x), _ptr(z), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(Bm), _ptr(Cm),
                                          _ptr(Dskip), _ptr(state), _ptr(y), Bsz, H, P, N, G,
                                          _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_ssd_state_update")
    _keep_alive_on(made, (stream,))
    return y


def m3_workspace_size(batch, seqlen, heads, rank=1, headdim=64, d_state=16, groups=1) -> int:
    return int(lib().mamba_m3_workspace_size(batch, seqlen, rank, heads, headdim, d_state, groups))


def m3_fwd(x, z, dt, trap, dt_bias, A, theta, Bm, Cm, Dskip, h0=None, x_prev=None, B_prev=None, *,
           headdim=64, y=None, h_last=None, workspace=None, stream=None):
    """The Mamba-3 form of the scan (mamba_m3_fwd): x, z [B,L,R,H*P] bf16
    (z may be None: no gate), dt and trap [B,L,H] bf16 (trap None: 1/2),
    dt_bias/A/Dskip [H] fp32 (dt_bias and Dskip may be None), theta [H,N/2]
    fp32, Bm/Cm [B,L,R,G,N] bf16, h0 [B,H,P,N] fp32 or None, x_prev [B,R,H*P]
    and B_prev [B,R,G,N] bf16 or None, P = headdim.  Returns (y [B,L,R,H*P]
    bf16, h_last [B,H,P,N] fp32), allocating any output not given."""
    import torch

    bf, f32 = torch.bfloat16, torch.float32
    Bsz, L, R, HP = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[3], Bm.shape[4]
    if HP != H * P:
        raise ValueError(f"x has {HP} channels, expected heads x headdim = {H * P}")
    dev = x.device
    made = []
    _check(x, "x", bf, (Bsz, L, R, H * P), dev)
    _check(z, "z", bf, (Bsz, L, R, H * P), dev)
    _check(dt, "dt", bf, (Bsz, L, H), dev)
    _check(trap, "trap", bf, (Bsz, L, H), dev)
    _check(dt_bias, "dt_bias", f32, (H,), dev)
    _check(A, "A", f32, (H,), dev)
    _check(theta, "theta", f32, (H, N // 2), dev)
    _check(Bm, "Bm", bf, (Bsz, L, R, G, N), dev)
    _check(Cm, "Cm", bf, (Bsz, L, R, G, N), dev)
    _check(Dskip, "Dskip", f32, (H,), dev)
    _check(h0, "h0", f32, (Bsz, H, P, N), dev)
    _check(x_prev, "x_prev", bf, (Bsz, R, H * P), dev)
    _check(B_prev, "B_prev", bf, (Bsz, R, G, N), dev)
    if y is None:
        y = torch.empty((Bsz, L, R, H * P), dtype=bf, device=dev)
        made.append(y)
    if h_last is None:
        h_last = torch.empty((Bsz, H, P, N), dtype=f32, device=dev)
        made.append(h_last)
    _check(y, "y", bf, (Bsz, L, R, H * P), dev)
    _check(h_last, "h_last", f32, (Bsz, H, P, N), dev)
    ws_bytes = m3_workspace_size(Bsz, L, H, R, P, N, G)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        made.append(workspace)
    with torch.cuda.device(dev):
        st = lib().mamba_m3_fwd(_ptr(x), _ptr(z), _ptr(dt), _ptr(trap), _ptr(dt_bias), _ptr(A), _ptr(theta),
                                _ptr(Bm), _ptr(Cm), _ptr(Dskip), _ptr(h0), _ptr(x_prev), _ptr(B_prev), _ptr(y),
                                _ptr(h_last), Bsz, L, R, H, P, N, G, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_m3_fwd")
    _keep_alive_on(made, (stream,))
    return y, h_last


def m3_state_update(x, z, dt, trap, dt_bias, A, theta, Bm, Cm, Dskip, state, x_prev=None, B_prev=None, *,
                    headdim=64, y=None, stream=None):
    """One token of the Mamba-3 form (mamba_m3_state_update), in place on
    state [B,H,P,N] fp32: x, z [B,R,H*P] bf16 (z may be None: no gate), dt and
    trap [B,H] bf16 (trap None: 1/2), dt_bias/A/Dskip [H] fp32 (dt_bias and
    Dskip may be None), theta [H,N/2] fp32, Bm/Cm [B,R,G,N] bf16, x_prev
    [B,R,H*P] and B_prev [B,R,G,N] bf16 (the previous token's) or None, P =
    headdim.  Returns y [B,R,H*P] bf16, allocated if not given."""
    import torch

    bf, f32 = torch.bfloat16, torch.float32
    Bsz, R, HP = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[2], Bm.shape[3]
    if HP != H * P:
        raise ValueError(f"x has {HP} channels, expected heads x headdim = {H * P}")
    dev = x.device
    made = []
    _check(x, "x", bf, (Bsz, R, H * P), dev)
    _check(z, "z", bf, (Bsz, R, H * P), dev)
    _check(dt, "dt", bf, (Bsz, H), dev)
    _check(trap, "trap", bf, (Bsz, H), dev)
    _check(dt_bias, "dt_bias", f32, (H,), dev)
    _check(A, "A", f32, (H,), dev)
    _check(theta, "theta", f32, (H, N // 2), dev)
    _check(Bm, "Bm", bf, (Bsz, R, G, N), dev)
    _check(Cm, "Cm", bf, (Bsz, R, G, N), dev)
    _check(Dskip, "Dskip", f32, (H,), dev)
    _check(state, "state", f32, (Bsz, H, P, N), dev)
    _check(x_prev, "x_prev", bf, (Bsz, R, H * P), dev)
    _check(B_prev, "B_prev", bf, (Bsz, R, G, N), dev)
    if y is None:
        y = torch.empty((Bsz, R, H * P), dtype=bf, device=dev)
        made.append(y)
    _check(y, "y", bf, (Bsz, R, H * P), dev)
    with torch.cuda.device(dev):
        st = lib().mamba_m3_state_update(_ptr(x), _ptr(z), _ptr(dt), _ptr(trap), _ptr(dt_bias), _ptr(A),
                                         _ptr(theta), _ptr(Bm), _ptr(Cm), _ptr(Dskip), _ptr(state), _ptr(x_prev),
                                         _ptr(B_prev), _ptr(y), Bsz, R, H, P, N, G, _stream_handle(stream))
    if st != 0:
        raise MixerError(st, "mamba_m3_state_update")
    _keep_alive_on(made, (stream,))
    return y

