"""fp64 CPU oracle for the Mamba mixer core -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline and
reference legs use this package.  The product path (the CUDA library and its binding) never imports
it, and the two share no code.

The arithmetic lives in ``mixer_oracle.c`` (plain C, double precision, libm);
this module compiles it with gcc on first use and marshals numpy arrays to it.
Channels (or decode rows) are independent, so ``threads > 1`` only splits the
channel range across threads; each thread runs the same sequential loop.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "mixer_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(_BUILD_DIR, "libmixer_oracle.so")

CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math"]

_lock = threading.Lock()
_lib = None


def compile_source(src: str, out: str) -> str:
    """Compile one oracle C source into a shared library at ``out``."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, src, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, LIB_PATH)
    return LIB_PATH


def _declare(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int64
    lib.oracle_mixer_fwd.restype = ctypes.c_int
    lib.oracle_mixer_fwd.argtypes = [P] * 17 + [I] * 7
    lib.oracle_state_update.restype = ctypes.c_int
    lib.oracle_state_update.argtypes = [P] * 13 + [I] * 7
    lib.oracle_rmsnorm_rows.restype = ctypes.c_int
    lib.oracle_rmsnorm_rows.argtypes = [P, P, ctypes.c_double, P, I, I]
    lib.oracle_matmul_nt.restype = ctypes.c_int
    lib.oracle_matmul_nt.argtypes = [P, P, P, I, I, I, I, I]
    lib.oracle_ssd_fwd.restype = ctypes.c_int
    lib.oracle_ssd_fwd.argtypes = [P] * 11 + [I] * 8
    lib.oracle_m3_fwd.restype = ctypes.c_int
    lib.oracle_m3_fwd.argtypes = [P] * 15 + [I] * 9
    return lib


def load_library(path: str):
    return _declare(ctypes.CDLL(path))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        import torch

        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ranges(total: int, parts: int):
    parts = max(1, min(parts, total)) if total > 0 else 1
    bounds = [total * i // parts for i in range(parts + 1)]
    return [(bounds[i], bounds[i + 1]) for i in range(parts)]


def mixer_fwd(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, conv_state_in=None,
              threads: int = 1, traces: bool = False, library=None):
    """Run the oracle forward.  Arrays may be numpy or torch (any dtype; they are
    widened to float64).  Returns a dict of float64 arrays: y [B,L,D],
    h_last [B,D,N], conv_state_out [B,D,W-1] and, with ``traces``, u, delta
    and pre (the conv output before SiLU), each [B,L,D]."""
    L_ = library or lib()
    xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in = map(
        _f64, (xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in))
    Bsz, L, twoD = xz.shape
    D = twoD // 2
    N = A.shape[-1]
    W = conv_w.shape[-1]
    assert A.shape == (D, N) and conv_w.shape == (D, W)
    assert dt.shape == (Bsz, L, D) and Bm.shape == (Bsz, L, N) and Cm.shape == (Bsz, L, N)
    y = np.zeros((Bsz, L, D))
    h_last = np.zeros((Bsz, D, N))
    cs_out = np.zeros((Bsz, D, max(W - 1, 0)))
    tr = [np.zeros((Bsz, L, D)) for _ in range(3)] if traces else [None, None, None]

    def run(rng):
        rc = L_.oracle_mixer_fwd(_p(xz), _p(conv_w), _p(conv_b), _p(dt), _p(dt_bias), _p(A),
                                 _p(Bm), _p(Cm), _p(Dskip), _p(h0), _p(conv_state_in),
                                 _p(y), _p(h_last), _p(cs_out), _p(tr[0]), _p(tr[1]), _p(tr[2]),
                                 Bsz, L, D, N, W, rng[0], rng[1])
        if rc != 0:
            raise ValueError(f"oracle_mixer_fwd rejected its arguments (rc={rc})")

    parts = _ranges(D, threads)
    if len(parts) == 1:
        run(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(run, parts))
    out = {"y": y, "h_last": h_last, "conv_state_out": cs_out}
    if traces:
        out.update(u=tr[0], delta=tr[1], pre=tr[2])
    return out


def state_update(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state,
                 threads: int = 1, library=None):
    """Run the oracle decode step on copies of the carried state.  Returns a dict
    with the new ssm_state [NL,B,D,N], conv_state [NL,B,D,W-1] and y [NL,B,D]."""
    L_ = library or lib()
    x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm = map(
        _f64, (x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm))
    ssm = _f64(ssm_state).copy()
    cs = _f64(conv_state).copy() if conv_state is not None else None
    NL, Bsz, D = x.shape
    N = A.shape[-1]
    W = conv_w.shape[-1]
    y = np.zeros((NL, Bsz, D))
    rows = NL * Bsz * D

    def run(rng):
        rc = L_.oracle_state_update(_p(x), _p(z), _p(dt), _p(conv_w), _p(conv_b), _p(dt_bias),
                                    _p(Dskip), _p(A), _p(Bm), _p(Cm), _p(ssm), _p(cs), _p(y),
                                    NL, Bsz, D, N, W, rng[0], rng[1])
        if rc != 0:
            raise ValueError(f"oracle_state_update rejected its arguments (rc={rc})")

    parts = _ranges(rows, threads)
    if len(parts) == 1:
        run(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(run, parts))
    return {"ssm_state": ssm, "conv_state": cs, "y": y}


def rmsnorm_rows(x, w, eps: float, library=None):
    """RMSNorm over the last axis with one weight per entry of that axis:
    x * w / sqrt(mean(x^2) + eps), in float64 (oracle_rmsnorm_rows)."""
    L_ = library or lib()
    x = _f64(x)
    w = _f64(w)
    n = x.shape[-1]
    assert w.shape == (n,)
    out = np.zeros_like(x)
    rc = L_.oracle_rmsnorm_rows(_p(x), _p(w), float(eps), _p(out), x.size // n, n)
    if rc != 0:
        raise ValueError(f"oracle_rmsnorm_rows rejected its arguments (rc={rc})")
    return out


def mixer_fwd_normed(xz, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, conv_state_in=None,
                     b_norm_w=None, c_norm_w=None, norm_eps: float = 1e-6, threads: int = 1, library=None):
    """The forward with B_t and C_t each RMS-normalised over d_state first
    (a weight of None leaves that input as it is)."""
    Bn = rmsnorm_rows(Bm, b_norm_w, norm_eps, library) if b_norm_w is not None else Bm
    Cn = rmsnorm_rows(Cm, c_norm_w, norm_eps, library) if c_norm_w is not None else Cm
    return mixer_fwd(xz, conv_w, conv_b, dt, dt_bias, A, Bn, Cn, Dskip, h0, conv_state_in, threads=threads,
                     library=library)


def state_update_normed(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, Bm, Cm, ssm_state, conv_state,
                        b_norm_w=None, c_norm_w=None, norm_eps: float = 1e-6, threads: int = 1, library=None):
    """The decode step with each layer's B and C rows RMS-normalised over
    d_state first, with that layer's weights ([NL, N]; None = not normalised)."""
    def per_layer(M, w):
        if w is None:
            return M
        M = _f64(M)
        w = _f64(w)
        return np.stack([rmsnorm_rows(M[l], w[l], norm_eps, library) for l in range(M.shape[0])])

    return state_update(x, z, dt, conv_w, conv_b, dt_bias, Dskip, A, per_layer(Bm, b_norm_w),
                        per_layer(Cm, c_norm_w), ssm_state, conv_state, threads=threads, library=library)


def matmul_nt(A, Bw, threads: int = 1, library=None):
    """C = A @ Bw^T in float64 with Bw stored [N, K] (oracle_matmul_nt); A may
    have leading batch dimensions, which are flattened into rows."""
    L_ = library or lib()
    A = _f64(A)
    Bw = _f64(Bw)
    K = A.shape[-1]
    N = Bw.shape[0]
    assert Bw.shape == (N, K)
    M = int(np.prod(A.shape[:-1]))
    A2 = A.reshape(M, K)
    C = np.zeros((M, N))

    def run(rng):
        rc = L_.oracle_matmul_nt(_p(A2), _p(Bw), _p(C), M, N, K, rng[0], rng[1])
        if rc != 0:
            raise ValueError(f"oracle_matmul_nt rejected its arguments (rc={rc})")

    parts = _ranges(M, threads)
    if len(parts) == 1:
        run(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(run, parts))
    return C.reshape(A.shape[:-1] + (N,))


def _store(a, store):
    """An intermediate as a bf16 implementation stores it: rounded to nearest
    even (torch's cast), then widened back; store=None keeps it exact."""
    if store is None:
        return a
    if store != "bf16":
        raise ValueError(f"unknown storage dtype {store!r}")
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float64).numpy()


def projected_fwd(xz, conv_w, conv_b, W_x, W_dt, dt_bias, A, Dskip, h0=None, conv_state_in=None,
                  dt_norm_w=None, b_norm_w=None, c_norm_w=None, norm_eps: float = 1e-6, store=None,
                  threads: int = 1, library=None):
    """The mixer with its producers, in the order the method runs them:
        u      = SiLU(causal conv(x))                        [B, L, D]
        x_dbl  = u @ W_x^T, W_x [R + 2N, D]                  [B, L, R + 2N]
        dt_low, B, C = x_dbl[..., :R], [..., R:R+N], [..., R+N:]
        (each optionally RMS-normalised over its own width)
        dt     = dt_low @ W_dt^T, W_dt [D, R]                [B, L, D]
        y, h_last, conv_state_out = the selective scan on (x, z, dt, B, C)
    With store="bf16" the intermediates an implementation keeps in memory
    between these steps (u, dt_low, B, C, dt) are rounded to bf16 where they are
    stored, as the bf16 activations they are; the arithmetic stays fp64.
    Returns the scan's outputs plus the intermediates u, dt_low, Bm, Cm, dt."""
    L_ = library or lib()
    xz_ = _f64(xz)
    Bsz, Lq, twoD = xz_.shape
    D = twoD // 2
    N = _f64(A).shape[-1]
    W_x = _f64(W_x)
    R = W_x.shape[0] - 2 * N
    # u: the scan's own conv + SiLU output, taken from its trace (B, C and dt do
    # not enter u, so zeros stand in for them)
    zeros_bc = np.zeros((Bsz, Lq, N))
    tr = mixer_fwd(xz_, conv_w, conv_b, np.zeros((Bsz, Lq, D)), None, A, zeros_bc, zeros_bc, None, None,
                   conv_state_in, threads=threads, traces=True, library=L_)
    u = _store(tr["u"], store)
    x_dbl = matmul_nt(u, W_x, threads=threads, library=L_)
    dt_low, Bm, Cm = x_dbl[..., :R], x_dbl[..., R:R + N], x_dbl[..., R + N:]
    if dt_norm_w is not None:
        dt_low = rmsnorm_rows(dt_low, dt_norm_w, norm_eps, L_)
    if b_norm_w is not None:
        Bm = rmsnorm_rows(Bm, b_norm_w, norm_eps, L_)
    if c_norm_w is not None:
        Cm = rmsnorm_rows(Cm, c_norm_w, norm_eps, L_)
    dt_low, Bm, Cm = _store(dt_low, store), _store(Bm, store), _store(Cm, store)
    dt = _store(matmul_nt(dt_low, W_dt, threads=threads, library=L_), store)
    out = mixer_fwd(xz_, conv_w, conv_b, dt, dt_bias, A, Bm, Cm, Dskip, h0, conv_state_in, threads=threads,
                    library=L_)
    out.update(u=u, dt_low=dt_low, Bm=Bm, Cm=Cm, dt=dt)
    return out



def ssd_fwd(x, z, dt, dt_bias, A, Bm, Cm, Dskip, h0=None, headdim: int = 64, threads: int = 1, library=None):
    """Run the oracle of the Mamba-2 form (scalar-times-identity state matrix
    per head, oracle_ssd_fwd).  x, z [B,L,H*P] (z None: no gate), dt [B,L,H],
    dt_bias [H] or None, A [H], Bm, Cm [B,L,G,N], Dskip [H] or None, h0
    [B,H,P,N] or None, P = headdim.  Returns y [B,L,H*P] and h_last [B,H,P,N]
    as float64 arrays."""
    L_ = library or lib()
    x, z, dt, dt_bias, A, Bm, Cm, Dskip, h0 = map(_f64, (x, z, dt, dt_bias, A, Bm, Cm, Dskip, h0))
    Bsz, L, C = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[2], Bm.shape[3]
    assert C == H * P and dt.shape == (Bsz, L, H) and Bm.shape == (Bsz, L, G, N) and Cm.shape == Bm.shape
    y = np.zeros((Bsz, L, C))
    h_last = np.zeros((Bsz, H, P, N))

    def run(rng):
        rc = L_.oracle_ssd_fwd(_p(x), _p(z), _p(dt), _p(dt_bias), _p(A), _p(Bm), _p(Cm), _p(Dskip), _p(h0),
                               _p(y), _p(h_last), Bsz, L, H, P, N, G, rng[0], rng[1])
        if rc != 0:
            raise ValueError(f"oracle_ssd_fwd rejected its arguments (rc={rc})")

    parts = _ranges(C, threads)
    if len(parts) == 1:
        run(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(run, parts))
    return {"y": y, "h_last": h_last}


def m3_fwd(x, z, dt, trap, dt_bias, A, theta, Bm, Cm, Dskip, h0=None, x_prev=None, B_prev=None,
           headdim: int = 64, threads: int = 1, library=None):
    """Run the oracle of the Mamba-3 form (oracle_m3_fwd): x, z [B,L,R,H*P]
    (z None: no gate), dt and trap [B,L,H] (trap None: 1/2), dt_bias [H] or
    None, A [H], theta [H,N/2], Bm, Cm [B,L,R,G,N], Dskip [H] or None, h0
    [B,H,P,N] or None, x_prev [B,R,H*P] and B_prev [B,R,G,N] (the token before
    the call) or None, P = headdim.  Returns y [B,L,R,H*P] and h_last
    [B,H,P,N] as float64 arrays."""
    L_ = library or lib()
    x, z, dt, trap, dt_bias, A, theta, Bm, Cm, Dskip, h0, x_prev, B_prev = map(
        _f64, (x, z, dt, trap, dt_bias, A, theta, Bm, Cm, Dskip, h0, x_prev, B_prev))
    Bsz, L, R, C = x.shape
    H = A.shape[0]
    P = int(headdim)
    G, N = Bm.shape[3], Bm.shape[4]
    assert C == H * P and dt.shape == (Bsz, L, H) and Bm.shape == (Bsz, L, R, G, N) and Cm.shape == Bm.shape
    assert theta.shape == (H, N // 2)
    y = np.zeros((Bsz, L, R, C))
    h_last = np.zeros((Bsz, H, P, N))

    def run(rng):
        rc = L_.oracle_m3_fwd(_p(x), _p(z), _p(dt), _p(trap), _p(dt_bias), _p(A), _p(theta), _p(Bm), _p(Cm),
                              _p(Dskip), _p(h0), _p(x_prev), _p(B_prev), _p(y), _p(h_last),
                              Bsz, L, R, H, P, N, G, rng[0], rng[1])
        if rc != 0:
            raise ValueError(f"oracle_m3_fwd rejected its arguments (rc={rc})")

    parts = _ranges(C, threads)
    if len(parts) == 1:
        run(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(run, parts))
    return {"y": y, "h_last": h_last}
