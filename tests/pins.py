"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself (closed forms, library routines, brute force, invariants).

Every pin takes the oracle's ctypes library as an argument so the same pins
can be run against deliberately broken copies of the oracle (see
test_oracle_mutants.py): a plausible mistake anywhere in the oracle must make
at least one pin fail.

Where the passages come from:
  * Jamba hybrid SSM-Transformer lesson, section "SSM in one page": the
    recurrence h_t = A h_{t-1} + B x_t, y_t = C h_t; constant memory and O(1)
    per token (only h_{t-1} and x_t are needed); S4's structured A evaluated as
    a long convolution; Mamba makes A, B, C data-dependent.
  * the mixer-core problem statement: conv width 4 + SiLU, Delta = softplus(dt +
    dt_bias), dA = exp(Delta A), h_t = dA h_{t-1} + Delta B_t x_t, y_t = C_t h_t +
    D x_t gated by SiLU(z), and the one-token decode step.
"""

from __future__ import annotations

import numpy as np
import scipy.signal
import scipy.special

import oracle

W = 4


def lib_silu(v):
    """SiLU through scipy's logistic function (library routine)."""
    return v * scipy.special.expit(v)


def lib_softplus(v):
    """softplus through numpy's logaddexp (library routine)."""
    return np.logaddexp(0.0, v)


def _rand_case(rng, B, L, D, N, *, h0=True, cs=True, conv_b=True, dskip=True):
    xz = rng.standard_normal((B, L, 2 * D))
    dt = 0.3 * rng.standard_normal((B, L, D))
    conv_w = rng.uniform(-0.6, 0.6, (D, W))
    cb = 0.2 * rng.standard_normal(D) if conv_b else None
    dt_bias = rng.uniform(-4.0, 0.5, D)
    A = -np.exp(rng.uniform(np.log(0.3), np.log(5.0), (D, N)))
    Bm = rng.standard_normal((B, L, N))
    Cm = rng.standard_normal((B, L, N))
    Dsk = rng.normal(1.0, 0.3, D) if dskip else None
    h0 = 0.5 * rng.standard_normal((B, D, N)) if h0 else None
    csi = rng.standard_normal((B, D, W - 1)) if cs else None
    return dict(xz=xz, conv_w=conv_w, conv_b=cb, dt=dt, dt_bias=dt_bias, A=A, Bm=Bm, Cm=Cm,
                Dskip=Dsk, h0=h0, conv_state_in=csi)


def _fwd(lib, case, **kw):
    return oracle.mixer_fwd(case["xz"], case["conv_w"], case["conv_b"], case["dt"], case["dt_bias"],
                            case["A"], case["Bm"], case["Cm"], case["Dskip"], case["h0"],
                            case["conv_state_in"], library=lib, **kw)


def _lib_conv(case):
    """Pre-activation conv through numpy.convolve with the reversed kernel:
    pre_t = conv_b + sum_k w[k] * xpad[t + k], xpad = (left context, x)."""
    xz = case["xz"]
    B, L, twoD = xz.shape
    D = twoD // 2
    pre = np.zeros((B, L, D))
    for b in range(B):
        for d in range(D):
            left = case["conv_state_in"][b, d] if case["conv_state_in"] is not None else np.zeros(W - 1)
            xp = np.concatenate([left, xz[b, :, d]])
            pre[b, :, d] = np.convolve(xp, case["conv_w"][d][::-1], mode="valid")
            if case["conv_b"] is not None:
                pre[b, :, d] += case["conv_b"][d]
    return pre


def _lib_u_delta(case):
    pre = _lib_conv(case)
    u = lib_silu(pre)
    bias = case["dt_bias"] if case["dt_bias"] is not None else 0.0
    delta = lib_softplus(case["dt"] + bias)
    return pre, u, delta


def _gate_z(case):
    D = case["xz"].shape[2] // 2
    return lib_silu(case["xz"][:, :, D:])


# --------------------------------------------------------------------------- P1
def pin_lti_closed_form(lib):
    """Constant Delta and time-invariant B, C: the recurrence is an LTI system,
    so y equals the long convolution of u with K_k = sum_n C_n a_n^k Delta B_n,
    plus the free response of h0 (S4 evaluated as a long convolution)."""
    rng = np.random.default_rng(101)
    B, L, D, N = 2, 48, 3, 6
    case = _rand_case(rng, B, L, D, N)
    case["dt"] = np.zeros((B, L, D))                         # Delta constant per channel
    bvec = rng.standard_normal((B, N))
    cvec = rng.standard_normal((B, N))
    case["Bm"] = np.repeat(bvec[:, None, :], L, axis=1)
    case["Cm"] = np.repeat(cvec[:, None, :], L, axis=1)
    got = _fwd(lib, case)

    _, u, _ = _lib_u_delta(case)
    g = _gate_z(case)
    for b in range(B):
        for d in range(D):
            dlt = lib_softplus(case["dt_bias"][d])
            a = np.exp(dlt * case["A"][d])                     # [N]
            k = np.arange(L)
            K = (cvec[b][None, :] * a[None, :] ** k[:, None] * dlt * bvec[b][None, :]).sum(1)
            free = (cvec[b][None, :] * a[None, :] ** (k[:, None] + 1) * case["h0"][b, d][None, :]).sum(1)
            ssm = np.convolve(u[b, :, d], K)[:L] + free
            y = (ssm + case["Dskip"][d] * u[b, :, d]) * g[b, :, d]
            np.testing.assert_allclose(got["y"][b, :, d], y, rtol=1e-10, atol=1e-12)
            hl = np.array([sum(a[n] ** j * dlt * bvec[b, n] * u[b, L - 1 - j, d] for j in range(L))
                           + a[n] ** L * case["h0"][b, d, n] for n in range(N)])
            np.testing.assert_allclose(got["h_last"][b, d], hl, rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------- P2
def pin_brute_force_selective(lib):
    """Selective case on tiny inputs against the materialised sum
    y_t = sum_{s<=t} C_t (prod_{r=s+1..t} dA_r) Delta_s B_s u_s
          + C_t (prod_{r=0..t} dA_r) h0 + D u_t, gated by SiLU(z_t)."""
    rng = np.random.default_rng(202)
    B, L, D, N = 2, 14, 3, 5
    case = _rand_case(rng, B, L, D, N)
    got = _fwd(lib, case)
    _, u, delta = _lib_u_delta(case)
    g = _gate_z(case)
    for b in range(B):
        for d in range(D):
            dA = np.exp(delta[b, :, d][:, None] * case["A"][d][None, :])   # [L, N]
            hs = np.zeros((L, N))
            for t in range(L):
                acc = np.prod(dA[0:t + 1], axis=0) * case["h0"][b, d]
                for s in range(t + 1):
                    acc = acc + np.prod(dA[s + 1:t + 1], axis=0) * delta[b, s, d] * case["Bm"][b, s] * u[b, s, d]
                hs[t] = acc
            y = ((case["Cm"][b] * hs).sum(1) + case["Dskip"][d] * u[b, :, d]) * g[b, :, d]
            np.testing.assert_allclose(got["y"][b, :, d], y, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(got["h_last"][b, d], hs[-1], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(got["conv_state_out"][b, d], case["xz"][b, L - (W - 1):, d], rtol=0, atol=0)


# --------------------------------------------------------------------------- P3
def pin_zero_input(lib):
    """x = 0, conv_b = 0, h0 = 0, zero conv context => y = 0 and h_last = 0."""
    rng = np.random.default_rng(303)
    B, L, D, N = 2, 17, 4, 16
    case = _rand_case(rng, B, L, D, N, h0=False, cs=False, conv_b=False)
    case["xz"][:, :, :D] = 0.0
    got = _fwd(lib, case)
    assert np.all(got["y"] == 0.0)
    assert np.all(got["h_last"] == 0.0)
    assert np.all(got["conv_state_out"] == 0.0)
    # and the output is not identically zero once x is not
    case["xz"][:, 3, :D] = 1.0
    got = _fwd(lib, case)
    assert np.abs(got["y"][:, 3:]).max() > 1e-3


# --------------------------------------------------------------------------- P4
def pin_split_equals_unsplit(lib):
    """Running the sequence in pieces, carrying (h_last, conv_state_out) into
    (h0, conv_state_in), equals the single run exactly: the state is all the
    history the next token needs.  Pieces shorter than the conv window included."""
    rng = np.random.default_rng(404)
    B, L, D, N = 2, 37, 3, 16
    case = _rand_case(rng, B, L, D, N)
    full = _fwd(lib, case)
    cuts = [0, 1, 3, 4, 20, 37]
    h, cs = case["h0"], case["conv_state_in"]
    ys = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        piece = dict(case)
        piece.update(xz=case["xz"][:, a:b], dt=case["dt"][:, a:b], Bm=case["Bm"][:, a:b],
                     Cm=case["Cm"][:, a:b], h0=h, conv_state_in=cs)
        out = _fwd(lib, piece)
        ys.append(out["y"])
        h, cs = out["h_last"], out["conv_state_out"]
    assert np.array_equal(np.concatenate(ys, axis=1), full["y"])
    assert np.array_equal(h, full["h_last"])
    assert np.array_equal(cs, full["conv_state_out"])


# --------------------------------------------------------------------------- P5
def _decode_case_from_scan(case, t, layers):
    """The decode-step arguments for token t of a stack of independent scans,
    one per layer (layer l uses scan case layers[l])."""
    D = case[0]["xz"].shape[2] // 2
    get = lambda k: np.stack([c[k] for c in case])  # noqa: E731
    x = np.stack([c["xz"][:, t, :D] for c in case])
    z = np.stack([c["xz"][:, t, D:] for c in case])
    dt = np.stack([c["dt"][:, t] for c in case])
    Bm = np.stack([c["Bm"][:, t] for c in case])
    Cm = np.stack([c["Cm"][:, t] for c in case])
    return dict(x=x, z=z, dt=dt, conv_w=get("conv_w"), conv_b=get("conv_b"), dt_bias=get("dt_bias"),
                Dskip=get("Dskip"), A=get("A"), Bm=Bm, Cm=Cm)


def pin_decode_equals_last_scan_step(lib):
    """The one-token state update applied to the state after L-1 tokens equals
    the scan's token L-1 (output, state, window); and k successive decode steps
    equal a k-token scan.  Two stacked layers with different parameters."""
    rng = np.random.default_rng(505)
    B, L, D, N, NL = 3, 9, 4, 16, 2
    cases = [_rand_case(rng, B, L, D, N) for _ in range(NL)]
    fulls = [_fwd(lib, c) for c in cases]
    # state after L-1 tokens, from the scan
    heads = []
    for c in cases:
        p = dict(c)
        p.update(xz=c["xz"][:, :L - 1], dt=c["dt"][:, :L - 1], Bm=c["Bm"][:, :L - 1], Cm=c["Cm"][:, :L - 1])
        heads.append(_fwd(lib, p))
    args = _decode_case_from_scan(cases, L - 1, NL)
    ssm = np.stack([hd["h_last"] for hd in heads])
    cs = np.stack([hd["conv_state_out"] for hd in heads])
    out = oracle.state_update(**args, ssm_state=ssm, conv_state=cs, library=lib)
    for l in range(NL):
        np.testing.assert_allclose(out["y"][l], fulls[l]["y"][:, L - 1], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(out["ssm_state"][l], fulls[l]["h_last"], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(out["conv_state"][l], fulls[l]["conv_state_out"], rtol=0, atol=0)
    # k decode steps from the initial state == k-token scan
    ssm = np.stack([c["h0"] for c in cases])
    cs = np.stack([c["conv_state_in"] for c in cases])
    for t in range(L):
        args = _decode_case_from_scan(cases, t, NL)
        out = oracle.state_update(**args, ssm_state=ssm, conv_state=cs, library=lib)
        for l in range(NL):
            np.testing.assert_allclose(out["y"][l], fulls[l]["y"][:, t], rtol=1e-12, atol=1e-13)
        ssm, cs = out["ssm_state"], out["conv_state"]
    for l in range(NL):
        np.testing.assert_allclose(ssm[l], fulls[l]["h_last"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(cs[l], fulls[l]["conv_state_out"], rtol=0, atol=0)


# --------------------------------------------------------------------------- P6
def pin_conv_stage(lib):
    """The conv stage equals numpy.convolve with the reversed kernel over the
    sequence left-padded by the carried window, and u = SiLU of it."""
    rng = np.random.default_rng(606)
    for with_cs in (True, False):
        case = _rand_case(rng, 2, 11, 5, 4, cs=with_cs)
        got = _fwd(lib, case, traces=True)
        pre, u, delta = _lib_u_delta(case)
        np.testing.assert_allclose(got["pre"], pre, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(got["u"], u, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(got["delta"], delta, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------- P7
def pin_first_order_iir(lib):
    """N = 1 with constant decay a: h_t = a h_{t-1} + b_t is the first-order IIR
    filter 1 / (1 - a z^-1); compare with scipy.signal.lfilter."""
    rng = np.random.default_rng(707)
    B, L, D, N = 1, 40, 3, 1
    case = _rand_case(rng, B, L, D, N, conv_b=False)
    case["dt"] = np.zeros((B, L, D))
    case["conv_w"] = np.tile(np.array([0.0, 0.0, 0.0, 1.0]), (D, 1))  # pre = x_t
    case["Cm"] = np.ones((B, L, N))
    case["Dskip"] = np.zeros(D)
    got = _fwd(lib, case)
    x = case["xz"][0, :, :D]
    g = _gate_z(case)[0]
    for d in range(D):
        dlt = lib_softplus(case["dt_bias"][d])
        a = np.exp(dlt * case["A"][d, 0])
        drive = dlt * case["Bm"][0, :, 0] * lib_silu(x[:, d])
        h, _ = scipy.signal.lfilter([1.0], [1.0, -a], drive, zi=[a * case["h0"][0, d, 0]])
        np.testing.assert_allclose(got["y"][0, :, d], h * g[:, d], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(got["h_last"][0, d, 0], h[-1], rtol=1e-11, atol=1e-13)


# --------------------------------------------------------------------------- P8
def pin_A_zero(lib):
    """A = 0: no decay, h_t = h0 + prefix sum of Delta u B."""
    rng = np.random.default_rng(808)
    B, L, D, N = 2, 25, 3, 7
    case = _rand_case(rng, B, L, D, N)
    case["A"] = np.zeros((D, N))
    got = _fwd(lib, case)
    _, u, delta = _lib_u_delta(case)
    g = _gate_z(case)
    for b in range(B):
        for d in range(D):
            hs = case["h0"][b, d][None, :] + np.cumsum((delta[b, :, d] * u[b, :, d])[:, None] * case["Bm"][b], axis=0)
            y = ((case["Cm"][b] * hs).sum(1) + case["Dskip"][d] * u[b, :, d]) * g[b, :, d]
            np.testing.assert_allclose(got["y"][b, :, d], y, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(got["h_last"][b, d], hs[-1], rtol=1e-11, atol=1e-13)


# --------------------------------------------------------------------------- P9
def pin_softplus_roundtrip(lib):
    """dt = 0 and dt_bias = inverse-softplus(v) give Delta = v; softplus is
    exact far into both tails."""
    rng = np.random.default_rng(909)
    D = 8
    v = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), D))
    case = _rand_case(rng, 1, 3, D, 2)
    case["dt"] = np.zeros((1, 3, D))
    case["dt_bias"] = np.log(np.expm1(v))
    got = _fwd(lib, case, traces=True)
    np.testing.assert_allclose(got["delta"][0], np.tile(v, (3, 1)), rtol=1e-13, atol=0)
    case["dt_bias"] = np.array([-60.0, -30.0, -1.0, 0.0, 1.0, 30.0, 60.0, 700.0])
    got = _fwd(lib, case, traces=True)
    expect = np.array([np.exp(-60.0), np.log1p(np.exp(-30.0)), np.log1p(np.exp(-1.0)), np.log(2.0),
                       1.0 + np.log1p(np.exp(-1.0)), 30.0 + np.exp(-30.0), 60.0, 700.0])
    np.testing.assert_allclose(got["delta"][0, 0], expect, rtol=1e-14, atol=0)


# --------------------------------------------------------------------------- P10
def pin_skip_and_gate(lib):
    """C = 0 removes the state from the output: y = D u SiLU(z); the gate
    is SiLU of z (not of x), applied after the skip is added."""
    rng = np.random.default_rng(1010)
    B, L, D, N = 2, 9, 4, 3
    case = _rand_case(rng, B, L, D, N)
    case["Cm"] = np.zeros((B, L, N))
    got = _fwd(lib, case)
    _, u, _ = _lib_u_delta(case)
    np.testing.assert_allclose(got["y"], case["Dskip"][None, None, :] * u * _gate_z(case), rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------- P11
def pin_channel_split(lib):
    """Channels are independent: splitting the channel range across threads
    gives bit-identical results."""
    rng = np.random.default_rng(1111)
    case = _rand_case(rng, 2, 13, 7, 16)
    a = _fwd(lib, case, threads=1)
    b = _fwd(lib, case, threads=3)
    for k in a:
        assert np.array_equal(a[k], b[k])


def pin_rmsnorm_constant_rows(lib):
    """A row of n equal entries c with unit weights normalises to
    c / sqrt(c^2 + eps) in every entry (closed form)."""
    n = 16
    for c, eps in ((3.0, 0.25), (-0.5, 1e-6), (0.0, 0.5), (1e-3, 1e-6)):
        out = oracle.rmsnorm_rows(np.full((2, n), c), np.ones(n), eps, library=lib)
        np.testing.assert_allclose(out, c / np.sqrt(c * c + eps), rtol=1e-14, atol=1e-300)


def pin_rmsnorm_library(lib):
    """Random rows and per-column weights against torch's rms_norm in float64
    (library routine), with a small and a large eps."""
    import torch

    rng = np.random.default_rng(41)
    x = rng.standard_normal((37, 16)) * rng.uniform(0.1, 5.0, (37, 1))
    w = rng.uniform(0.2, 2.0, 16)
    for eps in (1e-6, 0.3):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (16,), torch.from_numpy(w), eps).numpy()
        np.testing.assert_allclose(oracle.rmsnorm_rows(x, w, eps, library=lib), ref, rtol=1e-12, atol=1e-15)


def pin_rmsnorm_homogeneity(lib):
    """Scaling a row by a and eps by a^2 leaves the result unchanged; scaling
    the weights by k scales it by k; the normalised row/weight has mean square
    ms / (ms + eps)."""
    rng = np.random.default_rng(42)
    x = rng.standard_normal((9, 16))
    w = rng.uniform(0.5, 1.5, 16)
    base = oracle.rmsnorm_rows(x, w, 0.1, library=lib)
    np.testing.assert_allclose(oracle.rmsnorm_rows(7.0 * x, w, 0.1 * 49.0, library=lib), base, rtol=1e-13)
    np.testing.assert_allclose(oracle.rmsnorm_rows(x, 3.0 * w, 0.1, library=lib), 3.0 * base, rtol=1e-13)
    ms = np.mean(x ** 2, axis=-1)
    np.testing.assert_allclose(np.mean((base / w) ** 2, axis=-1), ms / (ms + 0.1), rtol=1e-13)


def pin_normed_forward_uses_normalised_B_and_C(lib):
    """With every B_t (and C_t) row constant, RMSNorm with weights w turns it
    into w * c / sqrt(c^2 + eps): the normed forward equals the plain forward
    on those values, and a weight of None leaves the input untouched."""
    rng = np.random.default_rng(43)
    case = _rand_case(rng, 1, 12, 3, 16)
    cb = rng.uniform(0.5, 2.0, (1, 12, 1))
    cc = rng.uniform(-2.0, -0.5, (1, 12, 1))
    case["Bm"] = np.repeat(cb, 16, axis=-1)
    case["Cm"] = np.repeat(cc, 16, axis=-1)
    wb, wc, eps = rng.uniform(0.5, 1.5, 16), rng.uniform(0.5, 1.5, 16), 0.2
    got = oracle.mixer_fwd_normed(case["xz"], case["conv_w"], case["conv_b"], case["dt"], case["dt_bias"],
                                  case["A"], case["Bm"], case["Cm"], case["Dskip"], case["h0"],
                                  case["conv_state_in"], b_norm_w=wb, c_norm_w=wc, norm_eps=eps, library=lib)
    want_case = dict(case, Bm=wb * cb / np.sqrt(cb * cb + eps), Cm=wc * cc / np.sqrt(cc * cc + eps))
    want = _fwd(lib, want_case)
    for k in ("y", "h_last"):
        np.testing.assert_allclose(got[k], want[k], rtol=1e-12, atol=1e-14)
    plain = oracle.mixer_fwd_normed(case["xz"], case["conv_w"], case["conv_b"], case["dt"], case["dt_bias"],
                                    case["A"], case["Bm"], case["Cm"], case["Dskip"], case["h0"],
                                    case["conv_state_in"], library=lib)
    np.testing.assert_array_equal(plain["y"], _fwd(lib, case)["y"])


def pin_matmul_library(lib):
    """The projection product against numpy's matmul on random operands
    (library routine), including an empty K and a single row."""
    rng = np.random.default_rng(51)
    for M, N, K in ((7, 5, 33), (1, 288, 64), (4, 3, 0)):
        A = rng.standard_normal((M, K))
        Bw = rng.standard_normal((N, K))
        np.testing.assert_allclose(oracle.matmul_nt(A, Bw, threads=2, library=lib), A @ Bw.T, rtol=1e-12,
                                   atol=1e-12)


def pin_matmul_selection(lib):
    """Rows of Bw that are unit vectors select columns of A (closed form), and
    a rank-one product a b^T times (c d^T)^T is (b . d) a c^T."""
    rng = np.random.default_rng(52)
    A = rng.standard_normal((6, 10))
    sel = np.array([3, 0, 9, 3])
    E = np.eye(10)[sel]
    np.testing.assert_array_equal(oracle.matmul_nt(A, E, library=lib), A[:, sel])
    a, b, c, d = (rng.standard_normal(n) for n in (6, 10, 4, 10))
    got = oracle.matmul_nt(np.outer(a, b), np.outer(c, d), library=lib)
    np.testing.assert_allclose(got, np.dot(b, d) * np.outer(a, c), rtol=1e-12, atol=1e-12)


def pin_projected_forward_wiring(lib):
    """The mixer with its projections: u from the conv + SiLU (checked against
    scipy's logistic and numpy's convolve), then x_proj's output split as
    [dt_low | B | C], optional norms, dt = dt_low W_dt^T, and the scan on those
    -- recomputed here with numpy's matmul and the plain forward."""
    rng = np.random.default_rng(53)
    Bsz, Lq, D, N, R = 2, 9, 6, 16, 5
    case = _rand_case(rng, Bsz, Lq, D, N)
    W_x = rng.standard_normal((R + 2 * N, D)) * 0.4
    W_dt = rng.standard_normal((D, R)) * 0.4
    wd, wb, wc = rng.uniform(0.5, 1.5, R), rng.uniform(0.5, 1.5, N), rng.uniform(0.5, 1.5, N)
    got = oracle.projected_fwd(case["xz"], case["conv_w"], case["conv_b"], W_x, W_dt, case["dt_bias"], case["A"],
                               case["Dskip"], case["h0"], case["conv_state_in"], dt_norm_w=wd, b_norm_w=wb,
                               c_norm_w=wc, norm_eps=0.1, library=lib)
    # u by library routines: the causal conv over [window, x] and x * logistic(x)
    x = case["xz"][..., :D]
    u = np.zeros((Bsz, Lq, D))
    for b in range(Bsz):
        for d in range(D):
            seq = np.concatenate([case["conv_state_in"][b, d], x[b, :, d]])
            pre = np.convolve(seq, case["conv_w"][d, ::-1], mode="valid") + case["conv_b"][d]
            u[b, :, d] = lib_silu(pre)
    np.testing.assert_allclose(got["u"], u, rtol=1e-12, atol=1e-12)

    def rms(v, w):
        return v * w / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + 0.1)

    x_dbl = u @ W_x.T
    dt_low, Bm, Cm = rms(x_dbl[..., :R], wd), rms(x_dbl[..., R:R + N], wb), rms(x_dbl[..., R + N:], wc)
    dt = dt_low @ W_dt.T
    for k, v in (("dt_low", dt_low), ("Bm", Bm), ("Cm", Cm), ("dt", dt)):
        np.testing.assert_allclose(got[k], v, rtol=1e-11, atol=1e-12)
    want = _fwd(lib, dict(case, dt=dt, Bm=Bm, Cm=Cm))
    for k in ("y", "h_last", "conv_state_out"):
        np.testing.assert_allclose(got[k], want[k], rtol=1e-10, atol=1e-12)
    # stored as bf16: each intermediate is the exact one rounded by torch's cast
    import torch

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(torch.float64).numpy()

    got_b = oracle.projected_fwd(case["xz"], case["conv_w"], case["conv_b"], W_x, W_dt, case["dt_bias"], case["A"],
                                 case["Dskip"], case["h0"], case["conv_state_in"], dt_norm_w=wd, b_norm_w=wb,
                                 c_norm_w=wc, norm_eps=0.1, store="bf16", library=lib)
    ub = bf(u)
    xb = ub @ W_x.T
    dlb, Bb, Cb = bf(rms(xb[..., :R], wd)), bf(rms(xb[..., R:R + N], wb)), bf(rms(xb[..., R + N:], wc))
    dtb = bf(dlb @ W_dt.T)
    np.testing.assert_array_equal(got_b["u"], ub)
    # the products are summed in another order than numpy's: a value next to a
    # rounding boundary may land one bf16 step (2^-7 relative) away
    for k, v in (("dt_low", dlb), ("Bm", Bb), ("Cm", Cb), ("dt", dtb)):
        np.testing.assert_allclose(got_b[k], v, rtol=2.0 ** -7, atol=1e-12)
    want_b = _fwd(lib, dict(case, dt=dtb, Bm=Bb, Cm=Cb))
    np.testing.assert_allclose(got_b["y"], want_b["y"], rtol=1e-6, atol=1e-9)


# ---------------------------------------------------------------- Mamba-2 form
def _ssd_case(rng, Bsz, L, H, P, N, G, *, z=True, h0=True, dskip=True, bias=True):
    return dict(
        x=rng.standard_normal((Bsz, L, H * P)),
        z=rng.standard_normal((Bsz, L, H * P)) if z else None,
        dt=0.4 * rng.standard_normal((Bsz, L, H)),
        dt_bias=rng.uniform(-3.0, 0.5, H) if bias else None,
        A=-np.exp(rng.uniform(np.log(0.2), np.log(4.0), H)),
        Bm=rng.standard_normal((Bsz, L, G, N)),
        Cm=rng.standard_normal((Bsz, L, G, N)),
        Dskip=rng.normal(1.0, 0.3, H) if dskip else None,
        h0=0.5 * rng.standard_normal((Bsz, H, P, N)) if h0 else None,
    )


def _ssd(lib, case, P, **kw):
    return oracle.ssd_fwd(case["x"], case["z"], case["dt"], case["dt_bias"], case["A"], case["Bm"], case["Cm"],
                          case["Dskip"], case["h0"], headdim=P, library=lib, **kw)


def pin_ssd_quadratic_form(lib):
    """The Mamba-2 form against its materialised (quadratic, attention-like)
    form, built here with numpy on tiny inputs: with decays a_t = exp(Delta_t A)
    of a scalar-times-identity state matrix,
        y_i = sum_{j<=i} (C_i . B_j) (prod_{k=j+1..i} a_k) Delta_j x_j
              + (prod_{k<=i} a_k) C_i . h0 + D x_i,   gated by SiLU(z),
        h_last = sum_j (prod_{k>j} a_k) Delta_j B_j x_j^T + (prod_k a_k) h0,
    softplus and SiLU through numpy's logaddexp and scipy's logistic."""
    rng = np.random.default_rng(71)
    Bsz, L, H, P, N, G = 2, 13, 4, 3, 5, 2
    for z in (True, False):
        case = _ssd_case(rng, Bsz, L, H, P, N, G, z=z)
        got = _ssd(lib, case, P)
        for b in range(Bsz):
            for h in range(H):
                g = h // (H // G)
                delta = lib_softplus(case["dt"][b, :, h] + case["dt_bias"][h])
                la = delta * case["A"][h]                     # log of each token's decay
                cum = np.cumsum(la)
                Bg, Cg = case["Bm"][b, :, g, :], case["Cm"][b, :, g, :]
                seg = cum[:, None] - cum[None, :]             # sum_{k=j+1..i} la_k
                Mq = np.where(np.tril(np.ones((L, L))) > 0, (Cg @ Bg.T) * np.exp(np.minimum(seg, 0.0)), 0.0)
                xs = case["x"][b, :, h * P:(h + 1) * P]       # [L, P]
                h0 = case["h0"][b, h]                         # [P, N]
                y = Mq @ (delta[:, None] * xs) + np.exp(cum)[:, None] * (Cg @ h0.T) + case["Dskip"][h] * xs
                if z:
                    y = y * lib_silu(case["z"][b, :, h * P:(h + 1) * P])
                np.testing.assert_allclose(got["y"][b, :, h * P:(h + 1) * P], y, rtol=1e-10, atol=1e-11)
                w = np.exp(cum[-1] - cum) * delta             # weight of token j in the final state
                hl = (w[:, None] * xs).T @ Bg + np.exp(cum[-1]) * h0
                np.testing.assert_allclose(got["h_last"][b, h], hl, rtol=1e-10, atol=1e-11)


def pin_ssd_first_order_iir(lib):
    """One head, one channel, one state, constant step: the state is the
    first-order filter h_t = a h_{t-1} + b_t, checked with scipy's lfilter
    (initial condition from h0), and y_t = C_t h_t + D x_t with no gate."""
    rng = np.random.default_rng(73)
    L = 40
    case = _ssd_case(rng, 1, L, 1, 1, 1, 1, z=False)
    case["dt"] = np.full((1, L, 1), 0.3)
    got = _ssd(lib, case, 1)
    delta = lib_softplus(0.3 + case["dt_bias"][0])
    a = np.exp(delta * case["A"][0])
    drive = delta * case["Bm"][0, :, 0, 0] * case["x"][0, :, 0]
    h0 = case["h0"][0, 0, 0, 0]
    h, _ = scipy.signal.lfilter([1.0], [1.0, -a], drive, zi=[a * h0])
    np.testing.assert_allclose(got["h_last"][0, 0, 0, 0], h[-1], rtol=1e-12, atol=1e-13)
    y = case["Cm"][0, :, 0, 0] * h + case["Dskip"][0] * case["x"][0, :, 0]
    np.testing.assert_allclose(got["y"][0, :, 0], y, rtol=1e-11, atol=1e-12)


def pin_ssd_zero_input(lib):
    """x = 0 and h0 = 0 give y = 0 and a zero final state, whatever dt, B, C, z."""
    rng = np.random.default_rng(79)
    case = _ssd_case(rng, 2, 9, 2, 3, 4, 1, h0=False)
    case["x"] = np.zeros_like(case["x"])
    got = _ssd(lib, case, 3)
    assert np.all(got["y"] == 0.0) and np.all(got["h_last"] == 0.0)


def pin_ssd_split_equals_unsplit(lib):
    """Running a sequence as two calls, the first call's final state carried
    into the second as h0, equals the single run exactly: the state is all the
    history the recurrence needs."""
    rng = np.random.default_rng(83)
    P = 2
    case = _ssd_case(rng, 2, 17, 4, P, 3, 2)
    full = _ssd(lib, case, P)
    cut = 6

    def part(lo, hi, h0):
        c = dict(case)
        for k in ("x", "z", "dt", "Bm", "Cm"):
            c[k] = case[k][:, lo:hi]
        c["h0"] = h0
        return _ssd(lib, c, P)

    first = part(0, cut, case["h0"])
    second = part(cut, 17, first["h_last"])
    np.testing.assert_array_equal(np.concatenate([first["y"], second["y"]], axis=1), full["y"])
    np.testing.assert_array_equal(second["h_last"], full["h_last"])


def pin_ssd_group_mapping(lib):
    """G groups split the H heads into G consecutive blocks: a 2-group run on
    4 heads equals two 1-group runs, heads 0-1 on group 0's B/C and heads 2-3
    on group 1's."""
    rng = np.random.default_rng(89)
    P = 2
    case = _ssd_case(rng, 1, 11, 4, P, 3, 2)
    got = _ssd(lib, case, P)
    for g in range(2):
        heads = slice(2 * g, 2 * g + 2)
        chans = slice(2 * g * P, (2 * g + 2) * P)
        sub = dict(x=case["x"][..., chans], z=case["z"][..., chans], dt=case["dt"][..., heads],
                   dt_bias=case["dt_bias"][heads], A=case["A"][heads], Bm=case["Bm"][:, :, g:g + 1],
                   Cm=case["Cm"][:, :, g:g + 1], Dskip=case["Dskip"][heads], h0=case["h0"][:, heads])
        one = _ssd(lib, sub, P)
        np.testing.assert_array_equal(got["y"][..., chans], one["y"])
        np.testing.assert_array_equal(got["h_last"][:, heads], one["h_last"])


# ---------------------------------------------------------------- Mamba-3 form
def _m3_case(rng, Bsz, L, R, H, P, N, G, *, z=True, h0=True, prev=True, trap=True, dskip=True):
    return dict(
        x=rng.standard_normal((Bsz, L, R, H * P)),
        z=rng.standard_normal((Bsz, L, R, H * P)) if z else None,
        dt=0.4 * rng.standard_normal((Bsz, L, H)),
        trap=rng.uniform(0.0, 1.0, (Bsz, L, H)) if trap else None,
        dt_bias=rng.uniform(-3.0, 0.5, H),
        A=-np.exp(rng.uniform(np.log(0.2), np.log(4.0), H)),
        theta=rng.uniform(-3.0, 3.0, (H, N // 2)),
        Bm=rng.standard_normal((Bsz, L, R, G, N)),
        Cm=rng.standard_normal((Bsz, L, R, G, N)),
        Dskip=rng.normal(1.0, 0.3, H) if dskip else None,
        h0=0.5 * rng.standard_normal((Bsz, H, P, N)) if h0 else None,
        x_prev=rng.standard_normal((Bsz, R, H * P)) if prev else None,
        B_prev=rng.standard_normal((Bsz, R, G, N)) if prev else None,
    )


def _m3(lib, case, P, **kw):
    return oracle.m3_fwd(case["x"], case["z"], case["dt"], case["trap"], case["dt_bias"], case["A"], case["theta"],
                         case["Bm"], case["Cm"], case["Dskip"], case["h0"], case["x_prev"], case["B_prev"],
                         headdim=P, library=lib, **kw)


def _cplx(v):
    """[..., N] real pairs (2k, 2k+1) as [..., N/2] complex numbers."""
    return v[..., 0::2] + 1j * v[..., 1::2]


def pin_m3_quadratic_form(lib):
    """The Mamba-3 form against its materialised form, built with numpy's
    complex arithmetic on tiny inputs.  With a_q = exp(Delta_q (A + i theta))
    per state pair, token s's input u_s = sum_r b_s[r] x_s[r] reaches the
    state after token t >= s with weight prod_{q=s+1..t} a_q times
    lambda_s Delta_s (its own step) plus, when s < t, (1 - lambda_{s+1})
    Delta_{s+1} (the next step's trapezoid tap); h0 and the previous call's
    input u_{-1} (weight (1 - lambda_0) Delta_0) reach it through
    prod_{q=0..t} a_q.  y reads Re(conj(c) s)."""
    rng = np.random.default_rng(97)
    Bsz, L, R, H, P, N, G = 2, 9, 2, 4, 2, 6, 2
    for trap in (True, False):          # no trap input: the plain trapezoid, lambda = 1/2
        _m3_quadratic_case(lib, _m3_case(rng, Bsz, L, R, H, P, N, G, trap=trap), P, G)


def _m3_quadratic_case(lib, case, P, G):
    got = _m3(lib, case, P)
    Bsz, L, R, C = case["x"].shape
    H = case["A"].shape[0]
    for b in range(Bsz):
        for h in range(H):
            g = h // (H // G)
            delta = lib_softplus(case["dt"][b, :, h] + case["dt_bias"][h])
            lam = case["trap"][b, :, h] if case["trap"] is not None else np.full(L, 0.5)
            la = delta[:, None] * (case["A"][h] + 1j * case["theta"][h][None, :])     # [L, K] log of a_q
            cum = np.cumsum(la, axis=0)
            bb = _cplx(case["Bm"][b, :, :, g, :])          # [L, R, K]
            cc = _cplx(case["Cm"][b, :, :, g, :])
            bp = _cplx(case["B_prev"][b, :, g, :])           # [R, K]
            for p in range(P):
                c = h * P + p
                xs = case["x"][b, :, :, c]                   # [L, R]
                u = np.einsum("lrk,lr->lk", bb, xs)          # [L, K]
                u_prev = np.einsum("rk,r->k", bp, case["x_prev"][b, :, c])
                s0 = _cplx(case["h0"][b, h, p])
                states = []
                for t in range(L):
                    st = np.exp(cum[t]) * (s0 + (1 - lam[0]) * delta[0] * u_prev)
                    for s_ in range(t + 1):
                        w = lam[s_] * delta[s_] + ((1 - lam[s_ + 1]) * delta[s_ + 1] if s_ < t else 0.0)
                        st = st + np.exp(cum[t] - cum[s_]) * w * u[s_]
                    states.append(st)
                    for r in range(R):
                        yv = np.real(np.sum(np.conj(cc[t, r]) * st)) + case["Dskip"][h] * xs[t, r]
                        yv = yv * lib_silu(case["z"][b, t, r, c])
                        np.testing.assert_allclose(got["y"][b, t, r, c], yv, rtol=1e-9, atol=1e-10)
                hl = got["h_last"][b, h, p]
                np.testing.assert_allclose(hl[0::2] + 1j * hl[1::2], states[-1], rtol=1e-9, atol=1e-10)


def pin_m3_rotary_equivalence(lib):
    """The complex state is a data-dependent rotary embedding: with the
    rotation frequencies theta, the run equals the theta = 0 run on B and C
    rotated by the cumulative phase Phi_t = theta * sum_{q<=t} Delta_q
    (numpy's complex exp), its final state rotated back by Phi_{L-1}.  One
    head per group, since the phase belongs to the head."""
    rng = np.random.default_rng(101)
    Bsz, L, R, H, P, N, G = 1, 14, 2, 2, 3, 8, 2
    case = _m3_case(rng, Bsz, L, R, H, P, N, G)
    got = _m3(lib, case, P)
    rot = dict(case, theta=np.zeros_like(case["theta"]), Bm=case["Bm"].copy(), Cm=case["Cm"].copy())
    phases = []
    for h in range(H):
        delta = lib_softplus(case["dt"][0, :, h] + case["dt_bias"][h])
        phi = np.cumsum(delta)[:, None] * case["theta"][h][None, :]        # [L, K]
        phases.append(phi)
        e = np.exp(-1j * phi)                                                # [L, K]
        for M_ in ("Bm", "Cm"):
            v = _cplx(case[M_][0, :, :, h, :]) * e[:, None, :]
            rot[M_][0, :, :, h, 0::2] = v.real
            rot[M_][0, :, :, h, 1::2] = v.imag
    plain = _m3(lib, rot, P)
    np.testing.assert_allclose(got["y"], plain["y"], rtol=1e-9, atol=1e-10)
    for h in range(H):
        back = _cplx(plain["h_last"][0, h]) * np.exp(1j * phases[h][-1])[None, :]
        np.testing.assert_allclose(_cplx(got["h_last"][0, h]), back, rtol=1e-9, atol=1e-10)


def pin_m3_euler_is_mamba2(lib):
    """With lambda = 1, theta = 0 and one input (R = 1) the form is the
    Mamba-2 recurrence (oracle_ssd_fwd, pinned on its own)."""
    rng = np.random.default_rng(103)
    Bsz, L, H, P, N, G = 2, 11, 4, 3, 6, 2
    case = _m3_case(rng, Bsz, L, 1, H, P, N, G)
    case.update(trap=np.ones((Bsz, L, H)), theta=np.zeros((H, N // 2)))
    got = _m3(lib, case, P)
    ref = oracle.ssd_fwd(case["x"][:, :, 0], case["z"][:, :, 0], case["dt"], case["dt_bias"], case["A"],
                         case["Bm"][:, :, 0], case["Cm"][:, :, 0], case["Dskip"], case["h0"], headdim=P,
                         library=lib)
    np.testing.assert_allclose(got["y"][:, :, 0], ref["y"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got["h_last"], ref["h_last"], rtol=1e-12, atol=1e-13)


def pin_m3_mimo_superposition(lib):
    """The R inputs share one state, which is linear in them: with no gate,
    the rank-2 run's output r equals the sum of two single-input runs (input
    0 with h0 and its previous token, input 1 with neither), both read out
    with output r's C and no skip, plus D x_r; its final state is the sum of
    theirs."""
    rng = np.random.default_rng(107)
    Bsz, L, H, P, N, G = 1, 10, 2, 2, 4, 1
    case = _m3_case(rng, Bsz, L, 2, H, P, N, G, z=False)
    got = _m3(lib, case, P)
    for r_out in range(2):
        total_y = np.zeros((Bsz, L, H * P))
        total_h = np.zeros((Bsz, H, P, N))
        for r_in in range(2):
            one = dict(case, x=case["x"][:, :, r_in:r_in + 1], Bm=case["Bm"][:, :, r_in:r_in + 1],
                       Cm=case["Cm"][:, :, r_out:r_out + 1], Dskip=None,
                       h0=case["h0"] if r_in == 0 else None,
                       x_prev=case["x_prev"][:, r_in:r_in + 1], B_prev=case["B_prev"][:, r_in:r_in + 1])
            o = _m3(lib, one, P)
            total_y += o["y"][:, :, 0]
            total_h += o["h_last"]
        want = total_y + case["Dskip"].repeat(P)[None, None, :] * case["x"][:, :, r_out]
        np.testing.assert_allclose(got["y"][:, :, r_out], want, rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(got["h_last"], total_h, rtol=1e-10, atol=1e-11)


def pin_m3_split_equals_unsplit(lib):
    """Two calls, the first one's final state carried as h0 and its last
    token's x and B passed as x_prev / B_prev, equal the single run exactly."""
    rng = np.random.default_rng(109)
    P = 2
    case = _m3_case(rng, 2, 15, 2, 4, P, 6, 2)
    full = _m3(lib, case, P)
    cut = 6

    def part(lo, hi, h0, xp, bp):
        c = dict(case)
        for k in ("x", "z", "dt", "trap", "Bm", "Cm"):
            c[k] = case[k][:, lo:hi]
        c.update(h0=h0, x_prev=xp, B_prev=bp)
        return _m3(lib, c, P)

    first = part(0, cut, case["h0"], case["x_prev"], case["B_prev"])
    second = part(cut, 15, first["h_last"], case["x"][:, cut - 1], case["Bm"][:, cut - 1])
    np.testing.assert_array_equal(np.concatenate([first["y"], second["y"]], axis=1), full["y"])
    np.testing.assert_array_equal(second["h_last"], full["h_last"])


def pin_m3_zero_input(lib):
    """x = 0, no h0 and no previous token give y = 0 and a zero state."""
    rng = np.random.default_rng(113)
    case = _m3_case(rng, 1, 7, 2, 2, 2, 4, 1, h0=False, prev=False)
    case["x"] = np.zeros_like(case["x"])
    got = _m3(lib, case, 2)
    assert np.all(got["y"] == 0.0) and np.all(got["h_last"] == 0.0)


ALL_PINS = [
    pin_m3_quadratic_form,
    pin_m3_rotary_equivalence,
    pin_m3_euler_is_mamba2,
    pin_m3_mimo_superposition,
    pin_m3_split_equals_unsplit,
    pin_m3_zero_input,
    pin_ssd_quadratic_form,
    pin_ssd_first_order_iir,
    pin_ssd_zero_input,
    pin_ssd_split_equals_unsplit,
    pin_ssd_group_mapping,
    pin_matmul_library,
    pin_matmul_selection,
    pin_projected_forward_wiring,
    pin_rmsnorm_constant_rows,
    pin_rmsnorm_library,
    pin_rmsnorm_homogeneity,
    pin_normed_forward_uses_normalised_B_and_C,
    pin_lti_closed_form,
    pin_brute_force_selective,
    pin_zero_input,
    pin_split_equals_unsplit,
    pin_decode_equals_last_scan_step,
    pin_conv_stage,
    pin_first_order_iir,
    pin_A_zero,
    pin_softplus_roundtrip,
    pin_skip_and_gate,
    pin_channel_split,
]
