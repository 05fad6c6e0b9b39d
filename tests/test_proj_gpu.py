"""The projections either side of the scan, on the tensor cores, against the
fp64 oracle: the projection product alone (mamba_proj_matmul, fp32 and bf16
output, ragged and full-size shapes), and the mixer with its producers
(mamba_mixer_fwd_projected: conv -> x_proj -> [dt_low | B | C] with optional
RMSNorms -> dt_proj -> scan)."""

import numpy as np
import pytest
import torch

import mamba_selective_scan_core_b200 as mm
import oracle
from gpu_util import THREADS, _record as gpu_util_record, assert_close, gpu_fwd, np64, to_dev
from workloads import CONFIGS, make_mixer_inputs, make_mixer_inputs_custom, make_norm_weights, \
    make_projection_weights

pytestmark = pytest.mark.gpu


def _bf16_randn(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def check_matmul(M, N, K, out_dtype, seed, rows=None):
    A = _bf16_randn((M, K), seed)
    W = _bf16_randn((N, K), seed + 1, scale=1.0 / np.sqrt(K))
    out = mm.proj_matmul(A.cuda(), W.cuda(), out_dtype=out_dtype)
    ws_status = None
    torch.cuda.synchronize()
    got = np64(out)
    if rows is not None:
        A, got = A[rows], got[rows]
    ref = oracle.matmul_nt(A, W, threads=THREADS)
    if out_dtype == torch.float32:
        # fp32 accumulation of K products: within 1e-5 of the output's scale per sqrt(K) terms
        bound = 1e-6 * np.sqrt(K) * (1.0 + np.sqrt(np.mean(ref ** 2)))
        err = float(np.max(np.abs(got - ref))) if got.size else 0.0
        assert err <= bound, (err, bound)
    else:
        assert_close(got, ref, "bf16", "out", stored_bf16=True)
    return ws_status


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (130, 24, 72), (300, 144, 200), (129, 288, 1024), (256, 520, 64),
                                   (128, 256, 4096)])
def test_matmul_shapes(M, N, K, out_dtype):
    check_matmul(M, N, K, out_dtype, seed=M * 7 + N + K)


def test_matmul_x_proj_shape_full_size():
    """x_proj at the Jamba size: 4096 tokens x 288 outputs x 8192 (sampled rows)."""
    rows = np.array(sorted(set(list(range(8)) + list(range(4088, 4096)) + list(range(8, 4088, 61)))))
    check_matmul(4096, 288, 8192, torch.float32, seed=5, rows=rows)


def test_matmul_dt_proj_shape_full_size():
    """dt_proj at the Jamba size: 4096 tokens x 8192 outputs x 256 (sampled rows)."""
    rows = np.array(sorted(set(list(range(4)) + list(range(4092, 4096)) + list(range(4, 4092, 127)))))
    check_matmul(4096, 8192, 256, torch.bfloat16, seed=6, rows=rows)


def test_matmul_status_is_clean():
    A = _bf16_randn((256, 64), 9).cuda()
    W = _bf16_randn((64, 64), 10).cuda()
    ws = torch.empty(mm.proj_matmul_workspace_size(256, 64, 64), dtype=torch.uint8, device="cuda")
    mm.proj_matmul(A, W, workspace=ws)
    assert mm.check_status(ws) == 0


def check_projected(inp, R, norms, seed, chans=None):
    D = inp["conv_w"].shape[0]
    W_x, W_dt, wd = make_projection_weights(D, R, seed=seed)
    wb, wc = make_norm_weights(seed=seed + 1)
    if not norms:
        wd = wb = wc = None
    dev = to_dev(inp)
    cuda = lambda t: t.cuda() if t is not None else None  # noqa: E731
    ws = torch.empty(mm.projected_workspace_size(*inp["xz"].shape[:2], D, R), dtype=torch.uint8, device="cuda")
    y, h, cs = mm.mixer_fwd_projected(dev["xz"], dev["conv_w"], dev["conv_b"], W_x.cuda(), W_dt.cuda(),
                                      dev["dt_bias"], dev["A"], dev["Dskip"], dev.get("h0"),
                                      dev.get("conv_state_in"), dt_norm_w=cuda(wd), b_norm_w=cuda(wb),
                                      c_norm_w=cuda(wc), norm_eps=1e-6, workspace=ws)
    assert mm.check_status(ws) == 0
    torch.cuda.synchronize()
    # the oracle stores the intermediates (u, dt_low, B, C, dt) as bf16, as the
    # library does between its kernels; its arithmetic stays fp64
    ref = oracle.projected_fwd(inp["xz"], inp["conv_w"], inp["conv_b"], W_x, W_dt, inp["dt_bias"], inp["A"],
                               inp["Dskip"], inp.get("h0"), inp.get("conv_state_in"), dt_norm_w=wd, b_norm_w=wb,
                               c_norm_w=wc, norm_eps=1e-6, store="bf16", threads=THREADS)
    Bsz, L, _ = inp["xz"].shape
    # 1. each stored intermediate within one bf16 rounding step of the oracle's
    inter = mm.projected_intermediates(ws, Bsz, L, D, R)
    for k in ("dt_low", "Bm", "Cm", "dt"):
        assert_close(np64(inter[k]), ref[k], "bf16", k, stored_bf16=True, rounded_steps=1)
    # 2. the chain's outputs are exactly the scan of those intermediates (the scan
    #    itself is checked against the oracle by the parity tests)
    y2, h2, cs2 = gpu_fwd(dict(dev, dt=inter["dt"].contiguous(), Bm=inter["Bm"].contiguous(),
                               Cm=inter["Cm"].contiguous()))
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(h, h2) and torch.equal(cs, cs2)
    np.testing.assert_array_equal(np64(cs), ref["conv_state_out"])
    # 3. end to end against the oracle's chain: the rms bound of the bf16 path.  A
    #    stored value that rounds one step differently moves y by up to 2^-7
    #    |C_n h_n| at its token, which exceeds any budget in |y| where the terms
    #    cancel, so the per-element check is the one of steps 1 and 2.
    got_y, got_h = np64(y), np64(h)
    ref_y, ref_h = ref["y"], ref["h_last"]
    if chans is not None:
        got_y, ref_y = got_y[..., chans], ref_y[..., chans]
        got_h, ref_h = got_h[:, chans], ref_h[:, chans]
    for got, want, name in ((got_y, ref_y, "y"), (got_h, ref_h, "h_last")):
        rms = float(np.sqrt(np.mean(want ** 2)))
        rerr = float(np.sqrt(np.mean((got - want) ** 2)))
        gpu_util_record(name + " (rms)", got.size, rerr / (2e-2 * rms))
        assert rerr <= 2e-2 * rms, (name, rerr, rms)


@pytest.mark.parametrize("norms", [False, True])
@pytest.mark.parametrize("B,L,D,R", [(1, 1, 64, 32), (2, 200, 128, 32), (1, 333, 256, 64), (3, 97, 192, 96)])
def test_projected_small(B, L, D, R, norms):
    inp = make_mixer_inputs_custom(B, L, D, act="bf16", seed=3000 + L + D, h0_std=0.3, conv_state_std=1.0,
                                   conv_b_std=0.2)
    check_projected(inp, R, norms, seed=L + R)


def test_projected_jamba_prefill_full():
    """The Jamba-shaped layer (4096 tokens, d_inner 8192, dt_rank 256) with
    the three RMSNorms, every channel against the oracle's chain."""
    inp = make_mixer_inputs(CONFIGS["jamba_prefill"])
    check_projected(inp, 256, True, seed=21)
