"""Child process of tests/test_checked_gpu.py: loads the checked build of the
library (MAMBA_MIXER_CHECKED=1 is set by the parent before this process
imports the package) and runs one case, printing one JSON line.

Cases:
  forward  -- a time-chunked bf16 forward (structured and general A) and a
              28-row decode, against the fp64 oracle; statuses must be clean.
  shrink   -- the same forward with MAMBA_MIXER_TEST_BOUNDS_SHRINK set: the
              kernels check y's stores against an extent short of the last
              elements (the buffer itself is whole), skip those stores and
              report MM_ERR_BOUNDS; everything else is still written.
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import mamba_selective_scan_core_b200 as mm  # noqa: E402
from gpu_util import THREADS, assert_close, np64, oracle_fwd, to_dev  # noqa: E402
import oracle  # noqa: E402
from workloads import make_decode_inputs_custom, make_mixer_inputs_custom  # noqa: E402


def fwd(d, ws, y=None):
    return mm.mixer_fwd(d["xz"], d["conv_w"], d["conv_b"], d["dt"], d["dt_bias"], d["A"], d["Bm"], d["Cm"],
                        d["Dskip"], d["h0"], d["conv_state_in"], y=y, workspace=ws)


def main(case):
    assert mm.library_path().endswith("libmamba_mixer_checked.so")
    out = {"lib": os.path.basename(mm.library_path())}
    mm.fault_status(reset=True)
    B, L, D = 2, 600, 512
    ratios = {}
    for A_mode in ("structured", "general"):
        inp = make_mixer_inputs_custom(B, L, D, act="bf16", seed=311, h0_std=0.4, conv_state_std=1.0,
                                       A_mode=A_mode)
        d = to_dev(inp)
        ws = torch.zeros(mm.workspace_size(B, L, D), dtype=torch.uint8, device="cuda")
        # y starts as NaN: in the shrink case the skipped stores leave their elements NaN
        y0 = torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        y, h, cs = fwd(d, ws, y=y0)
        torch.cuda.synchronize()
        out[f"status_{A_mode}"] = mm.check_status(ws)
        ref = oracle_fwd(inp)
        gy = np64(y)
        if case == "shrink":
            tail = gy.reshape(-1)[-int(os.environ["MAMBA_MIXER_TEST_BOUNDS_SHRINK"]):]
            out[f"tail_nan_{A_mode}"] = bool(np.isnan(tail).all())
            body = gy.reshape(-1)[:-len(tail)]
            ratios[f"y_{A_mode}"] = assert_close(body, ref["y"].reshape(-1)[:-len(tail)], "bf16", "y",
                                                 stored_bf16=True)
        else:
            ratios[f"y_{A_mode}"] = assert_close(gy, ref["y"], "bf16", "y", stored_bf16=True)
        ratios[f"h_{A_mode}"] = assert_close(np64(h), ref["h_last"], "bf16", "h_last")
    if case == "forward":
        dinp = make_decode_inputs_custom(4, 7, 512, act="bf16", seed=312)
        dd = to_dev(dinp)
        yd = mm.state_update(dd["x"], dd["z"], dd["dt"], dd["conv_w"], dd["conv_b"], dd["dt_bias"], dd["Dskip"],
                             dd["A"], dd["Bm"], dd["Cm"], dd["ssm_state"], dd["conv_state"])
        torch.cuda.synchronize()
        rd = oracle.state_update(dinp["x"], dinp["z"], dinp["dt"], dinp["conv_w"], dinp["conv_b"],
                                 dinp["dt_bias"], dinp["Dskip"], dinp["A"], dinp["Bm"], dinp["Cm"],
                                 dinp["ssm_state"], dinp["conv_state"], threads=THREADS)
        ratios["decode_y"] = assert_close(np64(yd), rd["y"], "bf16", "decode y", stored_bf16=True)
        ratios["decode_state"] = assert_close(np64(dd["ssm_state"]), rd["ssm_state"], "bf16", "decode state")
    out["ratios"] = ratios
    out["fault"] = mm.fault_status(reset=True)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main(sys.argv[1])
