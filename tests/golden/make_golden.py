"""Write tests/golden/oracle_small.json: the fp64 oracle's outputs on small
seeded cases, for the golden regression tests.

No page prints a worked numeric example for the mixer core (the recurrence is
given only symbolically, in the Jamba hybrid SSM-Transformer lesson, section
"SSM in one page"), so these stored values come from the oracle alone: this
script calls only ``oracle`` and the seeded input generators of
``workloads``, never the CUDA path.  The oracle itself is pinned by
tests/pins.py against closed forms, brute force and library routines; the
golden file guards against unintended changes to it, and gives the CUDA path
fixed expected values to meet.

    python tests/golden/make_golden.py
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import make_decode_inputs_custom, make_mixer_inputs_custom  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")

# (name, generator kwargs): fp32 inputs, so both sides see exactly these values
FORWARD_CASES = [
    ("fwd_structured", dict(batch=2, seqlen=37, d_inner=8, act="f32", seed=1201, h0_std=0.3,
                            conv_state_std=1.0, conv_b_std=0.2, A_mode="structured", dt_std=0.5)),
    ("fwd_general", dict(batch=1, seqlen=45, d_inner=8, act="f32", seed=1202, h0_std=0.0,
                         conv_state_std=0.0, A_mode="general")),
]
DECODE_CASES = [
    ("decode", dict(layers=2, batch=2, d_inner=8, act="f32", seed=1203)),
]


def main():
    out = {"_about": "fp64 oracle outputs on small seeded fp32 cases; written by tests/golden/make_golden.py "
                     "(calls only oracle/ and workloads/). Inputs are regenerated from the seeds.",
           "forward": {}, "decode": {}}
    for name, kw in FORWARD_CASES:
        inp = make_mixer_inputs_custom(**kw)
        r = oracle.mixer_fwd(inp["xz"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["dt_bias"], inp["A"],
                             inp["Bm"], inp["Cm"], inp["Dskip"], inp.get("h0"), inp.get("conv_state_in"))
        out["forward"][name] = {"inputs": kw, "y": r["y"].tolist(), "h_last": r["h_last"].tolist(),
                                "conv_state_out": r["conv_state_out"].tolist()}
    for name, kw in DECODE_CASES:
        inp = make_decode_inputs_custom(**kw)
        r = oracle.state_update(inp["x"], inp["z"], inp["dt"], inp["conv_w"], inp["conv_b"], inp["dt_bias"],
                                inp["Dskip"], inp["A"], inp["Bm"], inp["Cm"], inp["ssm_state"],
                                inp["conv_state"])
        out["decode"][name] = {"inputs": kw, "y": r["y"].tolist(), "ssm_state": r["ssm_state"].tolist(),
                               "conv_state": r["conv_state"].tolist()}
    with open(OUT, "w") as f:
        json.dump(out, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print(OUT, os.path.getsize(OUT), "bytes")


if __name__ == "__main__":
    main()
