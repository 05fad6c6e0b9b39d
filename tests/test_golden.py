"""Golden values: the fp64 oracle's outputs on small seeded fp32 cases,
stored in tests/golden/oracle_small.json by tests/golden/make_golden.py (which
calls only the oracle and the seeded input generators).

* CPU: the oracle, rebuilt here, reproduces the stored values (up to a few
  ulps of libm differences between machines): any change to its arithmetic
  shows up here and must come with a regenerated file.
* GPU: the CUDA path meets the stored values within the fp32 tolerance.
"""

import json
import os

import numpy as np
import pytest

import oracle
from workloads import make_decode_inputs_custom, make_mixer_inputs_custom

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_golden_file_covers_forward_and_decode():
    g = _golden()
    assert set(g["forward"]) == {"fwd_structured", "fwd_general"}
    assert set(g["decode"]) == {"decode"}


@pytest.mark.parametrize("name", ["fwd_structured", "fwd_general"])
def test_oracle_reproduces_golden_forward(name):
    case = _golden()["forward"][name]
    inp = make_mixer_inputs_custom(**case["inputs"])
    r = oracle.mixer_fwd(inp["xz"], inp["conv_w"], inp["conv_b"], inp["dt"], inp["dt_bias"], inp["A"],
                         inp["Bm"], inp["Cm"], inp["Dskip"], inp.get("h0"), inp.get("conv_state_in"))
    for key in ("y", "h_last", "conv_state_out"):
        np.testing.assert_allclose(r[key], np.array(case[key]), rtol=1e-12, atol=1e-14, err_msg=key)


def test_oracle_reproduces_golden_decode():
    case = _golden()["decode"]["decode"]
    inp = make_decode_inputs_custom(**case["inputs"])
    r = oracle.state_update(inp["x"], inp["z"], inp["dt"], inp["conv_w"], inp["conv_b"], inp["dt_bias"],
                            inp["Dskip"], inp["A"], inp["Bm"], inp["Cm"], inp["ssm_state"], inp["conv_state"])
    for key in ("y", "ssm_state", "conv_state"):
        np.testing.assert_allclose(r[key], np.array(case[key]), rtol=1e-12, atol=1e-14, err_msg=key)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["fwd_structured", "fwd_general"])
def test_cuda_forward_meets_golden(name):
    from gpu_util import assert_close, gpu_fwd, np64, to_dev

    case = _golden()["forward"][name]
    inp = make_mixer_inputs_custom(**case["inputs"])
    y, h, cs = gpu_fwd(to_dev(inp))
    assert_close(np64(y), np.array(case["y"]), "f32", "y")
    assert_close(np64(h), np.array(case["h_last"]), "f32", "h_last")
    np.testing.assert_array_equal(np64(cs), np.array(case["conv_state_out"]))


@pytest.mark.gpu
def test_cuda_decode_meets_golden():
    import mamba_selective_scan_core_b200 as mm
    from gpu_util import assert_close, decode_args, np64, to_dev

    case = _golden()["decode"]["decode"]
    d = to_dev(make_decode_inputs_custom(**case["inputs"]))
    y = mm.state_update(*decode_args(d), d["ssm_state"], d["conv_state"])
    assert_close(np64(y), np.array(case["y"]), "f32", "y")
    assert_close(np64(d["ssm_state"]), np.array(case["ssm_state"]), "f32", "ssm_state")
    np.testing.assert_array_equal(np64(d["conv_state"]), np.array(case["conv_state"]))
