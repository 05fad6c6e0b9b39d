"""The checked build of the library (libmamba_mixer_checked.so, compiled with
MM_CHECK_BOUNDS): the forward and decode kernels check every index they form
against its buffer; an access outside it is skipped and reported -- code
MM_ERR_BOUNDS in the call's status and a bit of the device fault word --
instead of faulting.  Each case runs in a child process that loads the
checked build (MAMBA_MIXER_CHECKED=1) and prints one JSON line.

  * On valid calls the checks pass silently: a time-chunked forward (both A
    forms) and a decode match the fp64 oracle, with clean statuses.
  * The test hook MAMBA_MIXER_TEST_BOUNDS_SHRINK=k makes the kernels check y's
    stores against an extent k elements short of the buffer (the buffer itself
    is whole, so nothing outside it is ever touched): those k stores are
    skipped, the call reports MM_ERR_BOUNDS, and every other output is still
    correct.
"""

import json
import os
import subprocess
import sys

import pytest

from mamba_selective_scan_core_b200 import build as mmbuild

pytestmark = pytest.mark.gpu

MM_ERR_BOUNDS = 13
CHILD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "checked_child.py")


def run_child(case, extra_env=None):
    mmbuild.build_checked()
    env = dict(os.environ, MAMBA_MIXER_CHECKED="1")
    env.pop("MAMBA_MIXER_TEST_BOUNDS_SHRINK", None)
    env.update(extra_env or {})
    r = subprocess.run([sys.executable, CHILD, case], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checked_build_valid_calls_match_oracle():
    out = run_child("forward")
    assert out["lib"] == "libmamba_mixer_checked.so"
    assert out["status_structured"] == 0 and out["status_general"] == 0
    assert out["fault"] == 0
    assert all(v <= 1.0 for v in out["ratios"].values()), out["ratios"]


def test_checked_build_reports_a_skipped_store():
    out = run_child("shrink", {"MAMBA_MIXER_TEST_BOUNDS_SHRINK": "2"})
    assert out["status_structured"] == MM_ERR_BOUNDS and out["status_general"] == MM_ERR_BOUNDS
    assert out["fault"] == MM_ERR_BOUNDS
    assert out["tail_nan_structured"] and out["tail_nan_general"]
    assert all(v <= 1.0 for v in out["ratios"].values()), out["ratios"]
