"""The bounds-checked build (libmxmoe_checks.so: -DMXMOE_CHECKS=1). Every index the kernels
compute from device data -- G / U rows, scale-array offsets and dprob partials in the fused
epilogues, gathered source rows in the quantiser, permuted rows in the routing scatter --
is checked against its buffer's extent; a failed check records MXMOE_ERR_DEVICE_CHECK with
the site's tag and skips the access (no trap, no out-of-bounds access).

Each build runs in its own process (tests/_checked_run.py, library chosen by MXMOE_LIB):
  * on a ragged problem with an empty expert the checked build reports no error and its
    outputs equal the release build's bit for bit -- the checks change no result;
  * with MXMOE_CHECKS_TRIP=1 the dprob-partial checks use half the real extent, so valid
    writes are flagged and skipped: the status word reads MXMOE_ERR_DEVICE_CHECK with that
    site's tag (66) -- the check path works end to end, with every access in bounds."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RUNNER = os.path.join(ROOT, "tests", "_checked_run.py")


def _run(tmp_path, lib, name, extra_env=None):
    out = str(tmp_path / f"{name}.npz")
    env = dict(os.environ, MXMOE_LIB=lib, **(extra_env or {}))
    r = subprocess.run([sys.executable, RUNNER, out], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(out))


@pytest.fixture(scope="module")
def libs():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for tests marked gpu")
    from mxfp8_grouped_gemm_moe_b200 import build as b
    b.build()
    b.build(checks=True)
    return b.LIB, b.LIB_CHECKS


def test_checked_build_matches_release_bit_for_bit(libs, tmp_path):
    rel, chk = libs
    a = _run(tmp_path, rel, "release")
    c = _run(tmp_path, chk, "checked")
    assert str(c["lib"]).endswith("libmxmoe_checks.so")
    assert a["status"][0] == 0 and c["status"][0] == 0, (a["status"], c["status"])
    for n in ("y", "dx", "dW1", "dW2", "dprobs"):
        np.testing.assert_array_equal(c[n], a[n], err_msg=n)


def test_checked_build_flags_and_skips(libs, tmp_path):
    _, chk = libs
    c = _run(tmp_path, chk, "tripped", {"MXMOE_CHECKS_TRIP": "1"})
    assert c["status"][0] == 6 and c["status"][1] == 66, c["status"]   # MXMOE_ERR_DEVICE_CHECK, dprob site
