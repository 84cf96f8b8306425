"""The bounds-checked build (-DDCN_CHECK_BOUNDS), the substitute for a memory
checker on this hardware: adversarial cases (offsets of +-1e4, samples exactly
on the image borders, a one-pixel image, a stride above the image, every
kernel and path) run against libdcncore_checked.so in a child process, which
must report no skipped access and match the oracle."""
import os
import subprocess
import sys

import pytest

from deformable_convolution_core_b200 import build as dcn_build
from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


def test_adversarial_cases_under_the_bounds_checked_build():
    lib = dcn_build.build(checked=True)
    env = dict(os.environ, DCN_CORE_LIBRARY=lib)
    env.pop("DCN_CORE_FORWARD", None)
    env.pop("DCN_CORE_BACKWARD", None)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bounds_checked_cases.py")],
                         env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "all cases passed" in res.stdout
