"""The parity suites under the bounds-checking build (FA_DEBUG_BOUNDS): every
global-memory access the kernels make outside TMA is checked against its
buffer's extent, and one out of range would be skipped and recorded as
FA_ERR_BOUNDS in the device status word.  Every parity test below asserts a
zero device status after its calls, so a single out-of-range index anywhere
in the forward, the three backward kernels or the general-layout paths fails
the run, and the results must still match the float64 oracle."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_fwd.py", "tests/test_gpu_bwd.py", "tests/test_gpu_general.py",
          "tests/test_gpu_wide.py", "tests/test_gpu_random_sweep.py"]


def test_parity_suites_under_the_bounds_checking_build(lib):
    from io_aware_exact_20_b200 import build
    env = dict(os.environ, FA_B200_LIBRARY=build.build_variant("bounds"))
    probe = ("import io_aware_exact_20_b200 as fa; "
             "assert fa.library().fa_debug_bounds_checking() == 1; print('bounds build')")
    r = subprocess.run([sys.executable, "-c", probe], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "bounds build" in r.stdout, r.stderr[-2000:]
    r = subprocess.run([sys.executable, "-m", "pytest", *SUITES, "-m", "gpu", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
