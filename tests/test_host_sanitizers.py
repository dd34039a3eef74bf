"""The library's host code under AddressSanitizer and UndefinedBehaviorSanitizer,
on the CPU: the `sanitize` build (host code instrumented, kernels unchanged)
is loaded into a Python process that preloads both runtimes, and the C-ABI
tests run there.  Every call in them fails validation before any launch, so
this exercises the argument checks, the workspace sizing, the status strings
and the general-layout descriptor resolution (tensor-map encoding needs the
driver and runs under the GPU tests).  Any sanitizer report aborts the
process (halt_on_error / -fno-sanitize-recover)."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name):
    gcc = shutil.which("gcc")
    if gcc is None:
        return None
    r = subprocess.run([gcc, f"-print-file-name={name}"], capture_output=True, text=True)
    path = os.path.realpath(r.stdout.strip())
    return path if os.path.isabs(path) and os.path.exists(path) else None


def _env(lib_path):
    env = dict(os.environ)
    env["LD_PRELOAD"] = " ".join([_runtime("libasan.so"), _runtime("libubsan.so")])
    env["ASAN_OPTIONS"] = "detect_leaks=0:halt_on_error=1:protect_shadow_gap=0"
    env["UBSAN_OPTIONS"] = "halt_on_error=1:print_stacktrace=1"
    env["FA_B200_LIBRARY"] = lib_path
    return env


def test_abi_calls_under_asan_and_ubsan(lib):
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc is needed to build the sanitizer variant")
    if _runtime("libasan.so") is None or _runtime("libubsan.so") is None:
        pytest.skip("the gcc sanitizer runtimes are not installed")
    from io_aware_exact_20_b200 import build
    path = build.build_variant("sanitize")
    env = _env(path)
    # the instrumented library and both runtimes are the ones in the process
    probe = ("import io_aware_exact_20_b200 as fa; fa.library(); "
             "maps = open('/proc/self/maps').read(); "
             "assert 'libfa_b200_sanitize.so' in maps and 'libasan' in maps "
             "and 'libubsan' in maps, 'not loaded'; print('loaded')")
    r = subprocess.run([sys.executable, "-c", probe], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "loaded" in r.stdout, r.stderr[-3000:]
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_abi.py", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    report = r.stdout[-3000:] + r.stderr[-3000:]
    assert r.returncode == 0, report
    assert "AddressSanitizer" not in r.stderr and "runtime error" not in r.stderr, report
