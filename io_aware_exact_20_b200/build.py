"""Builds the CUDA library ``libfa_b200.so`` in this package directory.

Every translation unit is compiled for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``) with ``-lineinfo``, in parallel,
then linked into one shared object with the CUDA runtime linked statically.
Run ``python -m io_aware_exact_20_b200.build`` or call ``build()``.

``build_variant(name)`` builds a checking copy of the same library under
``_build/<name>/`` (the binding loads it when ``FA_B200_LIBRARY`` names it):
``sanitize`` compiles the host code with AddressSanitizer and
UndefinedBehaviorSanitizer (the process must preload their runtimes), and
``bounds`` compiles the kernels with ``FA_DEBUG_BOUNDS``: every global-memory
access they make outside TMA is checked against the extent of its buffer, and
one out of range is skipped and recorded in the device status word
(FA_ERR_BOUNDS) instead of being made.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)

SOURCES = ["fa_api.cu", "fa_fwd.cu", "fa_bwd.cu", "fa_debug.cu", "fa_noalloc.cu",
           "fa_merge.cu", "fa_proj.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-v"]


def _nvcc():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")
    return nvcc


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "fa.h"))
    files.append(os.path.abspath(__file__))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src: str, log_dir: str, extra=()) -> str:
    obj = os.path.join(log_dir, os.path.splitext(src)[0] + ".o")
    cmd = [_nvcc(), *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c",
           os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(log_dir, src + ".log"), "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr[-4000:]}")
    return obj


def build(verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, BUILD_DIR), SOURCES))
    tmp = LIB_PATH + ".tmp"
    cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr[-4000:]}")
    os.replace(tmp, LIB_PATH)
    if verbose:
        for s in SOURCES:
            with open(os.path.join(BUILD_DIR, s + ".log")) as f:
                sys.stdout.write(f.read())
    return LIB_PATH


def ensure_built() -> str:
    if is_stale():
        build()
    return LIB_PATH


# name: (extra compile flags, extra link flags)
VARIANTS = {
    # (nvcc splits an -Xcompiler argument at commas: one option per flag)
    "sanitize": (["-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined",
                  "-Xcompiler", "-fno-omit-frame-pointer",
                  "-Xcompiler", "-fno-sanitize-recover=undefined"],
                 ["-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined"]),
    "bounds": (["-DFA_DEBUG_BOUNDS"], []),
}


def variant_path(name: str) -> str:
    return os.path.join(BUILD_DIR, name, f"libfa_b200_{name}.so")


def build_variant(name: str) -> str:
    """Builds (if missing or stale) the checking copy `name` of the library."""
    cflags, lflags = VARIANTS[name]
    path = variant_path(name)
    if os.path.exists(path) and all(os.path.getmtime(f) <= os.path.getmtime(path)
                                    for f in _inputs()):
        return path
    out = os.path.dirname(path)
    os.makedirs(out, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, out, cflags), SOURCES))
    tmp = path + ".tmp"
    r = subprocess.run([_nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static", *lflags],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link of {name} failed:\n{r.stderr[-4000:]}")
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB_PATH)
