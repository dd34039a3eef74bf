"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fa.h declares, and rejects bad arguments before any
launch (no device is touched by a call that fails validation)."""

import ctypes
import os
import re

import pytest

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for want in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string",
                 "fa_last_device_status", "fa_debug_dropout_mask"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    so = lib.library()
    for name in declared_functions():
        assert hasattr(so, name), name
    assert set(declared_functions()) == set(lib.SIGNATURES)


def test_status_strings(lib):
    so = lib.library()
    assert so.fa_status_string(0) == b"ok"
    assert so.fa_status_string(5).startswith(b"workspace")
    assert so.fa_status_string(99) == b"unknown status"


def test_workspace_size_formula(lib):
    so = lib.library()
    # per (b,h): Npad rows x (lse2 + delta + d accumulators) fp32, rounded to 256 B
    assert so.fa_bwd_workspace_size(2, 3, 300, 64) == 2 * 3 * 384 * (8 + 256)
    assert so.fa_bwd_workspace_size(1, 1, 128, 128) == 128 * (8 + 512)
    assert so.fa_bwd_workspace_size(1, 1, 128, 96) == 0
    assert so.fa_bwd_workspace_size(0, 1, 128, 64) == 0


A16 = 1 << 20  # a fake, 16-byte aligned address: validation fails before use


@pytest.mark.parametrize("args,code", [
    (dict(q=0), 1), (dict(k=A16 + 8), 1), (dict(B=0), 1), (dict(N=0), 1),
    (dict(d=96), 2), (dict(scale=0.0), 1), (dict(scale=float("inf")), 1),
    (dict(p=1.0), 1), (dict(p=-0.1), 1), (dict(p=float("nan")), 1),
    (dict(B=300, H=300), 2), (dict(lse=A16 + 2), 1),
    (dict(N=(1 << 23) + 1), 2),                       # N beyond 2^23
    (dict(B=65535, H=1, N=1 << 23), 2),               # 65535 x 65536 tiles > 2^31 - 1
])
def test_fwd_rejects_bad_arguments_without_launching(lib, args, code):
    so = lib.library()
    a = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=1, N=128, d=64, scale=0.125,
             causal=0, seqlens=None, p=0.0, seed=0, bm=None)
    a.update(args)
    got = so.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                    a["scale"], a["causal"], a["seqlens"], a["p"], a["seed"], a["bm"], None)
    assert got == code


def test_bwd_rejects_missing_or_small_workspace(lib):
    so = lib.library()
    need = so.fa_bwd_workspace_size(1, 1, 128, 64)
    call = lambda ws, n: so.fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, 1, 1, 128, 64,
                                   0.125, 0, None, 0.0, 0, None, ws, n, None)
    assert call(None, need) == 5
    assert call(A16, need - 1) == 5
    assert call(A16 + 16, need) == 5  # not 256-byte aligned
    assert so.fa_bwd(A16, A16, A16, A16, A16, None, A16, A16, A16, 1, 1, 128, 64, 0.125, 0,
                     None, 0.0, 0, None, A16, need, None) == 1


def test_product_path_has_no_cpu_fallback(lib):
    """Without a CUDA device the torch-level wrapper refuses CPU tensors."""
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lib.forward(q, q, q)
