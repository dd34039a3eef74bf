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
    assert so.fa_status_string(6).startswith(b"a kernel index was out of bounds")
    # grouped K / V heads with few units: split parts need fp32 dK / dV accumulators
    st, sk = lib.Strides(3 * 256 * 64, 256 * 64, 64), lib.Strides(1 * 384 * 64, 384 * 64, 64)
    a = _desc(lib, heads_kv=1, q=st, o=st, dout=st, dq=st, k=sk, v=sk, dk=sk, dv=sk)
    base = 2 * 3 * 256 * (8 + 256)
    lib.set_gqa_split(1)
    try:
        assert so.fa_bwd_ex_workspace_size(ctypes.byref(a)) == base
        lib.set_gqa_split(3)   # three parts of the group of 3: dK / dV slices of 2 x 384 x 64 each
        assert so.fa_bwd_ex_workspace_size(ctypes.byref(a)) == base + 3 * 2 * 4 * 2 * 384 * 64
        lib.set_gqa_split(2)   # does not divide the group: the automatic choice (3 here)
        assert so.fa_bwd_ex_workspace_size(ctypes.byref(a)) == base + 3 * 2 * 4 * 2 * 384 * 64
    finally:
        lib.set_gqa_split(0)
    # the default library is the production build (no bounds checks)
    if not os.environ.get("FA_B200_LIBRARY"):
        assert so.fa_debug_bounds_checking() == 0
    assert so.fa_status_string(0) == b"ok"
    assert so.fa_status_string(5).startswith(b"workspace")
    assert so.fa_status_string(99) == b"unknown status"


def test_workspace_size_formula(lib):
    so = lib.library()
    # per (b,h): Npad rows x (lse2 + delta + d accumulators) fp32, rounded to 256 B
    assert so.fa_bwd_workspace_size(2, 3, 300, 64) == 2 * 3 * 384 * (8 + 256)
    assert so.fa_bwd_workspace_size(1, 1, 128, 128) == 128 * (8 + 512)
    # d = 32 and 96 run the 64- and 128-wide kernels: accumulators of that width
    assert so.fa_bwd_workspace_size(1, 1, 128, 96) == 128 * (8 + 512)
    assert so.fa_bwd_workspace_size(1, 1, 128, 32) == 128 * (8 + 256)
    assert so.fa_bwd_workspace_size(1, 1, 128, 80) == 0
    assert so.fa_bwd_workspace_size(0, 1, 128, 64) == 0


A16 = 1 << 20  # a fake, 16-byte aligned address: validation fails before use


@pytest.mark.parametrize("args,code", [
    (dict(q=0), 1), (dict(k=A16 + 8), 1), (dict(B=0), 1), (dict(N=0), 1),
    (dict(d=80), 2), (dict(d=160), 2), (dict(d=512), 2), (dict(scale=0.0), 1),
    (dict(scale=float("inf")), 1),
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


def _desc(lib, **kw):
    a = lib.AttentionDesc()
    a.batch, a.heads, a.head_dim, a.seqlen_q, a.seqlen_k = 2, 3, 64, 256, 384
    a.softmax_scale = 0.125
    st = lib.Strides(3 * 256 * 64, 256 * 64, 64)
    sk = lib.Strides(3 * 384 * 64, 384 * 64, 64)
    for name in ("q", "o", "dout", "dq"):
        setattr(a, name, st)
    for name in ("k", "v", "dk", "dv"):
        setattr(a, name, sk)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("change,code", [
    (dict(), None),                                        # valid: workspace size > 0
    (dict(head_dim=80), 2), (dict(head_dim=160), 2), (dict(head_dim=512), 2),
    (dict(batch=0), 1), (dict(seqlen_k=0), 1), (dict(dropout_p=1.0), 1),
    (dict(cu_seqlens_q=A16), 1),                           # packed needs both offsets
    (dict(cu_seqlens_q=A16, cu_seqlens_k=A16), 1),          # ... and total_q, total_k >= 1
    (dict(cu_seqlens_q=A16 + 2, cu_seqlens_k=A16, total_q=5, total_k=5), 1),
    (dict(q=(3 * 256 * 64, 256 * 64, 60)), 1),              # row stride not a multiple of 8
    (dict(k=(3 * 384 * 64, 0, 64)), 1),                     # heads sharing memory
    (dict(o=(0, 256 * 64, 64)), 1),                         # batch entries sharing memory
    (dict(seqlen_q=(1 << 23) + 1), 2),
    (dict(dropout_row0=128, dropout_key0=64), None),       # valid dropout positions
    (dict(dropout_key0=4), 1),                             # not a multiple of 8
    (dict(dropout_row0=-1), 1), (dict(dropout_key0=-8), 1),
    (dict(dropout_row0=(1 << 31) - 256), 1),               # row0 + seqlen_q past 2^31 - 1
    (dict(dropout_key0=(1 << 40)), 1),
    (dict(heads_kv=1), None), (dict(heads_kv=3), None),   # grouped K / V heads (3 query heads)
    (dict(heads_kv=2), 1), (dict(heads_kv=4), 1), (dict(heads_kv=-1), 1),
    (dict(batch=1, heads=32768, heads_kv=1), 2),           # group too large for the walk
])
def test_general_entry_points_validate_before_launching(lib, change, code):
    so = lib.library()
    kw = {k: (lib.Strides(*v) if isinstance(v, tuple) else v) for k, v in change.items()}
    a = _desc(lib, **kw)
    ws = so.fa_bwd_ex_workspace_size(ctypes.byref(a))
    if code is None:
        # padded layout: B * H * ceil(N_q / 128) * 128 rows of 8 + 4 * 64 bytes,
        # and with grouped K / V heads the split units' dK / dV accumulators
        # (a valid description is never launched here: the addresses are fake)
        if change.get("heads_kv", 3) == 3:
            assert ws == 2 * 3 * 256 * (8 + 256)
        else:
            assert ws > 2 * 3 * 256 * (8 + 256)
        return
    assert ws == 0
    assert so.fa_fwd_ex(ctypes.byref(a), A16, A16, A16, A16, A16, None) == code
    assert so.fa_bwd_ex(ctypes.byref(a), A16, A16, A16, A16, A16, A16, A16, A16, A16, A16,
                        1 << 30, None) == code


def test_general_workspace_size_of_packed_layout(lib):
    """Packed: H * (ceil(total_q / 128) * 128 + 256 B) rows, each 8 + 4 D bytes."""
    so = lib.library()
    a = _desc(lib, cu_seqlens_q=A16, cu_seqlens_k=A16, total_q=1000, total_k=900, head_dim=96)
    for name in ("q", "k", "v", "o", "dout", "dq", "dk", "dv"):
        setattr(a, name, lib.Strides(0, 96, 3 * 96))
    rows = 3 * (1024 + 256 * 2)
    assert so.fa_bwd_ex_workspace_size(ctypes.byref(a)) == (rows * (8 + 512) + 255) // 256 * 256
    assert so.fa_fwd_ex(None, A16, A16, A16, A16, A16, None) == 1


def test_qkv_projection_rejects_bad_shapes(lib):
    so = lib.library()
    a = A16
    assert so.fa_qkv_projection(a, a, None, a, a, a, 1, 128, 1, 64, 64, None) == 2  # H d = 64
    assert so.fa_qkv_projection(a, a, None, a, a, a, 1, 128, 2, 96, 64, None) == 2  # d = 96
    assert so.fa_qkv_projection(a, a, None, a, a, a, 1, 128, 2, 64, 60, None) == 1  # d_model % 8
    assert so.fa_qkv_projection(a + 8, a, None, a, a, a, 1, 128, 2, 64, 64, None) == 1
    assert so.fa_qkv_projection(a, a, a + 2, a, a, a, 1, 128, 2, 64, 64, None) == 1  # bias align


def test_general_binding_rejects_host_tensors_and_bad_layouts(lib):
    """The general-layout binding checks its tensors before it marshals a call:
    host tensors, an unknown layout and a tensor of the wrong rank raise."""
    import torch
    q = torch.zeros((1, 2, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="device of q"):
        lib.forward_general(q, q, q)
    with pytest.raises(ValueError, match="unknown layout"):
        lib.forward_general(q, q, q, layout="sbhd")
    with pytest.raises(ValueError, match="3-D tensor"):
        lib.forward_general(q, q, q, layout="thd")
    with pytest.raises(ValueError, match="device of q"):
        lib.backward_general(q, q, q, q, torch.zeros((1, 2, 128)), q)


def test_backward_at_width_256(lib):
    """d = 192 / 256 run the 256-wide backward (two CTAs per key tile): the
    workspace holds 256 accumulators per row, and a grid that fits one CTA
    per key tile but not two is refused (FA_ERR_UNSUPPORTED) before any
    launch, where d = 128 at the same size passes that check and stops at the
    workspace (FA_ERR_WORKSPACE), also before any launch."""
    so = lib.library()
    assert so.fa_bwd_workspace_size(1, 1, 128, 256) == 128 * (8 + 1024)
    assert so.fa_bwd_workspace_size(1, 1, 128, 192) == 128 * (8 + 1024)
    assert so.fa_bwd_workspace_size(2, 3, 300, 256) == 2 * 3 * 384 * (8 + 1024)
    st, sk = lib.Strides(3 * 256 * 256, 256 * 256, 256), lib.Strides(3 * 384 * 256, 384 * 256, 256)
    a = _desc(lib, head_dim=256, q=st, o=st, dout=st, dq=st, k=sk, v=sk, dk=sk, dv=sk)
    assert so.fa_bwd_ex_workspace_size(ctypes.byref(a)) == a.batch * a.heads * 256 * (8 + 1024)
    # 65535 x 32768 key tiles < 2^31 - 1 < twice that
    big = (65535, 1, 1 << 22)
    for d, code in ((256, 2), (192, 2), (128, 5)):
        assert so.fa_bwd(A16, A16, A16, A16, A16, A16, A16, A16, A16, *big, d, 0.1, 0, None,
                         0.0, 0, None, A16, 1 << 30, None) == code, d

def test_merge_partial_head_dims(lib):
    """fa_merge_partial takes every head dim of the attention kernels (32 to
    256) and refuses others before any launch; zero rows launch nothing."""
    so = lib.library()
    for d in (32, 64, 96, 128, 192, 256):
        assert so.fa_merge_partial(A16, A16, A16, A16, 0, d, None) == 0, d
    for d in (16, 80, 160, 320, 512):
        assert so.fa_merge_partial(A16, A16, A16, A16, 5, d, None) == 2, d


def test_nvtx_ranges_wrap_the_entry_points(lib, monkeypatch):
    """With NVTX on, an entry point runs inside a range named after it, popped
    even when the call raises; off (the default), no range is pushed."""
    import torch
    calls = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: calls.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: calls.append(("pop",)))
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)  # host tensors: refused before any launch
    lib.set_nvtx(True)
    try:
        with pytest.raises(ValueError):
            lib.forward(q, q, q)
        with pytest.raises(ValueError):
            lib.forward_general(q, q, q)
    finally:
        lib.set_nvtx(False)
    assert calls == [("push", "fa.forward"), ("pop",), ("push", "fa.forward_general"), ("pop",)]
    calls.clear()
    with pytest.raises(ValueError):
        lib.forward(q, q, q)
    assert calls == []


def test_gqa_split_is_chosen_from_the_units(lib):
    """Grouped K / V heads: a backward unit is split into the fewest parts
    (a divisor of the group) giving about four units per SM (592); the parts'
    dK / dV slices show in the workspace size."""
    so = lib.library()
    N, d = 16384, 128

    def ws(B, H, Hkv):
        st, sk = lib.Strides(H * N * d, N * d, d), lib.Strides(Hkv * N * d, N * d, d)
        a = _desc(lib, batch=B, heads=H, heads_kv=Hkv, head_dim=d, seqlen_q=N, seqlen_k=N,
                  q=st, o=st, dout=st, dq=st, k=sk, v=sk, dk=sk, dv=sk)
        return so.fa_bwd_ex_workspace_size(ctypes.byref(a))

    def base(B, H):
        return B * H * N * (8 + 4 * d)

    acc = lambda S, B, Hkv: S * 2 * 4 * B * Hkv * N * d  # noqa: E731  dK / dV slice per part
    assert ws(1, 16, 16) == base(1, 16)                  # no grouping: no split
    assert ws(1, 16, 1) == base(1, 16) + acc(8, 1, 1)    # 128 units: split into 8 parts
    assert ws(1, 16, 4) == base(1, 16) + acc(2, 1, 4)    # 512 units: 2 parts
    assert ws(2, 16, 4) == base(2, 16)                   # 1024 units: whole groups
