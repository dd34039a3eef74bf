"""Exact (FlashAttention-style) softmax attention for B200 / sm_100a.

A thin Python binding over the C ABI declared in ``include/fa.h`` and
implemented by ``libfa_b200.so`` (built in this directory by
``io_aware_exact_20_b200.build``).  The binding only marshals arguments:
PyTorch supplies device memory and the current stream; every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or the tensors are not on a CUDA device, the call raises.

Entry points mirror the C names: ``fa_fwd`` / ``fa_bwd`` take raw pointers
exactly like the C functions; ``forward`` / ``backward`` wrap them for torch
tensors of layout [B, H, N, d].
"""

from __future__ import annotations

import ctypes
import functools
import os

from .build import LIB_PATH

__all__ = [
    "FaError", "library", "forward", "backward", "backward_phases", "bwd_workspace_size",
    "forward_general", "backward_general", "general_workspace_size",
    "merge_partial", "accumulate_bf16", "convert_f32_bf16", "qkv_projection",
    "dropout_mask", "last_device_status", "set_wait_timeout_ns", "set_block_mask_bitmap",
    "wait_timeout_probe", "set_nvtx", "STATUS",
]

STATUS = {
    0: "FA_OK",
    1: "FA_ERR_INVALID_ARG",
    2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_CUDA",
    4: "FA_ERR_TIMEOUT",
    5: "FA_ERR_WORKSPACE",
    6: "FA_ERR_BOUNDS",
}


# NVTX ranges around the entry points below, for timeline profilers: off unless
# FA_NVTX is set to a non-zero value or set_nvtx(True) is called.
_NVTX = os.environ.get("FA_NVTX", "0") not in ("", "0")


def set_nvtx(enabled):
    """Marks each call of the entry points with an NVTX range ("fa.forward",
    "fa.backward", ...) when enabled."""
    global _NVTX
    _NVTX = bool(enabled)


def _nvtx(name):
    def deco(fn):
        @functools.wraps(fn)
        def wrapped(*args, **kwargs):
            if not _NVTX:
                return fn(*args, **kwargs)
            import torch
            torch.cuda.nvtx.range_push(name)
            try:
                return fn(*args, **kwargs)
            finally:
                torch.cuda.nvtx.range_pop()
        return wrapped
    return deco


class FaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_LIB = None
_vp, _i, _f, _u64, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                          ctypes.c_uint64, ctypes.c_size_t)

class Strides(ctypes.Structure):
    """fa_strides_t: element strides of a [batch, head, row, d] view."""
    _fields_ = [("batch", ctypes.c_int64), ("head", ctypes.c_int64), ("row", ctypes.c_int64)]


class AttentionDesc(ctypes.Structure):
    """fa_attention_desc_t (include/fa.h), field for field."""
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("seqlen_q", ctypes.c_int), ("seqlen_k", ctypes.c_int),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("total_q", ctypes.c_int), ("total_k", ctypes.c_int),
        ("seqlens_k", ctypes.c_void_p),
        ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int),
        ("dropout_p", ctypes.c_float), ("seed", ctypes.c_uint64),
        ("block_mask", ctypes.c_void_p),
        ("q", Strides), ("k", Strides), ("v", Strides), ("o", Strides), ("dout", Strides),
        ("dq", Strides), ("dk", Strides), ("dv", Strides),
        ("dropout_row0", ctypes.c_int64), ("dropout_key0", ctypes.c_int64),
        ("heads_kv", ctypes.c_int),
    ]


_DP = ctypes.POINTER(AttentionDesc)

# name -> (restype, argtypes); must match include/fa.h
SIGNATURES = {
    "fa_fwd_ex": (_i, [_DP, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fa_bwd_ex_workspace_size": (_sz, [_DP]),
    "fa_bwd_ex": (_i, [_DP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fa_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _f, _u64, _vp, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp,
                    _f, _u64, _vp, _vp, _sz, _vp]),
    "fa_bwd_prepare": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "fa_bwd_main": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _f, _u64,
                         _vp, _vp, _sz, _vp]),
    "fa_bwd_finish": (_i, [_vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "fa_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                            _vp, _f, _u64, _vp, _vp]),
    "fa_qkv_projection": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "fa_merge_partial": (_i, [_vp, _vp, _vp, _vp, ctypes.c_int64, _i, _vp]),
    "fa_accumulate_bf16": (_i, [_vp, _vp, ctypes.c_int64, _vp]),
    "fa_convert_f32_bf16": (_i, [_vp, _vp, ctypes.c_int64, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_last_device_status": (_i, [_vp]),
    "fa_set_wait_timeout_ns": (None, [_u64]),
    "fa_debug_dropout_mask": (_i, [_vp, _i, _i, _i, _f, _u64, _vp]),
    "fa_debug_wait_timeout": (_i, [_vp]),
    "fa_debug_set_block_mask_bitmap": (None, [_i]),
    "fa_debug_bounds_checking": (_i, []),
    "fa_debug_set_gqa_split": (None, [_i]),
}


def library():
    """The loaded C library (raises if it has not been built).  The
    environment variable FA_B200_LIBRARY may name another build of it (one of
    the checking variants of `build.build_variant`)."""
    global _LIB
    if _LIB is None:
        path = os.environ.get("FA_B200_LIBRARY") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m io_aware_exact_20_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _check(code, where):
    if code != 0:
        raise FaError(code, where)


def _stream_ptr(device):
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_qkv(*ts):
    import torch
    ref = ts[0]
    if ref.dim() != 4:
        raise ValueError("tensors must be [B, H, N, d]")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bfloat16")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")
        if t.shape != ref.shape or t.device != ref.device:
            raise ValueError("q, k, v (and o, dout) must share shape and device")


def _masks(seqlens, block_mask, device):
    import torch
    sl = None
    if seqlens is not None:
        sl = torch.as_tensor(seqlens, dtype=torch.int32, device=device).contiguous()
    bm = None
    if block_mask is not None:
        bm = torch.as_tensor(block_mask, dtype=torch.uint8, device=device).contiguous()
    return sl, bm


@_nvtx("fa.forward")
def forward(q, k, v, scale=None, causal=False, seqlens=None, dropout_p=0.0, seed=0,
            block_mask=None, out=None, lse=None):
    """O, LSE = attention(q, k, v) for bf16 CUDA tensors [B, H, N, d]."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    sl, bm = _masks(seqlens, block_mask, q.device)
    code = library().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                            float(scale), int(bool(causal)), _ptr(sl), float(dropout_p),
                            int(seed) & 0xFFFFFFFFFFFFFFFF, _ptr(bm), _stream_ptr(q.device))
    _check(code, "fa_fwd")
    return out, lse


def bwd_workspace_size(B, H, N, d):
    return int(library().fa_bwd_workspace_size(B, H, N, d))


@_nvtx("fa.backward")
def backward(q, k, v, o, lse, dout, scale=None, causal=False, seqlens=None, dropout_p=0.0,
             seed=0, block_mask=None, workspace=None, dq=None, dk=None, dv=None):
    """dQ, dK, dV of attention for bf16 CUDA tensors [B, H, N, d]."""
    import torch
    _check_qkv(q, k, v, o, dout)
    B, H, N, d = q.shape
    if scale is None:
        scale = d ** -0.5
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    sl, bm = _masks(seqlens, block_mask, q.device)
    code = library().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                            _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                            int(bool(causal)), _ptr(sl), float(dropout_p),
                            int(seed) & 0xFFFFFFFFFFFFFFFF, _ptr(bm), _ptr(workspace),
                            workspace.numel() * workspace.element_size(),
                            _stream_ptr(q.device))
    _check(code, "fa_bwd")
    return dq, dk, dv


@_nvtx("fa.backward_phases")
def backward_phases(q, k, v, o, lse, dout, scale=None, causal=False, seqlens=None,
                    dropout_p=0.0, seed=0, block_mask=None, workspace=None, dq=None, dk=None,
                    dv=None):
    """The three launches of ``backward`` as three callables (prepare, main,
    finish) bound to the same buffers, plus the outputs: lets a caller put
    events or other work between them."""
    import torch
    _check_qkv(q, k, v, o, dout)
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, H, N, d), dtype=torch.uint8,
                                device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    sl, bm = _masks(seqlens, block_mask, q.device)
    ws, nws = _ptr(workspace), workspace.numel() * workspace.element_size()
    lib = library()
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF

    def prepare():
        _check(lib.fa_bwd_prepare(_ptr(o), _ptr(lse), _ptr(dout), B, H, N, d, ws, nws,
                                  _stream_ptr(q.device)), "fa_bwd_prepare")

    def main():
        _check(lib.fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv), B, H,
                               N, d, float(scale), int(bool(causal)), _ptr(sl),
                               float(dropout_p), seed, _ptr(bm), ws, nws,
                               _stream_ptr(q.device)), "fa_bwd_main")

    def finish():
        _check(lib.fa_bwd_finish(_ptr(dq), B, H, N, d, float(scale), ws, nws,
                                 _stream_ptr(q.device)), "fa_bwd_finish")

    return (prepare, main, finish), (dq, dk, dv), (sl, bm, workspace)


def dropout_mask(B, H, N, dropout_p, seed, device="cuda"):
    """Keep bits [B, H, N, N] (uint8) from the library's device generator."""
    import torch
    keep = torch.empty((B, H, N, N), dtype=torch.uint8, device=device)
    code = library().fa_debug_dropout_mask(_ptr(keep), B, H, N, float(dropout_p),
                                           int(seed) & 0xFFFFFFFFFFFFFFFF,
                                           _stream_ptr(keep.device))
    _check(code, "fa_debug_dropout_mask")
    return keep


def last_device_status(device=None):
    import torch
    return library().fa_last_device_status(_stream_ptr(device or torch.cuda.current_device()))


def set_wait_timeout_ns(ns):
    library().fa_set_wait_timeout_ns(int(ns))


def set_gqa_split(parts):
    """Test support: parts per backward unit under grouped K / V heads (0 =
    chosen from the problem's size; ignored unless it divides the group)."""
    library().fa_debug_set_gqa_split(int(parts))


def set_block_mask_bitmap(enabled):
    """Test support: False makes later launches walk block masks byte by byte."""
    library().fa_debug_set_block_mask_bitmap(1 if enabled else 0)


def wait_timeout_probe(device=None):
    import torch
    _check(library().fa_debug_wait_timeout(_stream_ptr(device or torch.cuda.current_device())),
           "fa_debug_wait_timeout")


# ---------------------------------------------------------------------------
# general layouts: [B, H, N, d] / [B, N, H, d] with any strides, packed
# variable-length batches [T, H, d], N_q != N_k, d in {32, 64, 96, 128}
# ---------------------------------------------------------------------------

def _strides(t, layout):
    if t is None:
        return Strides(0, 0, 0)
    if t.stride(-1) != 1:
        raise ValueError("the head dimension must be contiguous")
    if layout == "bhsd":
        return Strides(t.stride(0), t.stride(1), t.stride(2))
    if layout == "bshd":
        return Strides(t.stride(0), t.stride(2), t.stride(1))
    if layout == "thd":
        return Strides(0, t.stride(1), t.stride(0))
    raise ValueError(f"unknown layout {layout!r}")


def _dims(t, layout):
    """(batch, rows, heads, d) of a tensor in the given layout."""
    if layout == "bhsd":
        return t.shape[0], t.shape[2], t.shape[1], t.shape[3]
    if layout == "bshd":
        return t.shape[0], t.shape[1], t.shape[2], t.shape[3]
    return None, t.shape[0], t.shape[1], t.shape[2]


# the tensors of a call that have Q's shape; the others (k, v, dk, dv) have K's
_Q_SIDE = ("q", "o", "dout", "dq")


def _desc(q, k, layout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, scale, causal,
          seqlens_k, dropout_p, seed, block_mask, tensors, dropout_pos=(0, 0)):
    import torch
    if layout not in ("bhsd", "bshd", "thd"):
        raise ValueError(f"unknown layout {layout!r}")
    want_dim = 3 if layout == "thd" else 4
    for name, t in tensors.items():
        if t.dim() != want_dim:
            raise ValueError(f"{name}: a {want_dim}-D tensor is expected for layout {layout!r}")
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.device != q.device:
            raise ValueError(f"{name}: bfloat16 on the device of q is expected")
        ref = q if name in _Q_SIDE else k
        if t.shape != ref.shape:
            raise ValueError(f"{name}: shape {tuple(t.shape)} differs from "
                             f"{'q' if name in _Q_SIDE else 'k'} {tuple(ref.shape)}")
    Bq, Nq, H, d = _dims(q, layout)
    Bk, Nk, Hk, dk = _dims(k, layout)
    if d != dk or Hk < 1 or H % Hk:
        raise ValueError("q and k must have the same head dim, and q's heads must be a multiple "
                         "of k's (grouped-query attention)")
    keep = []
    a = AttentionDesc()
    a.heads, a.head_dim, a.heads_kv = H, d, Hk
    if layout == "thd":
        if cu_seqlens_q is None or cu_seqlens_k is None:
            raise ValueError("the packed layout needs cu_seqlens_q and cu_seqlens_k")
        cq = torch.as_tensor(cu_seqlens_q, dtype=torch.int32, device=q.device).contiguous()
        ck = torch.as_tensor(cu_seqlens_k, dtype=torch.int32, device=q.device).contiguous()
        keep += [cq, ck]
        a.batch = cq.numel() - 1
        a.cu_seqlens_q, a.cu_seqlens_k = cq.data_ptr(), ck.data_ptr()
        a.total_q, a.total_k = Nq, Nk
        if max_seqlen_q is None or max_seqlen_k is None:
            raise ValueError("the packed layout needs max_seqlen_q and max_seqlen_k")
        a.seqlen_q, a.seqlen_k = int(max_seqlen_q), int(max_seqlen_k)
    else:
        if Bq != Bk:
            raise ValueError("q and k must have the same batch size")
        a.batch, a.seqlen_q, a.seqlen_k = Bq, Nq, Nk
    sl, bm = _masks(seqlens_k, block_mask, q.device)
    keep += [sl, bm]
    a.seqlens_k = _ptr(sl)
    a.block_mask = _ptr(bm)
    a.softmax_scale = float(d ** -0.5 if scale is None else scale)
    a.causal = int(bool(causal))
    a.dropout_p = float(dropout_p)
    a.seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    a.dropout_row0, a.dropout_key0 = (int(x) for x in dropout_pos)
    for name, t in tensors.items():
        setattr(a, name, _strides(t, layout))
    return a, keep


@_nvtx("fa.forward_general")
def forward_general(q, k, v, *, layout="bhsd", cu_seqlens_q=None, cu_seqlens_k=None,
                    max_seqlen_q=None, max_seqlen_k=None, scale=None, causal=False,
                    seqlens_k=None, dropout_p=0.0, seed=0, block_mask=None, out=None, lse=None,
                    dropout_row0=0, dropout_key0=0):
    """O, LSE for a general layout (fa_fwd_ex).

    layout "bhsd": q [B, H, N_q, d], k / v [B, H, N_k, d]; "bshd": q [B, N_q, H, d],
    k / v [B, N_k, H, d]; "thd": packed q [T_q, H, d], k / v [T_k, H, d] with int32
    offsets cu_seqlens_q / cu_seqlens_k ([B + 1]) and the longest lengths.  Any
    strides with d contiguous (multiples of 8 elements).  The causal mask is
    bottom-right aligned per sequence.  LSE: [B, H, N_q] or [H, T_q] (packed).
    k and v may have fewer heads than q, a divisor of them (grouped-query
    attention: query head h reads K / V head h // (H / H_kv)).
    dropout_row0 / dropout_key0: positions of the call's first query row and
    first key in the sequence the dropout bits are keyed by (a block of a
    longer sequence); the key position a multiple of 8.
    """
    import torch
    if out is None:
        out = torch.empty_like(q)
    a, keep = _desc(q, k, layout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, scale,
                    causal, seqlens_k, dropout_p, seed, block_mask,
                    dict(q=q, k=k, v=v, o=out), (dropout_row0, dropout_key0))
    if lse is None:
        lse = torch.empty(_lse_shape(q, layout), dtype=torch.float32, device=q.device)
    _check_lse(lse, q, layout)
    code = library().fa_fwd_ex(ctypes.byref(a), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                               _stream_ptr(q.device))
    _check(code, "fa_fwd_ex")
    del keep
    return out, lse


def _lse_shape(q, layout):
    """[B, H, N_q] (padded layouts) or [H, T_q] (packed)."""
    if layout == "thd":
        return (q.shape[1], q.shape[0])
    B, Nq, H, _ = _dims(q, layout)
    return (B, H, Nq)


def _check_lse(lse, q, layout):
    import torch
    shape = _lse_shape(q, layout)
    if (lse.dtype != torch.float32 or lse.device != q.device or tuple(lse.shape) != shape
            or not lse.is_contiguous()):
        raise ValueError(f"lse: contiguous float32 {shape} on the device of q is expected")


def general_workspace_size(q, k, **kw):
    """Workspace bytes of backward_general for these tensors and options."""
    a, keep = _desc(q, k, kw.get("layout", "bhsd"), kw.get("cu_seqlens_q"),
                    kw.get("cu_seqlens_k"), kw.get("max_seqlen_q"), kw.get("max_seqlen_k"),
                    kw.get("scale"), kw.get("causal", False), kw.get("seqlens_k"),
                    kw.get("dropout_p", 0.0), kw.get("seed", 0), kw.get("block_mask"),
                    dict(q=q, k=k, v=k, o=q, dout=q, dq=q, dk=k, dv=k))
    return int(library().fa_bwd_ex_workspace_size(ctypes.byref(a)))


@_nvtx("fa.backward_general")
def backward_general(q, k, v, o, lse, dout, *, layout="bhsd", cu_seqlens_q=None,
                     cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None, scale=None,
                     causal=False, seqlens_k=None, dropout_p=0.0, seed=0, block_mask=None,
                     workspace=None, dq=None, dk=None, dv=None, dropout_row0=0, dropout_key0=0):
    """dQ, dK, dV for a general layout (fa_bwd_ex); arguments as forward_general."""
    import torch
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    a, keep = _desc(q, k, layout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, scale,
                    causal, seqlens_k, dropout_p, seed, block_mask,
                    dict(q=q, k=k, v=v, o=o, dout=dout, dq=dq, dk=dk, dv=dv),
                    (dropout_row0, dropout_key0))
    _check_lse(lse, q, layout)
    lib = library()
    need = int(lib.fa_bwd_ex_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    elif not workspace.is_cuda or workspace.device != q.device:
        raise ValueError("workspace: a tensor on the device of q is expected")
    code = lib.fa_bwd_ex(ctypes.byref(a), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                         _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream_ptr(q.device))
    _check(code, "fa_bwd_ex")
    del keep
    return dq, dk, dv


# ---------------------------------------------------------------------------
# combining partial results (context-parallel attention)
# ---------------------------------------------------------------------------

@_nvtx("fa.merge_partial")
def merge_partial(o_acc, lse_acc, o_part, lse_part):
    """o_acc (fp32 [..., d]), lse_acc (fp32 [...]) <- merge with the partial
    result o_part (bf16 [..., d]), lse_part (fp32 [...]); in place."""
    import torch
    for t, dt in ((o_acc, torch.float32), (lse_acc, torch.float32), (o_part, torch.bfloat16),
                  (lse_part, torch.float32)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError("merge_partial: contiguous CUDA tensors of the documented dtypes")
    d = o_acc.shape[-1]
    rows = o_acc.numel() // d
    if o_part.numel() != o_acc.numel() or lse_acc.numel() != rows or lse_part.numel() != rows:
        raise ValueError("merge_partial: shapes differ")
    _check(library().fa_merge_partial(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part),
                                      rows, d, _stream_ptr(o_acc.device)), "fa_merge_partial")


@_nvtx("fa.accumulate_bf16")
def accumulate_bf16(acc, part):
    """acc (fp32) += part (bf16), elementwise, in place."""
    import torch
    if acc.dtype != torch.float32 or part.dtype != torch.bfloat16 or acc.numel() != part.numel():
        raise ValueError("accumulate_bf16: fp32 accumulator and bf16 part of one size")
    if not (acc.is_cuda and part.is_cuda and acc.is_contiguous() and part.is_contiguous()):
        raise ValueError("accumulate_bf16: contiguous CUDA tensors")
    _check(library().fa_accumulate_bf16(_ptr(acc), _ptr(part), acc.numel(),
                                        _stream_ptr(acc.device)), "fa_accumulate_bf16")


@_nvtx("fa.convert_f32_bf16")
def convert_f32_bf16(src, out=None):
    """bf16 copy of an fp32 tensor (round to nearest even)."""
    import torch
    if src.dtype != torch.float32 or not src.is_cuda or not src.is_contiguous():
        raise ValueError("convert_f32_bf16: a contiguous fp32 CUDA tensor")
    out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device) if out is None else out
    _check(library().fa_convert_f32_bf16(_ptr(out), _ptr(src), src.numel(),
                                         _stream_ptr(src.device)), "fa_convert_f32_bf16")
    return out


# ---------------------------------------------------------------------------
# fused QKV projection
# ---------------------------------------------------------------------------

@_nvtx("fa.qkv_projection")
def qkv_projection(x, weight, bias, batch, heads, head_dim, q=None, k=None, v=None):
    """Q, K, V [B, H, N, d] = split_heads(x @ weight.T + bias) in one kernel.

    x: bf16 [B * N, d_model] (or [B, N, d_model]); weight: bf16 [3 H d, d_model];
    bias: bf16 [3 H d] or None."""
    import torch
    x2 = x.reshape(-1, x.shape[-1])
    for t in (x2, weight) + (() if bias is None else (bias,)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("qkv_projection: contiguous bf16 CUDA tensors")
    T, dm = x2.shape
    if T % batch:
        raise ValueError("qkv_projection: tokens not divisible by the batch size")
    N = T // batch
    shape = (batch, heads, N, head_dim)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device=x.device) if t is None else t
               for t in (q, k, v))
    code = library().fa_qkv_projection(_ptr(x2), _ptr(weight), _ptr(bias), _ptr(q), _ptr(k),
                                       _ptr(v), batch, N, heads, head_dim, dm,
                                       _stream_ptr(x.device))
    _check(code, "fa_qkv_projection")
    return q, k, v
