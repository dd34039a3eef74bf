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
import os

from .build import LIB_PATH

__all__ = [
    "FaError", "library", "forward", "backward", "backward_phases", "bwd_workspace_size",
    "dropout_mask", "last_device_status", "set_wait_timeout_ns",
    "wait_timeout_probe", "STATUS",
]

STATUS = {
    0: "FA_OK",
    1: "FA_ERR_INVALID_ARG",
    2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_CUDA",
    4: "FA_ERR_TIMEOUT",
    5: "FA_ERR_WORKSPACE",
}


class FaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_LIB = None
_vp, _i, _f, _u64, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                          ctypes.c_uint64, ctypes.c_size_t)

# name -> (restype, argtypes); must match include/fa.h
SIGNATURES = {
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
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_last_device_status": (_i, [_vp]),
    "fa_set_wait_timeout_ns": (None, [_u64]),
    "fa_debug_dropout_mask": (_i, [_vp, _i, _i, _i, _f, _u64, _vp]),
    "fa_debug_wait_timeout": (_i, [_vp]),
}


def library():
    """The loaded C library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m io_aware_exact_20_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
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


def wait_timeout_probe(device=None):
    import torch
    _check(library().fa_debug_wait_timeout(_stream_ptr(device or torch.cuda.current_device())),
           "fa_debug_wait_timeout")
