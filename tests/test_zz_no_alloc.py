"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(for example code running inside an allocator or memory-pool callback, which
must not re-enter the allocator, or a host that reserves all device memory up
front).  Its workspace is a fixed array inside the library.

Checked through the C ABI on two calls in a row (the second call finds the
first call's leftovers in the shared array): every call returns FA_OK (the
first one on the device also does the array's one-time set-up), and its
dQ, dK, dV match both the float64 oracle and the workspace-taking fa_bwd
within the backward tolerance of the other parity tests.  A request too large
for the array is refused before any launch.

Kept in a file of its own that pytest collects last."""

import numpy as np
import pytest

from oracle import attention_backward
from io_aware_exact_20_b200.workloads import make_qkvdo, make_seqlens

REL_L2 = 2e-2  # the backward parity bound used by the other tests


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    return np.linalg.norm(a - ref) / np.linalg.norm(ref)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal,lens,p", [
    (2, 3, 300, 64, True, None, 0.1),
    (1, 2, 520, 128, False, (200, 520), 0.0),
    (1, 2, 400, 256, True, None, 0.1),          # the 256-wide backward (two CTAs per key tile)
])
def test_noalloc_backward_matches_oracle_and_workspace_backward(lib, B, H, N, d, causal, lens,
                                                                p):
    import torch
    hq, hk, hv, hdo = make_qkvdo(B, H, N, d, 17)
    q, k, v, do = (x.cuda() for x in (hq, hk, hv, hdo))
    lens_h = None if lens is None else make_seqlens(B, lens[0], lens[1], 18)
    sl = None if lens_h is None else torch.as_tensor(lens_h).cuda()
    scale, seed = d ** -0.5, 99
    kw = dict(scale=scale, causal=causal, seqlens=sl, dropout_p=p, seed=seed)
    o, lse = lib.forward(q, k, v, **kw)
    ref = lib.backward(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    oracle = attention_backward(f64(hq), f64(hk), f64(hv), f64(hdo), scale, causal, lens_h, p,
                                seed)
    so = lib.library()
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    for _ in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        code = so.fa_bwd_noalloc(ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse), ptr(do), ptr(dq),
                                 ptr(dk), ptr(dv), B, H, N, d, scale, int(causal), ptr(sl), p,
                                 seed, None, stream)
        assert code == 0
        torch.cuda.synchronize()
        assert lib.last_device_status() == 0
        for a, r, g in zip((dq, dk, dv), ref, oracle):
            assert np.isfinite(f64(a)).all()
            assert rel_l2(f64(a), g) <= REL_L2
            assert rel_l2(f64(a), f64(r)) <= REL_L2


@pytest.mark.gpu
def test_noalloc_rejects_requests_beyond_its_array(lib):
    so = lib.library()
    a16 = 1 << 20  # never dereferenced: the size check comes first
    B, H, N, d = 1, 64, 8192, 128  # workspace 272 MB > 64 MiB
    assert so.fa_bwd_workspace_size(B, H, N, d) > (64 << 20)
    code = so.fa_bwd_noalloc(a16, a16, a16, a16, a16, a16, a16, a16, a16, B, H, N, d, 0.1, 0,
                             None, 0.0, 0, None, None)
    assert code == 5  # FA_ERR_WORKSPACE
