"""General layouts through fa_fwd_ex / fa_bwd_ex against the float64 oracle:
token-major [B, N, H, d] tensors, strided views into a fused QKV buffer,
N_q != N_k with the bottom-right causal alignment, head dims 32 and 96, and
packed variable-length batches (the BERT-shaped workload without padding).

Bounds as in the other parity tests: O within 1e-2 + 2^-8 |O_ref| (strict
1e-2 where |O_ref| < 2), LSE within 1e-3, dQ / dK / dV relative L2 <= 2e-2.
"""

import numpy as np
import pytest

from oracle import (
    attention_backward,
    attention_backward_varlen,
    attention_forward,
    attention_forward_varlen,
)
from io_aware_exact_20_b200.workloads import make_block_mask, make_qkvdo, make_seqlens
from test_gpu_fwd import compare

pytestmark = pytest.mark.gpu

REL_L2 = 2e-2


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    n = np.linalg.norm(ref)
    return np.linalg.norm(a - ref) / n if n > 0 else np.linalg.norm(a)


def randn(shape, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def check_grads(got, ref, record=None):
    errs = {}
    for name, a, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(a).all(), name
        errs[name] = rel_l2(a, r)
        assert errs[name] <= REL_L2, (name, errs[name])
    if record is not None:
        record(**{f"{k}_rel_l2": float(v) for k, v in errs.items()})


# ---------------------------------------------------------------------------
# padded layouts: [B, N, H, d], strided views, N_q != N_k, d = 32 / 96
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,lens,density,p", [
    (2, 3, 300, 300, 64, True, None, None, 0.1),      # token-major, same lengths
    (2, 2, 200, 520, 64, True, None, None, 0.0),      # fewer queries than keys
    (2, 2, 520, 200, 128, True, None, None, 0.1),     # more queries: leading rows see no key
    (1, 2, 384, 1000, 128, False, (300, 1000), None, 0.0),
    (2, 2, 640, 384, 64, True, (100, 384), 0.5, 0.2),  # every mask with N_q > N_k
    (2, 3, 333, 333, 32, True, None, None, 0.1),      # d = 32 on the 64-wide kernel
    (2, 2, 400, 300, 96, True, (150, 300), None, 0.1),  # d = 96 on the 128-wide kernel
    (1, 2, 129, 1, 96, False, None, None, 0.0),
])
@pytest.mark.parametrize("layout", ["bshd", "bhsd"])
def test_general_padded_layouts_match_oracle(lib, parity_record, layout, B, H, Nq, Nk, d, causal,
                                             lens, density, p):
    import torch
    qh, doh = randn((B, H, Nq, d), 1), randn((B, H, Nq, d), 2)
    kh, vh = randn((B, H, Nk, d), 3), randn((B, H, Nk, d), 4)
    seqlens = None if lens is None else make_seqlens(B, lens[0], lens[1], 5)
    bm = None
    if density is not None:
        nbq, nbk = (Nq + 127) // 128, (Nk + 127) // 128
        bm = (np.random.default_rng(6).random((nbq, nbk)) < density).astype(np.uint8)
        bm[0, :] = 1
    scale, seed = d ** -0.5, 77

    def dev(x):  # the layout's tensor on the GPU
        x = x.cuda()
        return x.transpose(1, 2).contiguous() if layout == "bshd" else x

    def host(x):  # back to [B, H, N, d] for the oracle
        x = x.transpose(1, 2) if layout == "bshd" else x
        return f64(x)

    kw = dict(layout=layout, scale=scale, causal=causal, seqlens_k=seqlens, dropout_p=p,
              seed=seed, block_mask=bm)
    q, k, v, do = dev(qh), dev(kh), dev(vh), dev(doh)
    o, lse = lib.forward_general(q, k, v, **kw)
    dq, dk, dv = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = attention_forward(f64(qh), f64(kh), f64(vh), scale, causal, seqlens, p, seed, bm)
    compare(host(o), f64(lse), ro, rl, parity_record)
    ref = attention_backward(f64(qh), f64(kh), f64(vh), f64(doh), scale, causal, seqlens, p, seed,
                             bm)
    check_grads((host(dq), host(dk), host(dv)), ref, parity_record)


def test_general_strided_views_of_a_fused_qkv_buffer(lib, parity_record):
    """q, k, v as views into one [B, N, 3, H, d] buffer (row stride 3 H d) and
    gradients written into the matching views of a fused dQKV buffer."""
    import torch
    B, N, H, d = 2, 300, 4, 64
    qkv = randn((B, N, 3, H, d), 8).cuda()
    do = randn((B, N, H, d), 9).cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    dqkv = torch.full_like(qkv, float("nan"))
    kw = dict(layout="bshd", causal=True, dropout_p=0.1, seed=3)
    o, lse = lib.forward_general(q, k, v, **kw)
    lib.backward_general(q, k, v, o, lse, do, dq=dqkv[:, :, 0], dk=dqkv[:, :, 1],
                         dv=dqkv[:, :, 2], **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    t = lambda x: f64(x.transpose(1, 2))  # noqa: E731  [B, N, H, d] -> [B, H, N, d]
    ro, rl = attention_forward(t(q), t(k), t(v), d ** -0.5, True, None, 0.1, 3)
    compare(t(o), f64(lse), ro, rl, parity_record)
    ref = attention_backward(t(q), t(k), t(v), t(do), d ** -0.5, True, None, 0.1, 3)
    check_grads((t(dqkv[:, :, 0]), t(dqkv[:, :, 1]), t(dqkv[:, :, 2])), ref, parity_record)


# ---------------------------------------------------------------------------
# packed variable-length batches
# ---------------------------------------------------------------------------

def run_packed(lib, lq, lk, H, d, causal, p, seed=21, key_lens=None, density=None, extra_rows=0,
               data_seed=11):
    import torch
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    Tq, Tk = int(cu_q[-1]) + extra_rows, int(cu_k[-1]) + extra_rows
    qh, doh = randn((Tq, H, d), data_seed), randn((Tq, H, d), data_seed + 1)
    kh, vh = randn((Tk, H, d), data_seed + 2), randn((Tk, H, d), data_seed + 3)
    mq, mk = max(max(lq), 1), max(max(lk), 1)
    bm = None
    if density is not None:
        bm = (np.random.default_rng(7).random(((mq + 127) // 128, (mk + 127) // 128))
              < density).astype(np.uint8)
    kw = dict(layout="thd", cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=mq,
              max_seqlen_k=mk, scale=d ** -0.5, causal=causal, seqlens_k=key_lens, dropout_p=p,
              seed=seed, block_mask=bm)
    q, k, v, do = (x.cuda() for x in (qh, kh, vh, doh))
    o = torch.full_like(q, float("nan"))
    lse = torch.full((H, Tq), float("nan"), dtype=torch.float32, device="cuda")
    lib.forward_general(q, k, v, out=o, lse=lse, **kw)
    dq, dk, dv = (torch.full_like(x, float("nan")) for x in (q, k, v))
    lib.backward_general(q, k, v, o, lse, do, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    n_q, n_k = int(cu_q[-1]), int(cu_k[-1])
    ro, rl = attention_forward_varlen(f64(qh)[:n_q], f64(kh)[:n_k], f64(vh)[:n_k], cu_q, cu_k,
                                      d ** -0.5, causal, key_lens, p, seed, bm)
    rg = attention_backward_varlen(f64(qh)[:n_q], f64(kh)[:n_k], f64(vh)[:n_k], f64(doh)[:n_q],
                                   cu_q, cu_k, d ** -0.5, causal, key_lens, p, seed, bm)
    return (o, lse, dq, dk, dv), (ro, rl, rg), (n_q, n_k)


@pytest.mark.parametrize("lq,lk,H,d,causal,p,key_lens,density", [
    ([300, 1, 129, 512, 77], [300, 1, 129, 512, 77], 2, 64, False, 0.1, None, None),
    ([300, 1, 129, 512, 77], [300, 1, 129, 512, 77], 2, 128, True, 0.1, None, None),
    ([100, 0, 260, 64], [250, 3, 130, 300], 2, 64, True, 0.0, None, None),   # N_q != N_k per sequence
    ([200, 333, 5], [180, 400, 40], 3, 128, True, 0.2, [150, 399, 1], 0.6),  # every mask
    ([129, 257], [64, 700], 2, 96, False, 0.1, None, None),
    ([200, 90], [90, 200], 2, 32, True, 0.0, None, None),
])
def test_packed_varlen_matches_oracle(lib, parity_record, lq, lk, H, d, causal, p, key_lens,
                                     density):
    got, ref, (n_q, n_k) = run_packed(lib, lq, lk, H, d, causal, p,
                                      key_lens=None if key_lens is None else
                                      np.array(key_lens, dtype=np.int32), density=density)
    o, lse, dq, dk, dv = got
    ro, rl, rg = ref
    oo = f64(o)
    ll = lse.cpu().numpy().astype(np.float64)
    # [T, H, d] -> [1, H, T, d] so that compare() sees one "batch entry"
    compare(oo.transpose(1, 0, 2)[None], ll[None], ro.transpose(1, 0, 2)[None], rl[None],
            parity_record)
    check_grads((f64(dq), f64(dk), f64(dv)), rg, parity_record)


def test_packed_varlen_writes_no_row_outside_the_sequences(lib):
    """Rows past cu[B] belong to no sequence: O, LSE, dQ, dK, dV there keep the
    NaN they held before the calls (nothing is computed or written for them)."""
    got, ref, (n_q, n_k) = run_packed(lib, [130, 40], [100, 70], 2, 64, True, 0.1,
                                      extra_rows=37)
    o, lse, dq, dk, dv = got
    assert np.isnan(f64(o)[n_q:]).all() and np.isnan(lse.cpu().numpy()[:, n_q:]).all()
    assert np.isnan(f64(dq)[n_q:]).all()
    assert np.isnan(f64(dk)[n_k:]).all() and np.isnan(f64(dv)[n_k:]).all()
    assert np.isfinite(f64(o)[:n_q]).all() and np.isfinite(f64(dk)[:n_k]).all()


def test_packed_bert_shaped_batch(lib, parity_record):
    """The BERT-large-shaped workload packed: 16 sequences of lengths
    U[256, 512], 16 heads, d = 64, dropout 0.1, no padding rows at all."""
    lens = make_seqlens(16, 256, 512, 2003)
    got, ref, _ = run_packed(lib, list(lens), list(lens), 16, 64, False, 0.1, seed=0x5EED0003)
    o, lse, dq, dk, dv = got
    ro, rl, rg = ref
    compare(f64(o).transpose(1, 0, 2)[None], lse.cpu().numpy().astype(np.float64)[None],
            ro.transpose(1, 0, 2)[None], rl[None], parity_record)
    check_grads((f64(dq), f64(dk), f64(dv)), rg, parity_record)


def test_packed_equals_padded_with_key_lengths(lib):
    """The packed BERT-shaped batch and the padded one with key padding give
    the same O on every real row and the same dK / dV on every real key (the
    padded run's extra query rows add to dK / dV, so they are zeroed in dO)."""
    import torch
    B, H, N, d, p, seed = 6, 2, 512, 64, 0.1, 5
    lens = make_seqlens(B, 256, 512, 2003)
    q, k, v, do = make_qkvdo(B, H, N, d, 31)
    for b, n in enumerate(lens):
        do[b, :, n:] = 0
    kw = dict(scale=d ** -0.5, dropout_p=p, seed=seed)
    gq, gk, gv, gdo = (x.cuda() for x in (q, k, v, do))
    o_pad, lse_pad = lib.forward(gq, gk, gv, seqlens=lens, **kw)
    _, dk_pad, dv_pad = lib.backward(gq, gk, gv, o_pad, lse_pad, gdo, seqlens=lens, **kw)
    pack = lambda x: torch.cat([x[b, :, :n].transpose(0, 1) for b, n in enumerate(lens)])  # noqa
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    gkw = dict(layout="thd", cu_seqlens_q=cu, cu_seqlens_k=cu, max_seqlen_q=N, max_seqlen_k=N,
               **kw)
    pq, pk, pv, pdo = (pack(x).contiguous() for x in (gq, gk, gv, gdo))
    o, lse = lib.forward_general(pq, pk, pv, **gkw)
    _, dk, dv = lib.backward_general(pq, pk, pv, o, lse, pdo, **gkw)
    torch.cuda.synchronize()
    assert (pack(o_pad) - o).abs().max().item() == 0.0  # same tiles, same arithmetic
    assert rel_l2(f64(pack(dk_pad)), f64(dk)) < 1e-2
    assert rel_l2(f64(pack(dv_pad)), f64(dv)) < 1e-2


@pytest.mark.parametrize("d", [64, 128, 256])
def test_dropout_positions_of_a_block(lib, parity_record, d):
    """A call that evaluates one block of a longer sequence (queries at
    positions 256.., keys at 128..) with dropout keys its bits by those
    positions: O, LSE and the gradients equal the oracle's for the same
    block with the same positions (its own softmax over the block's keys)."""
    import torch
    from oracle import head_backward_block, head_forward_rows
    B, H, Nq, Nk, row0, key0, p, seed = 1, 2, 200, 328, 256, 128, 0.2, 0x5EED0099
    qh, doh = randn((B, H, Nq, d), 31), randn((B, H, Nq, d), 32)
    kh, vh = randn((B, H, Nk, d), 33), randn((B, H, Nk, d), 34)
    scale = d ** -0.5
    kw = dict(scale=scale, dropout_p=p, seed=seed, dropout_row0=row0, dropout_key0=key0)
    q, k, v, do = (x.cuda() for x in (qh, kh, vh, doh))
    o, lse = lib.forward_general(q, k, v, **kw)
    dq, dk, dv = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    ro, rl = np.zeros((B, H, Nq, d)), np.zeros((B, H, Nq))
    rg = [np.zeros((B, H, Nq, d)), np.zeros((B, H, Nk, d)), np.zeros((B, H, Nk, d))]
    for h in range(H):
        a = [f64(x)[0, h] for x in (qh, kh, vh, doh)]
        ro[0, h], rl[0, h] = head_forward_rows(a[0], a[1], a[2], scale, np.arange(Nq),
                                               dropout_p=p, seed=seed, b=0, h=h, row0=row0,
                                               key0=key0)
        delta = (a[3] * ro[0, h]).sum(-1)
        g = head_backward_block(a[0], a[1], a[2], a[3], rl[0, h], delta, scale, False, Nq, Nk,
                                row0, key0, p, seed, 0, h)
        for i in range(3):
            rg[i][0, h] = g[i]
    compare(f64(o), f64(lse), ro, rl, parity_record)
    check_grads((f64(dq), f64(dk), f64(dv)), rg, parity_record)
