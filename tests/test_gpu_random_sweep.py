"""A seeded random sweep over the input space of fa_fwd_ex / fa_bwd_ex against
the float64 oracle.  The hand-picked parity cases each vary one or two
features; here every case draws all of them at once, so that combinations no
one wrote down get exercised: the layout (classic [B, H, N, d], token-major
[B, N, H, d], packed variable-length), every head dim (32 to 256, the
forward and the backward), N_q != N_k with the
bottom-right causal alignment, ragged tails, sequences up to 3000 rows, key
padding, block masks with whole tile rows and columns removed, dropout, and a
scale other than d^-1/2.

The cases come from one fixed generator seed, so a failure names a case that
reruns identically.  Bounds as in the other parity tests: O within
1e-2 + 2^-8 |O_ref| (strict 1e-2 where |O_ref| < 2), LSE within 1e-3, rows
without keys O = 0 and LSE = -inf on both sides, dQ / dK / dV relative L2
<= 2e-2."""

import numpy as np
import pytest

from oracle import attention_backward_gqa, attention_forward_gqa, gqa_expand, gqa_reduce
from oracle.varlen_ref import attention_backward_varlen, attention_forward_varlen
from test_gpu_fwd import compare

REL_L2 = 2e-2
N_CASES = 96
HEAD_DIMS = (32, 64, 96, 128, 192, 256)


def _draw_cases(n, seed=20250611):
    rng = np.random.default_rng(seed)
    cases = []
    for c in range(n):
        layout = ("bhsd", "bshd", "thd")[c % 3]
        d = int(rng.choice(HEAD_DIMS))
        B, H = int(rng.integers(1, 4)), int(rng.integers(1, 5))
        Hkv = H  # grouped K / V heads now and then: a proper divisor of H
        if H > 1 and rng.random() < 0.35:
            Hkv = int(rng.choice([x for x in range(1, H) if H % x == 0]))
        if layout == "thd":
            # lengths per sequence, zero-length ones included
            lq = rng.integers(0, 520, size=B)
            lk = lq.copy() if rng.random() < 0.4 else rng.integers(0, 700, size=B)
            if B > 1 and rng.random() < 0.6:
                lq[rng.integers(0, B)] = 0  # a sequence without queries
            if B > 1 and rng.random() < 0.4:
                lk[rng.integers(0, B)] = 0  # a sequence without keys
            lq[rng.integers(0, B)] = max(int(lq.max()), 1)  # at least one query row
            nq, nk = int(lq.max()), max(int(lk.max()), 1)
            lens = (lq.astype(np.int32).tolist(), lk.astype(np.int32).tolist())
        else:
            hi = 3000 if rng.random() < 0.15 else 700  # now and then many tiles
            nq = int(rng.integers(1, hi))
            nk = nq if rng.random() < 0.5 else int(rng.integers(1, hi + 100))
            lens = None
        causal = bool(rng.random() < 0.5)
        kv_pad = None
        if rng.random() < 0.3:
            kv_pad = rng.integers(0, nk + 1, size=B).astype(np.int32).tolist()
        mask = None
        if rng.random() < 0.35:
            nbq, nbk = (nq + 127) // 128, (nk + 127) // 128
            bm = (rng.random((nbq, nbk)) < rng.uniform(0.3, 0.9)).astype(np.uint8)
            if nbq > 1 and rng.random() < 0.5:
                bm[rng.integers(0, nbq), :] = 0  # a query tile with no keys
            if nbk > 1 and rng.random() < 0.5:
                bm[:, rng.integers(0, nbk)] = 0  # a key tile no query sees
            mask = bm.tolist()
        p = float(rng.choice([0.0, 0.0, 0.1, 0.3]))
        scale = float(d ** -0.5 * rng.uniform(0.5, 1.5))
        cases.append(dict(case=c, layout=layout, d=d, B=B, H=H, Hkv=Hkv, nq=nq, nk=nk, lens=lens,
                          causal=causal, kv_pad=kv_pad, mask=mask, p=p, scale=scale,
                          seed=int(rng.integers(0, 2 ** 63))))
    return cases


CASES = _draw_cases(N_CASES)


def _case_id(c):
    parts = [f"c{c['case']:02d}", c["layout"], f"d{c['d']}",
             f"B{c['B']}H{c['H']}" + (f"kv{c['Hkv']}" if c["Hkv"] != c["H"] else ""),
             f"q{c['nq']}k{c['nk']}"]
    if c["causal"]:
        parts.append("causal")
    if c["kv_pad"] is not None:
        parts.append("kvpad")
    if c["mask"] is not None:
        parts.append("bmask")
    if c["p"] > 0:
        parts.append(f"p{c['p']}")
    return "-".join(parts)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    n = np.linalg.norm(ref)
    return np.linalg.norm(a - ref) / n if n > 0 else np.linalg.norm(a)


def test_sweep_covers_every_feature():
    """The drawn cases reach every layout, head dim and mask kind, and the
    64-, 128- and 256-wide kernels in every layout (checked without a device)."""
    seen = {(c["layout"], min(w for w in (64, 128, 256) if c["d"] <= w)) for c in CASES}
    assert len(seen) == 9, seen
    assert {c["d"] for c in CASES} == set(HEAD_DIMS)
    assert any(c["nq"] != c["nk"] and c["layout"] != "thd" for c in CASES)
    assert any(c["mask"] is not None and c["causal"] for c in CASES)
    assert any(c["kv_pad"] is not None for c in CASES)
    assert any(c["p"] > 0 and c["mask"] is not None for c in CASES)
    assert any(c["lens"] is not None and 0 in c["lens"][0] for c in CASES)
    assert any(c["lens"] is not None and 0 in c["lens"][1] for c in CASES)
    assert {c["layout"] for c in CASES if c["Hkv"] != c["H"]} == {"bhsd", "bshd", "thd"}


@pytest.mark.gpu
@pytest.mark.parametrize("c", CASES, ids=_case_id)
def test_random_case_matches_oracle(lib, parity_record, c):
    import torch
    g = torch.Generator().manual_seed(c["seed"] % (2 ** 62))
    B, H, Hkv, d, layout = c["B"], c["H"], c["Hkv"], c["d"], c["layout"]
    G = H // Hkv
    bm = None if c["mask"] is None else np.array(c["mask"], dtype=np.uint8)
    kv_pad = None if c["kv_pad"] is None else np.array(c["kv_pad"], dtype=np.int32)
    kw = dict(layout=layout, scale=c["scale"], causal=c["causal"], seqlens_k=kv_pad,
              dropout_p=c["p"], seed=c["seed"], block_mask=bm)

    def rnd(*shape):
        return torch.randn(*shape, generator=g).to(torch.bfloat16)

    if layout == "thd":
        lq, lk = c["lens"]
        cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
        cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
        hq, hdo = rnd(int(cu_q[-1]), H, d), rnd(int(cu_q[-1]), H, d)
        hk, hv = rnd(int(cu_k[-1]), Hkv, d), rnd(int(cu_k[-1]), Hkv, d)
        kw.update(cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=c["nq"],
                  max_seqlen_k=c["nk"])
        to_dev = lambda x: x.cuda()  # noqa: E731
        to_host = f64
    else:
        hq, hdo = rnd(B, H, c["nq"], d), rnd(B, H, c["nq"], d)
        hk, hv = rnd(B, Hkv, c["nk"], d), rnd(B, Hkv, c["nk"], d)
        if layout == "bshd":
            to_dev = lambda x: x.transpose(1, 2).contiguous().cuda()  # noqa: E731
            to_host = lambda x: f64(x.transpose(1, 2))  # noqa: E731
        else:
            to_dev = lambda x: x.cuda()  # noqa: E731
            to_host = f64

    q, k, v, do = (to_dev(x) for x in (hq, hk, hv, hdo))
    o, lse = lib.forward_general(q, k, v, **kw)
    grads = lib.backward_general(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0

    ref_args = (c["scale"], c["causal"], kv_pad, c["p"], c["seed"], bm)
    if layout == "thd":
        ek, ev = gqa_expand(f64(hk), G), gqa_expand(f64(hv), G)  # [T, H, d]
        ro, rl = attention_forward_varlen(f64(hq), ek, ev, cu_q, cu_k, *ref_args)
        # packed O [T, H, d] and LSE [H, T] viewed as one batch entry
        as_bhsd = lambda x: np.transpose(x, (1, 0, 2))[None]  # noqa: E731
        compare(as_bhsd(to_host(o)), lse.cpu().numpy().astype(np.float64)[None], as_bhsd(ro),
                rl[None], parity_record)
    else:
        ro, rl = attention_forward_gqa(f64(hq), f64(hk), f64(hv), *ref_args)
        compare(to_host(o), lse.cpu().numpy().astype(np.float64), ro, rl, parity_record)

    if layout == "thd":
        rq, rk, rv = attention_backward_varlen(f64(hq), ek, ev, f64(hdo), cu_q, cu_k, *ref_args)
        rg = (rq, gqa_reduce(rk, G), gqa_reduce(rv, G))
    else:
        rg = attention_backward_gqa(f64(hq), f64(hk), f64(hv), f64(hdo), *ref_args)
    errs = {}
    for name, a, r in zip(("dq", "dk", "dv"), grads, rg):
        got = to_host(a)
        assert np.isfinite(got).all(), name
        errs[name] = rel_l2(got, r)
    parity_record(**{f"{k}_rel_l2": float(v) for k, v in errs.items()})
    for name, e in errs.items():
        assert e <= REL_L2, (name, e)
