"""Context-parallel ring attention (io_aware_exact_20_b200.context_parallel).

CPU part (no GPU): two gloo ranks run the ring's schedule and exchanges
(torch.distributed point-to-point) with the float64 oracle standing in for
the kernels; the chunks they return must equal the oracle's attention over
the whole sequence.  This checks the ring: which chunk meets which, the
causal skips, the merge of partial results and the journey of the dK / dV
accumulators back to their owner.

GPU part: the same ring with the library's kernels, W ranks emulated in one
process on one device (run one after the other; no kernel waits on another),
against the float64 oracle on the whole sequence.
"""

import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleKernels:
    """The oracle in the kernels' place (float64 torch CPU tensors)."""

    def forward(self, q, k, v, scale, causal, drop=None):
        import torch
        from oracle import head_forward_rows
        p, seed, row0, key0 = drop if drop is not None else (0.0, 0, 0, 0)
        B, H, n, d = q.shape
        o, lse = np.zeros(q.shape), np.zeros(q.shape[:-1])
        for b in range(B):
            for h in range(H):
                o[b, h], lse[b, h] = head_forward_rows(
                    q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), scale, np.arange(n),
                    causal, dropout_p=p, seed=seed, b=b, h=h, row0=row0, key0=key0)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def backward(self, q, k, v, o, lse, do, scale, causal, drop=None):
        import torch
        from oracle import head_backward_block
        p, seed, row0, key0 = drop if drop is not None else (0.0, 0, 0, 0)
        B, H, n, d = q.shape
        dq, dk, dv = (np.zeros(t.shape) for t in (q, k, v))
        delta = (do.numpy() * o.numpy()).sum(-1)
        for b in range(B):
            for h in range(H):
                # sequence positions q0 = row0, k0 = key0 with n_q = n_k: the
                # causal mask of a diagonal chunk is the local one
                g = head_backward_block(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(),
                                        do[b, h].numpy(), lse[b, h].numpy(), delta[b, h], scale,
                                        causal, 0, 0, row0, key0, p, seed, b, h)
                dq[b, h], dk[b, h], dv[b, h] = g
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)

    def zeros_acc(self, like):
        import torch
        return torch.zeros(like.shape, dtype=torch.float64)

    def empty_lse(self, q):
        import torch
        return torch.full(q.shape[:-1], float("-inf"), dtype=torch.float64)

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        import torch
        from oracle import merge_partials
        o, lse = merge_partials(o_acc.numpy(), lse_acc.numpy(), o_part.numpy(), lse_part.numpy())
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(lse))

    def accumulate(self, acc, part):
        acc += part

    def finish(self, acc):
        return acc


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir, causal, p):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from io_aware_exact_20_b200 import context_parallel as cp

    rng = np.random.default_rng(71)
    B, H, N, d = 1, 2, 96, 8
    full = [rng.standard_normal((B, H, N, d)) for _ in range(4)]
    n = N // world
    q, k, v, do = (torch.from_numpy(x[:, :, rank * n:(rank + 1) * n].copy()) for x in full)
    kern = OracleKernels()
    o, lse = cp.attention_forward(q, k, v, 0.3, causal, kern=kern, dropout_p=p, seed=SEED)
    dq, dk, dv = cp.attention_backward(q, k, v, o, lse, do, 0.3, causal, kern=kern, dropout_p=p,
                                       seed=SEED)
    np.savez(os.path.join(outdir, f"r{rank}.npz"), o=o.numpy(), lse=lse.numpy(), dq=dq.numpy(),
             dk=dk.numpy(), dv=dv.numpy())
    dist.barrier()
    dist.destroy_process_group()


SEED = 0x5EED0042


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal,p", [(False, 0.0), (True, 0.0), (True, 0.2)])
def test_ring_schedule_on_gloo_ranks_equals_full_attention(tmp_path, world, causal, p):
    """With dropout too: each chunk pair keys its bits by sequence positions,
    so the ring equals the unsplit attention with the same seed."""
    import torch.multiprocessing as mp

    from oracle import attention_backward, attention_forward
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), causal, p),
                       nprocs=world, join=True, start_method="spawn")
    rng = np.random.default_rng(71)
    B, H, N, d = 1, 2, 96, 8
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    ro, rl = attention_forward(q, k, v, 0.3, causal, None, p, SEED)
    rdq, rdk, rdv = attention_backward(q, k, v, do, 0.3, causal, None, p, SEED)
    n = N // world
    for r in range(world):
        got = np.load(tmp_path / f"r{r}.npz")
        s = slice(r * n, (r + 1) * n)
        assert np.abs(got["o"] - ro[:, :, s]).max() < 1e-12
        assert np.abs(got["lse"] - rl[:, :, s]).max() < 1e-12
        assert np.abs(got["dq"] - rdq[:, :, s]).max() < 1e-10
        assert np.abs(got["dk"] - rdk[:, :, s]).max() < 1e-10
        assert np.abs(got["dv"] - rdv[:, :, s]).max() < 1e-10


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("p", [0.0, 0.25])
def test_emulated_ring_with_oracle_kernels_on_cpu(world, p):
    """run_emulated drives all ranks in one process: same results as above."""
    import torch
    sys.path.insert(0, ROOT)
    from io_aware_exact_20_b200 import context_parallel as cp
    from oracle import attention_backward, attention_forward
    rng = np.random.default_rng(72)
    B, H, N, d = 1, 1, 48, 4
    full = [rng.standard_normal((B, H, N, d)) for _ in range(4)]
    n = N // world
    ch = [[torch.from_numpy(x[:, :, r * n:(r + 1) * n].copy()) for x in full]
          for r in range(world)]
    kern = OracleKernels()
    outs = cp.run_emulated([cp.ring_forward(r, world, *ch[r][:3], 0.5, True, kern, p, SEED)
                            for r in range(world)])
    grads = cp.run_emulated([cp.ring_backward(r, world, *ch[r][:3], outs[r][0], outs[r][1],
                                              ch[r][3], 0.5, True, kern, p, SEED)
                             for r in range(world)])
    ro, _ = attention_forward(*full[:3], 0.5, True, None, p, SEED)
    rg = attention_backward(*full, 0.5, True, None, p, SEED)
    for r in range(world):
        s = slice(r * n, (r + 1) * n)
        assert np.abs(outs[r][0].numpy() - ro[:, :, s]).max() < 1e-12
        for a, b in zip(grads[r], rg):
            assert np.abs(a.numpy() - b[:, :, s]).max() < 1e-10


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("d,causal,p", [(64, True, 0.0), (96, True, 0.0), (128, False, 0.0),
                                        (128, True, 0.0), (192, False, 0.0), (256, True, 0.0),
                                        (64, True, 0.1), (128, False, 0.2), (256, True, 0.1)])
def test_ring_with_library_kernels_on_one_gpu(lib, parity_record, world, d, causal, p):
    """The ring with the library's kernels (fa_fwd_ex, fa_bwd_ex, merge and
    accumulate kernels), W ranks emulated on one device, against the oracle
    over the whole sequence; with dropout, each call keys its bits by the
    positions of its chunks (dropout_row0 / dropout_key0), so the ring draws
    the bits of the unsplit attention."""
    import torch

    from io_aware_exact_20_b200 import context_parallel as cp
    from io_aware_exact_20_b200.workloads import make_qkvdo
    from oracle import attention_backward, attention_forward
    B, H, N = 1, 2, 192 * world
    q, k, v, do = make_qkvdo(B, H, N, d, 81)
    n = N // world
    ch = [[x[:, :, r * n:(r + 1) * n].contiguous().cuda() for x in (q, k, v, do)]
          for r in range(world)]
    kern = cp.LibraryKernels(lib)
    scale = d ** -0.5
    outs = cp.run_emulated([cp.ring_forward(r, world, *ch[r][:3], scale, causal, kern, p, SEED)
                            for r in range(world)])
    grads = cp.run_emulated([cp.ring_backward(r, world, *ch[r][:3], outs[r][0], outs[r][1],
                                              ch[r][3], scale, causal, kern, p, SEED)
                             for r in range(world)])
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    ro, rl = attention_forward(f(q), f(k), f(v), scale, causal, None, p, SEED)
    rg = attention_backward(f(q), f(k), f(v), f(do), scale, causal, None, p, SEED)
    _check_ring(outs, grads, ro, rl, rg, world, parity_record)


def _check_ring(outs, grads, ro, rl, rg, world, parity_record):
    from test_gpu_fwd import compare
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    o = np.concatenate([f(outs[r][0]) for r in range(world)], axis=2)
    lse = np.concatenate([outs[r][1].cpu().numpy() for r in range(world)], axis=2)
    compare(o, lse.astype(np.float64), ro, rl, parity_record)
    for i, name in enumerate(("dq", "dk", "dv")):
        g = np.concatenate([f(grads[r][i]) for r in range(world)], axis=2)
        e = np.linalg.norm(g - rg[i]) / np.linalg.norm(rg[i])
        assert e <= 2e-2, (name, e)


@pytest.mark.gpu
@pytest.mark.parametrize("world,Hkv,p", [(2, 1, 0.1), (4, 2, 0.0)])
def test_ring_with_grouped_kv_heads(lib, parity_record, world, Hkv, p):
    """The ring passes K / V chunks with fewer heads than the queries (grouped
    K / V heads): every call reads K / V head h // (H / H_kv), and the dK / dV
    accumulators that travel with a chunk have its K / V heads."""
    import torch

    from io_aware_exact_20_b200 import context_parallel as cp
    from io_aware_exact_20_b200.workloads import make_qkvdo
    from oracle import attention_backward_gqa, attention_forward_gqa
    B, H, N, d = 1, 4, 192 * world, 128
    q, _, _, do = make_qkvdo(B, H, N, d, 83)
    _, k, v, _ = make_qkvdo(B, Hkv, N, d, 84)
    n = N // world
    ch = [[x[:, :, r * n:(r + 1) * n].contiguous().cuda() for x in (q, k, v, do)]
          for r in range(world)]
    kern = cp.LibraryKernels(lib)
    scale = d ** -0.5
    outs = cp.run_emulated([cp.ring_forward(r, world, *ch[r][:3], scale, True, kern, p, SEED)
                            for r in range(world)])
    grads = cp.run_emulated([cp.ring_backward(r, world, *ch[r][:3], outs[r][0], outs[r][1],
                                              ch[r][3], scale, True, kern, p, SEED)
                             for r in range(world)])
    torch.cuda.synchronize()
    assert lib.last_device_status() == 0
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    ro, rl = attention_forward_gqa(f(q), f(k), f(v), scale, True, None, p, SEED)
    rg = attention_backward_gqa(f(q), f(k), f(v), f(do), scale, True, None, p, SEED)
    _check_ring(outs, grads, ro, rl, rg, world, parity_record)
