"""Context-parallel exact attention: one sequence split across GPUs.

The pages name multi-GPU IO-aware attention as the next step beyond one GPU
(suanlizi.com FlashAttention summary, future-work section on multi-GPU IO
optimisation).  Here the sequence is cut into W equal chunks, rank r holding
the queries, keys and values of chunk r ([B, H, N / W, d] each).  The K / V
chunks travel around a ring (rank r sends to r + 1 and receives from r - 1,
NCCL point-to-point into a local buffer, while the current chunk is being
computed on), so that every rank meets every chunk once:

  forward, step s:  c = (r - s) mod W;  (O_c, LSE_c) = fa_fwd_ex(Q_r, K_c, V_c)
                    merged into the running (O, LSE) by fa_merge_partial
  backward, step s: dQ_r += dQ part, dK_c += dK part, dV_c += dV part from
                    fa_bwd_ex(Q_r, K_c, V_c, O_r, LSE_r, dO_r) with the final O
                    and LSE (so the kernel's D and P are those of the full row);
                    the fp32 dK / dV accumulators travel with their chunk and
                    reach its owner after W exchanges.

Under the causal mask chunk c is skipped by rank r when c > r (every pair
masked) and computed with the causal mask when c = r (equal chunk sizes, so
the bottom-right alignment is the usual one); c < r is unmasked.  Dropout keys
its bits by positions in the whole sequence: every call tells the kernels the
positions of its first query row (r N / W) and first key (c N / W), so the
ring draws exactly the bits of the unsplit attention (the chunk length must
then be a multiple of 8, the keys of one generator call).

Every arithmetic step runs in the library's kernels (fa_fwd_ex, fa_bwd_ex,
fa_merge_partial, fa_accumulate_bf16, fa_convert_f32_bf16); torch supplies the
buffers, the streams and torch.distributed.  No TMA multicast and no library
kernel ever reads another GPU's memory: the received chunks are local copies.

The algorithm is written once, as a generator per rank that yields its
exchanges; ``run_ring`` drives it with torch.distributed on a real process
group, ``run_emulated`` drives W of them in one process (one after the other,
no kernel waits for another) so the ring can be checked on a single device.
"""

from __future__ import annotations


class LibraryKernels:
    """The library's kernels, as the ring algorithm calls them."""

    def __init__(self, fa=None):
        if fa is None:
            import io_aware_exact_20_b200 as fa
        self.fa = fa

    def forward(self, q, k, v, scale, causal, drop=None):
        """drop: None, or (dropout_p, seed, position of q's first row, of k's first key)."""
        kw = {} if drop is None else dict(dropout_p=drop[0], seed=drop[1], dropout_row0=drop[2],
                                          dropout_key0=drop[3])
        return self.fa.forward_general(q, k, v, scale=scale, causal=causal, **kw)

    def backward(self, q, k, v, o, lse, do, scale, causal, drop=None):
        kw = {} if drop is None else dict(dropout_p=drop[0], seed=drop[1], dropout_row0=drop[2],
                                          dropout_key0=drop[3])
        return self.fa.backward_general(q, k, v, o, lse, do, scale=scale, causal=causal, **kw)

    def zeros_acc(self, like):
        import torch
        return torch.zeros(like.shape, dtype=torch.float32, device=like.device)

    def empty_lse(self, q):
        import torch
        return torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)

    def merge(self, o_acc, lse_acc, o_part, lse_part):
        self.fa.merge_partial(o_acc, lse_acc, o_part, lse_part)

    def accumulate(self, acc, part):
        self.fa.accumulate_bf16(acc, part)

    def finish(self, acc):
        return self.fa.convert_f32_bf16(acc)


def _drop(dropout_p, seed, rank, c, n):
    """The kernels' dropout argument for queries of chunk `rank`, keys of chunk c."""
    if not dropout_p:
        return None
    if n % 8:
        raise ValueError("dropout in the ring needs a chunk length that is a multiple of 8")
    return (dropout_p, seed, rank * n, c * n)


def ring_forward(rank, world, q, k, v, scale, causal, kern, dropout_p=0.0, seed=0):
    """Generator of one rank's forward.  Yields ("start", tensors): send them to
    rank + 1 and answer with same-shaped buffers that will receive rank - 1's;
    then ("wait",): answer once those have arrived.  Returns (O, LSE)."""
    n = q.shape[-2]
    o_acc = kern.zeros_acc(q)
    lse_acc = kern.empty_lse(q)
    cur = [k, v]
    for s in range(world):
        c = (rank - s) % world
        last = s + 1 == world
        nxt = None if last else (yield ("start", cur))
        if not causal or c <= rank:
            o_p, l_p = kern.forward(q, cur[0], cur[1], scale, causal and c == rank,
                                    _drop(dropout_p, seed, rank, c, n))
            kern.merge(o_acc, lse_acc, o_p, l_p)
        if not last:
            yield ("wait",)
            cur = nxt
    return kern.finish(o_acc), lse_acc


def ring_backward(rank, world, q, k, v, o, lse, do, scale, causal, kern, dropout_p=0.0, seed=0):
    """Generator of one rank's backward (same protocol as ring_forward).
    Returns (dQ, dK, dV) of this rank's chunk."""
    n = q.shape[-2]
    dq_acc = kern.zeros_acc(q)
    acc = [kern.zeros_acc(k), kern.zeros_acc(v)]  # dK, dV of the chunk held now
    cur = [k, v]
    for s in range(world):
        c = (rank - s) % world
        last = s + 1 == world
        nxt = None if last else (yield ("start", cur))
        if not causal or c <= rank:
            dq_p, dk_p, dv_p = kern.backward(q, cur[0], cur[1], o, lse, do, scale,
                                             causal and c == rank,
                                             _drop(dropout_p, seed, rank, c, n))
            kern.accumulate(dq_acc, dq_p)
            kern.accumulate(acc[0], dk_p)
            kern.accumulate(acc[1], dv_p)
        if not last:
            yield ("wait",)
            cur = nxt
        if world > 1:
            # the chunk's accumulators follow it; after the last step they go home
            acc = yield ("start", acc)
            yield ("wait",)
    return kern.finish(dq_acc), kern.finish(acc[0]), kern.finish(acc[1])


def run_ring(gen, group=None):
    """Drives one rank's generator over torch.distributed point-to-point
    transfers (NCCL on GPUs, gloo on CPUs); returns the generator's result."""
    import torch
    import torch.distributed as dist

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt = dist.get_global_rank(group, nxt)
        prv = dist.get_global_rank(group, prv)
    works = []
    try:
        msg = next(gen)
        while True:
            if msg[0] == "start":
                send = msg[1]
                recv = [torch.empty_like(t) for t in send]
                ops = [dist.P2POp(dist.isend, t, nxt, group) for t in send]
                ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
                works = dist.batch_isend_irecv(ops)
                msg = gen.send(recv)
            else:
                for w in works:
                    w.wait()
                works = []
                msg = gen.send(None)
    except StopIteration as e:
        return e.value


def run_emulated(gens):
    """Drives the generators of all W ranks in one process, in lock step:
    at each exchange rank r receives a copy of rank r - 1's tensors."""
    world = len(gens)
    results = [None] * world
    msgs = []
    for r, g in enumerate(gens):
        try:
            msgs.append(next(g))
        except StopIteration as e:
            msgs.append(None)
            results[r] = e.value
    while any(m is not None for m in msgs):
        kinds = {m[0] for m in msgs if m is not None}
        if len(kinds) != 1 or any(m is None for m in msgs):
            raise RuntimeError("ranks left lock step")
        if kinds == {"start"}:
            sends = [m[1] for m in msgs]
            answers = [[t.clone() for t in sends[(r - 1) % world]] for r in range(world)]
        else:
            answers = [None] * world
        for r, g in enumerate(gens):
            try:
                msgs[r] = g.send(answers[r])
            except StopIteration as e:
                msgs[r] = None
                results[r] = e.value
    return results


def attention_forward(q, k, v, scale=None, causal=False, group=None, kern=None, dropout_p=0.0,
                      seed=0):
    """This rank's chunk of O and LSE: q, k, v are its [B, H, N / W, d] chunks."""
    import torch.distributed as dist
    kern = kern or LibraryKernels()
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    return run_ring(ring_forward(dist.get_rank(group), dist.get_world_size(group), q, k, v,
                                 scale, causal, kern, dropout_p, seed), group)


def attention_backward(q, k, v, o, lse, do, scale=None, causal=False, group=None, kern=None,
                       dropout_p=0.0, seed=0):
    """This rank's chunk of dQ, dK, dV (O, LSE from attention_forward; the
    same dropout_p and seed)."""
    import torch.distributed as dist
    kern = kern or LibraryKernels()
    scale = q.shape[-1] ** -0.5 if scale is None else scale
    return run_ring(ring_backward(dist.get_rank(group), dist.get_world_size(group), q, k, v, o,
                                  lse, do, scale, causal, kern, dropout_p, seed), group)
