#!/usr/bin/env python
"""Throughput of exact attention (forward + backward) on B200.

One step = one forward (fa_fwd) and one backward (fa_bwd_prepare,
fa_bwd_main, fa_bwd_finish) over one batch of a workload, with every input
already resident in device memory.  Timing: W untimed warm-up steps, then the
timed steps, each bracketed by CUDA events on the launching stream, with a
256 MiB write between steps so that no step finds its inputs in the 126 MB
L2.  A barrier and a device synchronisation bracket the timed steps; the
reported time is the maximum over ranks.  Nothing is recorded between the
launches of a timed step (the library's kernels may start launching under
their predecessor's last wave); the per-launch split comes from a second
pass of the same steps with an event between every two launches.

The default run times every workload (tiny, GPT-2, BERT, long d=64, long
d=128, long d=256, block-sparse) one after the other, plus the BERT batch
packed and the long d=128 workload with grouped K / V heads (4 for the 16
query heads) through the general entry points.  The headline ``value`` is the
dense long-sequence case (B=1 H=16 N=16384 d=128 causal) timed over exactly
K steps; ``per_config`` holds each workload (that one included, timed again
for at least half a second so the clock record has many samples) with its
forward, backward and fwd+bwd TFLOP/s, nominal and effective, the dominant
kernel against the roofline, the clocks seen, and the float64 CPU oracle on
a bounded sample.  For the GPT-2 and long d=128 workloads the unfused
standard-attention program (separate PyTorch matmul / mask / softmax /
dropout / matmul kernels) is timed beside it on the same inputs.

FLOPs: nominal = 4 B H N^2 d for the forward, 2.5 times that for the
backward, halved under a causal mask.  Effective = nominal times the share of
(query, key) pairs the masks leave (mean key length / N under key padding,
the realised block density under a block mask); it is the count the roofline
fraction uses, so that a block-sparse run cannot read above the peak.

Rank r of an N-rank run (torchrun, one process per GPU) processes its own
batch of every workload (independent (b, h) problems, no collective on the
data path): weak scaling.  ``value`` is the FLOPs of all ranks divided by the
slowest rank's time.

``--impl reference`` times the float64 CPU oracle instead (rank 0 only), on
the headline workload: each step is one 256-row query slab of one (b, h)
head, forward and backward.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from io_aware_exact_20_b200.workloads import WORKLOADS, attention_flops, make_inputs  # noqa: E402

METRIC = "attention fwd+bwd TFLOP/s (bf16, N=512–64K) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
HEADLINE = "long128"
ORDER = ["tiny", "gpt2", "bert", "long64", "long128", "long256", "sparse"]
UNFUSED_CONFIGS = ("gpt2", "long128")
FLUSH_BYTES = 256 << 20
# per_config entries through fa_fwd_ex / fa_bwd_ex: name -> (workload, case class)
GENERAL_CASES = {"bert_packed": ("bert", "PackedCase"), "long128_gqa4": ("long128", "GqaCase")}
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "fwd_kernel": ["fa_fwd.cu", "ptx.cuh", "philox.cuh", "kernels.h"],
    "bwd_main_kernel": ["fa_bwd.cu", "ptx.cuh", "philox.cuh", "kernels.h"],
}
SLAB = 256  # rows of one CPU-oracle sample
PROJ_SHAPES = {
    # fused QKV projection measurements, name: (B, N, H, d, d_model)
    "qkv_proj_gpt2": (8, 1024, 12, 64, 768),
    "qkv_proj_long128": (1, 16384, 16, 128, 2048),
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all"] + sorted(WORKLOADS) + sorted(PROJ_SHAPES)
                    + sorted(GENERAL_CASES),
                    default="all",
                    help="'all' (default): headline plus every workload in per_config; a name: "
                         "that workload alone as the headline (profiling); a qkv_proj_* name: "
                         "that fused-projection measurement alone; bert_packed / long128_gqa4: "
                         "that general-layout per_config entry alone")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch size (single-workload profiling only)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the sequence length (single-workload profiling only)")
    ap.add_argument("--dropout", type=float, default=None,
                    help="override the dropout probability (single-workload ablations only)")
    ap.add_argument("--min-seconds", type=float, default=0.5,
                    help="shortest timed region of each per_config entry")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="bound on the CPU-oracle sample of the headline workload")
    ap.add_argument("--cpu-seconds-per-config", type=float, default=2.0,
                    help="bound on the CPU-oracle sample of each per_config entry")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-unfused", action="store_true")
    ap.add_argument("--unfused-sweep", action="store_true",
                    help="instead of the bench line: fused vs unfused time and peak memory "
                         "for N = 1K..32K (B=1 H=4 d=128 causal)")
    args = ap.parse_args(argv)
    if (args.workload == "all" or args.workload in PROJ_SHAPES
            or args.workload in GENERAL_CASES) and (
            args.batch or args.seqlen or args.dropout is not None):
        ap.error("--batch/--seqlen/--dropout need a single attention --workload")
    return args


# ---------------------------------------------------------------------------
# workload bookkeeping (host only)
# ---------------------------------------------------------------------------

def describe(w):
    return (f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d}"
            + (" causal" if w.causal else "")
            + (f" dropout={w.dropout_p}" if w.dropout_p else "")
            + (f" key-lengths U[{w.seqlen_range[0]},{w.seqlen_range[1]}]" if w.seqlen_range else "")
            + (f" block-mask diag+{w.block_density:g}" if w.block_density else ""))


def workload_config(w, rank_batch=None):
    return {
        "workload": describe(w),
        "B": w.B if rank_batch is None else rank_batch, "H": w.H, "N": w.N, "d": w.d,
        "causal": w.causal, "dropout_p": w.dropout_p, "scale": w.scale,
        "seqlen_range": w.seqlen_range, "block_density": w.block_density,
        "l2": "flushed: 256 MiB write before every timed step",
        "flops": "nominal: fwd 4*B*H*N^2*d, bwd 2.5x, halved if causal; "
                 "effective: nominal x share of (query, key) pairs the masks leave",
    }


def effective_fraction(inp, w):
    """Share of the nominal (query, key) pairs the masks leave: mean key
    length / N under key padding, realised block density under a block mask."""
    import numpy as np
    frac = 1.0
    if inp.get("seqlens") is not None:
        frac *= float(np.mean(np.clip(inp["seqlens"], 0, w.N))) / w.N
    if inp.get("block_mask") is not None:
        frac *= float(np.asarray(inp["block_mask"]).astype(bool).mean())
    return frac


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        float(d["bf16_tflops"])
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def source_sha(files):
    """Hash of the kernel sources with their comments and blank space removed
    (a comment-only edit builds the same kernel and keeps its records)."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "io_aware_exact_20_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's
    sources are unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        r = rec[kernel][workload]
    except Exception:
        return None
    if r.get("source_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return r.get("bytes_per_launch")


def tflops(flops, ms):
    return flops / (ms * 1e-3) / 1e12 if ms > 0 else None


def job_throughput(world, flops_per_step, steps, total_ms):
    """Whole-job TFLOP/s: every rank ran `steps` steps of `flops_per_step`."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def rank_workload(w, rank):
    """The workload one rank runs: the same shape, its own batch of data (the
    data seed is shifted by the rank), so ranks share no (b, h) problem."""
    from dataclasses import replace
    return replace(w, data_seed=w.data_seed + 7919 * rank)


def selected_workload(name, args=None):
    from dataclasses import replace
    w = WORKLOADS[name]
    if args is None:
        return w
    if args.batch is not None:
        w = replace(w, B=args.batch)
    if args.seqlen is not None:
        lens = w.seqlen_range
        if lens is not None:
            lens = (min(lens[0], args.seqlen), min(lens[1], args.seqlen))
        w = replace(w, N=args.seqlen, seqlen_range=lens)
    if args.dropout is not None:
        w = replace(w, dropout_p=args.dropout)
    return w


def max_over_ranks(x, world, device):
    """Largest value of x over all ranks (the whole job ends with the slowest)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kernel_summary(w, eff, fwd_ms, pre_ms, main_ms, post_ms, peak, traffic_key=None,
                   step_ms=None):
    """Per-kernel and per-pass TFLOP/s (nominal and effective) of one workload
    and its dominant kernel against the peak (effective count).  step_ms: the
    step timed without events between its launches (default: their sum)."""
    f_fwd, f_bwd = attention_flops(w.B, w.H, w.N, w.d, w.causal)
    bwd_ms = pre_ms + main_ms + post_ms
    tot_ms = fwd_ms + bwd_ms if step_ms is None else step_ms
    out = {
        "ms": {"fwd": fwd_ms, "bwd_pre": pre_ms, "bwd_main": main_ms, "bwd_post": post_ms,
               "step": tot_ms, "step_with_events_between_launches": fwd_ms + bwd_ms},
        "nominal_tflops": {"fwd": tflops(f_fwd, fwd_ms), "bwd_main": tflops(f_bwd, main_ms),
                           "bwd": tflops(f_bwd, bwd_ms), "fwd_bwd": tflops(f_fwd + f_bwd, tot_ms)},
        "effective_tflops": {"fwd": tflops(eff * f_fwd, fwd_ms),
                             "bwd_main": tflops(eff * f_bwd, main_ms),
                             "bwd": tflops(eff * f_bwd, bwd_ms),
                             "fwd_bwd": tflops(eff * (f_fwd + f_bwd), tot_ms)},
        "effective_pair_fraction": eff,
        "flops_per_launch": {"fwd_kernel": f_fwd, "bwd_main_kernel": f_bwd},
    }
    dom = "bwd_main_kernel" if main_ms >= fwd_ms else "fwd_kernel"
    ach = tflops(eff * out["flops_per_launch"][dom], main_ms if dom == "bwd_main_kernel" else fwd_ms)
    out["dominant"] = {"kernel": dom, "achieved_effective_tflops": ach, "peak": peak,
                       "frac": ach / peak,
                       "traffic": recorded_traffic(dom, traffic_key or w.name)}
    out["pct_of_peak"] = {k: (100.0 * v / peak if v is not None else None)
                          for k, v in out["effective_tflops"].items()}
    return out


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index, interval_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - reported, not fatal
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(self.interval)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()
        if self._h is not None and not self.samples:
            try:  # a region shorter than one interval still gets one sample
                self._sample()
            except Exception:
                pass

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml"}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline; test infrastructure, not product)
# ---------------------------------------------------------------------------

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def oracle_slab(w, inp, b, h, r0, rows=SLAB):
    """Forward and backward work of one query slab of one head in the oracle:
    O and LSE of the slab's rows, their dQ rows, and the slab's contribution
    to dK and dV of every key (the backward is the sum of these over slabs).
    Returns the nominal FLOPs the slab stands for."""
    import numpy as np
    from oracle import head_backward_cols, head_backward_rows, head_forward_rows

    f64 = lambda t: t[b, h].float().numpy().astype(np.float64)  # noqa: E731
    q, k, v, do = (f64(inp[x]) for x in ("q", "k", "v", "do"))
    rr = np.arange(r0, min(w.N, r0 + rows))
    kv_len = None if inp["seqlens"] is None else int(inp["seqlens"][b])
    kw = dict(causal=w.causal, kv_len=kv_len, block_mask=inp["block_mask"],
              dropout_p=w.dropout_p, seed=w.dropout_seed, b=b, h=h)
    head_forward_rows(q, k, v, w.scale, rr, **kw)
    head_backward_rows(q, k, v, do, w.scale, rr, **kw)
    head_backward_cols(q, k, v, do, w.scale, np.arange(w.N), rows=rr, **kw)
    ff, fb = attention_flops(1, 1, w.N, w.d, w.causal)
    return (ff + fb) * rr.size / w.N


def time_oracle(w, inp, seconds, max_slabs=None):
    """Oracle slabs of the workload (heads in order, slabs in order) until
    `seconds` have passed (at least one slab).  Returns (flops, s, slabs)."""
    per_head = math.ceil(w.N / SLAB)
    B = inp["q"].shape[0]
    units = [(b, h, s * SLAB) for b in range(B) for h in range(w.H) for s in range(per_head)]
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    for (b, h, r0) in units:
        flops += oracle_slab(w, inp, b, h, r0)
        done += 1
        if max_slabs is not None and done >= max_slabs:
            break
        if time.perf_counter() - t0 >= seconds:
            break
    return flops, time.perf_counter() - t0, done, len(units)


def cpu_baseline(w, inp, seconds):
    fl, el, n, total = time_oracle(w, inp, seconds)
    return {"value": fl / el / 1e12, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} of {total} {SLAB}-row query slabs of the workload's heads "
                      f"(forward + backward of each slab), float64 numpy, {el:.1f} s; "
                      f"FLOPs counted as the slab's share of the nominal count"}


# ---------------------------------------------------------------------------
# reference arm: the oracle as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    single = args.workload in WORKLOADS
    name = args.workload if single else HEADLINE
    w = selected_workload(name, args if single else None)
    inp = make_inputs(w, B=1)
    per_head = math.ceil(w.N / SLAB)
    units = [(0, h, s * SLAB) for h in range(w.H) for s in range(per_head)]
    units = [units[i % len(units)] for i in range(args.warmup + args.steps)]
    for (b, h, r0) in units[:args.warmup]:
        oracle_slab(w, inp, b, h, r0)
    t0 = time.perf_counter()
    fl = 0.0
    for (b, h, r0) in units[args.warmup:]:
        fl += oracle_slab(w, inp, b, h, r0)
    el = time.perf_counter() - t0
    value = fl / el / 1e12
    sample = (f"one {SLAB}-row query slab of one (b, h) head of the workload per step "
              f"(forward + backward of the slab), float64 numpy; FLOPs counted as the "
              f"slab's share of the nominal count")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, rank_batch=1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Case:
    """One workload resident on the device, with its four launches bound."""

    def __init__(self, fa, w, rank, dev):
        import torch
        self.w = w
        self.inp = make_inputs(rank_workload(w, rank))
        self.eff = effective_fraction(self.inp, w)
        self.q, self.k, self.v, self.do = (self.inp[x].to(dev) for x in ("q", "k", "v", "do"))
        B, H, N, d = self.q.shape
        self.kw = dict(scale=w.scale, causal=w.causal, seqlens=self.inp["seqlens"],
                       dropout_p=w.dropout_p, seed=w.dropout_seed,
                       block_mask=self.inp["block_mask"])
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        (self.prep, self.main, self.fin), (self.dq, self.dk, self.dv), keep = \
            fa.backward_phases(self.q, self.k, self.v, self.o, self.lse, self.do, **self.kw)
        sl, bm, self.ws = keep
        self.fkw = dict(self.kw, seqlens=sl, block_mask=bm)
        self.fa = fa

    def step(self, stream, ev=None):
        fa = self.fa
        if ev is not None:
            ev[0].record(stream)
        fa.forward(self.q, self.k, self.v, out=self.o, lse=self.lse, **self.fkw)
        if ev is not None:
            ev[1].record(stream)
        self.prep()
        if ev is not None:
            ev[2].record(stream)
        self.main()
        if ev is not None:
            ev[3].record(stream)
        self.fin()
        if ev is not None:
            ev[4].record(stream)


class PackedCase:
    """The BERT-shaped workload stored packed (fa_fwd_ex / fa_bwd_ex): every
    sequence's rows back to back, no padding rows, so no query row beyond a
    sequence's length is computed.  The backward's three launches are one
    call here, timed as one."""

    def __init__(self, fa, w, rank, dev):
        import numpy as np
        import torch
        self.w = w
        self.inp = make_inputs(rank_workload(w, rank))
        lens = np.asarray(self.inp["seqlens"], dtype=np.int64)
        self.lens = lens
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        pack = lambda x: torch.cat([x[b, :, :n].transpose(0, 1) for b, n in enumerate(lens)])  # noqa
        self.q, self.k, self.v, self.do = (pack(self.inp[x]).contiguous().to(dev)
                                           for x in ("q", "k", "v", "do"))
        T, H, d = self.q.shape
        self.kw = dict(layout="thd", cu_seqlens_q=torch.as_tensor(cu, device=dev),
                       cu_seqlens_k=torch.as_tensor(cu, device=dev), max_seqlen_q=w.N,
                       max_seqlen_k=w.N, scale=w.scale, causal=w.causal, dropout_p=w.dropout_p,
                       seed=w.dropout_seed)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.ws = torch.empty(fa.general_workspace_size(self.q, self.k, **self.kw),
                              dtype=torch.uint8, device=dev)
        self.fa = fa
        f = 4.0 * H * d * float((lens.astype(np.float64) ** 2).sum())
        self.flops = (f, 2.5 * f)

    def step(self, stream, ev=None):
        fa = self.fa
        if ev is not None:
            ev[0].record(stream)
        fa.forward_general(self.q, self.k, self.v, out=self.o, lse=self.lse, **self.kw)
        if ev is not None:
            ev[1].record(stream)
            ev[2].record(stream)
        fa.backward_general(self.q, self.k, self.v, self.o, self.lse, self.do, dq=self.dq,
                            dk=self.dk, dv=self.dv, workspace=self.ws, **self.kw)
        if ev is not None:
            ev[3].record(stream)
            ev[4].record(stream)


class GqaCase(PackedCase):
    """The long causal d=128 workload with grouped K / V heads (4 K / V heads
    for the 16 query heads: each shared by a group of 4), through fa_fwd_ex /
    fa_bwd_ex.  The FLOPs are those of the same attention without grouping."""

    KV_HEADS = 4

    def __init__(self, fa, w, rank, dev):
        import torch
        self.w = w
        inp = make_inputs(rank_workload(w, rank))
        self.q, self.do = (inp[x].contiguous().to(dev) for x in ("q", "do"))
        self.k, self.v = (inp[x][:, :self.KV_HEADS].contiguous().to(dev) for x in ("k", "v"))
        self.kw = dict(scale=w.scale, causal=w.causal, dropout_p=w.dropout_p,
                       seed=w.dropout_seed)
        B, H, N, d = self.q.shape
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(x) for x in (self.q, self.k, self.v))
        self.ws = torch.empty(fa.general_workspace_size(self.q, self.k, **self.kw),
                              dtype=torch.uint8, device=dev)
        self.fa = fa
        f = attention_flops(B, H, N, d, w.causal)[0]
        self.flops = (f, 2.5 * f)


def measure_packed(fa, w, args, rank, dev, flush, stream, world, local, peak, case_cls=None):
    """per_config entry of the packed BERT-shaped batch (or, with case_cls, of
    another fa_fwd_ex / fa_bwd_ex case)."""
    import torch
    case = (case_cls or PackedCase)(fa, w, rank, dev)
    for _ in range(args.warmup):
        flush.zero_()
        case.step(stream)
    torch.cuda.synchronize(dev)
    steps = args.steps
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        flush.zero_()
        case.step(stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    est_ms = a.elapsed_time(b) / 3
    steps = int(min(5000, max(args.steps, math.ceil(args.min_seconds * 1e3 / max(est_ms, 1e-3)))))
    steps = int(max_over_ranks(steps, world, dev))
    (fwd_ms, _, bwd_ms, _), total_ms, clocks = timed_region(case, steps, flush, stream, dev, world,
                                                           local)
    f_fwd, f_bwd = case.flops
    if isinstance(case, GqaCase):
        label = describe(w) + f" with {case.KV_HEADS} K / V heads (fa_fwd_ex / fa_bwd_ex)"
        note = "as the same attention without grouping: 4 B H N^2 d forward, 2.5x backward, halved causal"
    else:
        label = describe(w) + " packed (fa_fwd_ex / fa_bwd_ex, no padding rows)"
        note = "4 H d sum_b len_b^2 forward, 2.5x backward: every counted pair is valid"
    entry = {"workload": label,
             "steps": steps, "timed_s": total_ms * 1e-3, "clocks": clocks,
             "device_status": fa.last_device_status(),
             "ms": {"fwd": fwd_ms, "bwd": bwd_ms, "step": total_ms / steps,
                    "step_with_events_between_launches": fwd_ms + bwd_ms},
             "flops_per_launch": {"fwd_kernel": f_fwd, "bwd (3 launches)": f_bwd},
             "tflops": {"fwd": tflops(f_fwd, fwd_ms), "bwd": tflops(f_bwd, bwd_ms),
                        "fwd_bwd": tflops(f_fwd + f_bwd, total_ms / steps)},
             "flops": note}
    if not isinstance(case, GqaCase):
        entry["tokens"] = int(case.lens.sum())
    entry["pct_of_peak"] = {k: 100.0 * v / peak for k, v in entry["tflops"].items()}
    del case
    torch.cuda.empty_cache()
    return entry


def measure_projection(fa, name, args, rank, dev, flush, stream, world, local, peak):
    """The fused QKV projection (one kernel: GEMM + head-major epilogue) against
    the unfused program (cuBLAS linear, then a permute copy into [B, H, N, d])."""
    import torch
    B, N, H, d, dm = PROJ_SHAPES[name]
    g = torch.Generator(device="cpu").manual_seed(5)
    x = torch.randn(B * N, dm, generator=g).to(torch.bfloat16).to(dev)
    w = (torch.randn(3 * H * d, dm, generator=g) / dm ** 0.5).to(torch.bfloat16).to(dev)
    bias = torch.randn(3 * H * d, generator=g).to(torch.bfloat16).to(dev)
    outs = [torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev) for _ in range(3)]

    def fused():
        fa.qkv_projection(x, w, bias, B, H, d, *outs)

    def unfused():
        y = torch.nn.functional.linear(x, w, bias)
        return y.view(B, N, 3, H, d).permute(2, 0, 3, 1, 4).contiguous()

    def run(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        n = int(min(5000, max(args.steps, math.ceil(args.min_seconds * 1e3 /
                                                   max(a.elapsed_time(b) + 0.05, 1e-3)))))
        n = int(max_over_ranks(n, world, dev))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        with ClockSampler(local) as clk:
            for e0, e1 in ev:
                flush.zero_()
                e0.record(stream)
                fn()
                e1.record(stream)
            torch.cuda.synchronize(dev)
        return max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in ev) / n, world, dev), n, clk

    ms, n, clk = run(fused)
    ms_u, n_u, _ = run(unfused)
    flops = 2.0 * B * N * dm * 3 * H * d
    alg_bytes = 2.0 * (B * N * dm + 3 * H * d * dm + 3 * B * N * H * d + 3 * H * d)
    ach = tflops(flops, ms)
    return {"shape": f"x [{B * N}, {dm}] @ w[{3 * H * d}, {dm}]^T + bias -> Q, K, V "
                     f"[{B}, {H}, {N}, {d}]",
            "steps": n, "ms": ms, "tflops": ach, "roofline": {
                "bound": "tensor", "achieved": ach, "peak": peak, "frac": ach / peak,
                "algorithmic_bytes": alg_bytes, "gbs": alg_bytes / (ms * 1e-3) / 1e9},
            "clocks": clk.summary(), "device_status": fa.last_device_status(),
            "unfused": {"what": "torch linear (cuBLAS) + permute(...).contiguous()",
                        "ms": ms_u, "steps": n_u, "tflops": tflops(flops, ms_u),
                        "fused_speedup": ms_u / ms}}


def timed_region(case, steps, flush, stream, dev, world, clk_index):
    """Times `steps` steps, L2 flushed before each, in two passes: the steps
    alone, one event before and one after each (nothing between the launches,
    which may then start under their predecessor's last wave), for the step
    time; then again with an event between every two launches, for the
    per-launch split.  Returns the per-launch means of the second pass, the
    total of the first (ms, max over ranks) and the first pass's clock record."""
    import torch
    import torch.distributed as dist
    ends = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(steps)]
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(clk_index) as clk:
        for a, b in ends:
            flush.zero_()
            a.record(stream)
            case.step(stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in ends), world, dev)
    for i in range(steps):
        flush.zero_()
        case.step(stream, events[i])
    torch.cuda.synchronize(dev)
    parts = [[e[a].elapsed_time(e[a + 1]) for e in events] for a in range(4)]
    sums = [max_over_ranks(sum(p), world, dev) for p in parts]
    return [s / steps for s in sums], total, clk.summary()


def time_unfused(case, dev, flush, stream, min_seconds, world):
    """Standard attention (separate PyTorch ops, S and P in HBM) on the same
    inputs: fwd+bwd time and peak device memory."""
    import torch
    from baselines.unfused_attention import UnfusedStep
    w = case.w
    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    try:
        st = UnfusedStep(case.q, case.k, case.v, case.do, w.scale, w.causal, case.inp["seqlens"],
                         w.dropout_p, case.inp["block_mask"])
        for _ in range(2):
            st()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        st()
        b.record(stream)
        torch.cuda.synchronize(dev)
        est = a.elapsed_time(b)
        n = max(3, min(200, int(min_seconds * 1e3 / max(est, 1e-3))))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for x, y in ev:
            flush.zero_()
            x.record(stream)
            st()
            y.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in ev) / n, world, dev)
        peak = torch.cuda.max_memory_allocated(dev) - base
        del st
    except torch.OutOfMemoryError as e:  # reported, not fatal
        torch.cuda.empty_cache()
        return {"error": f"out of memory: {str(e)[:120]}"}
    torch.cuda.empty_cache()
    f_fwd, f_bwd = attention_flops(w.B, w.H, w.N, w.d, w.causal)
    return {"ms_per_step": ms, "steps": n, "nominal_tflops": tflops(f_fwd + f_bwd, ms),
            "peak_extra_bytes": int(peak),
            "what": "torch.matmul, masked_fill, softmax, dropout, matmul + autograd (bf16)"}


def fused_extra_bytes(case):
    """Device bytes the fused path needs beyond Q, K, V, dO: O, LSE, dQ, dK,
    dV and the backward workspace (all O(N))."""
    n = sum(t.numel() * t.element_size() for t in (case.o, case.lse, case.dq, case.dk, case.dv))
    return int(n + case.ws.numel() * case.ws.element_size())


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    import io_aware_exact_20_b200 as fa

    peaks, peak_src = read_peaks()
    peak = float(peaks["bf16_tflops"])
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if args.unfused_sweep:
        return run_unfused_sweep(args, fa, dev, flush, stream, world, rank)
    if args.workload in PROJ_SHAPES or args.workload in GENERAL_CASES:
        if args.workload in PROJ_SHAPES:
            r = measure_projection(fa, args.workload, args, rank, dev, flush, stream, world, local,
                                   peak)
        else:
            base, cls = GENERAL_CASES[args.workload]
            r = measure_packed(fa, WORKLOADS[base], args, rank, dev, flush, stream, world, local,
                               peak, case_cls=globals()[cls])
        if rank == 0:
            print(json.dumps({"workload": args.workload, **r}), flush=True)
        return 0

    single = args.workload != "all"
    head_name = args.workload if single else HEADLINE
    w_head = selected_workload(head_name, args if single else None)

    # ----------------------------------------------------------- headline
    case = Case(fa, w_head, rank, dev)
    for _ in range(args.warmup):
        flush.zero_()
        case.step(stream)
    torch.cuda.synchronize(dev)
    st = fa.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up is {st}, not ok")
    (fwd_ms, pre_ms, main_ms, post_ms), total_ms, clocks = timed_region(
        case, args.steps, flush, stream, dev, world, local)
    status = fa.last_device_status()
    launches = 4 * args.steps
    w = w_head
    f_fwd, f_bwd = attention_flops(w.B, w.H, w.N, w.d, w.causal)
    value = job_throughput(world, f_fwd + f_bwd, args.steps, total_ms)
    summ = kernel_summary(w, case.eff, fwd_ms, pre_ms, main_ms, post_ms, peak,
                          step_ms=total_ms / args.steps)
    dom = summ["dominant"]
    roofline = {"bound": "tensor", "kernel": dom["kernel"],
                "achieved": dom["achieved_effective_tflops"], "peak": peak, "unit": "TFLOP/s",
                "frac": dom["frac"], "traffic": dom["traffic"],
                "peak_source": f"{peak_src} bf16_tflops (burst; cuBLAS bf16 GEMM)",
                "flops": "effective count per launch / event-timed mean launch duration",
                "per_kernel_ms": summ["ms"]}

    # ------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(case, fa, args, dev, world, f_fwd + f_bwd)

    # ------------------------------------------------------ CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, case.inp, args.cpu_seconds)

    head_eff = case.eff
    del case
    torch.cuda.empty_cache()

    # ------------------------------------------------------ per workload
    per_config = {}
    if not single:
        jobs = []
        for name in ORDER:
            jobs.append((name, measure_config, WORKLOADS[name]))
            if name == "bert":
                jobs.append(("bert_packed", measure_packed, WORKLOADS[name]))
            if name == "long128":
                jobs.append(("long128_gqa4", lambda *a: measure_packed(*a, case_cls=GqaCase),
                             WORKLOADS[name]))
        for name in PROJ_SHAPES:
            jobs.append((name, measure_projection, name))
        for name, fn, wl in jobs:
            try:
                per_config[name] = fn(fa, wl, args, rank, dev, flush, stream, world, local, peak)
            except Exception as e:  # reported in the line; the other entries still run
                per_config[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
                torch.cuda.synchronize(dev)
                torch.cuda.empty_cache()
            if per_config[name].get("device_status", 0) != 0:
                status = status or per_config[name]["device_status"]

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(w),
            "pct_of_peak": 100.0 * value / peak,
            "pct_of_datasheet_dense_bf16": 100.0 * value / DATASHEET_BF16_TFLOPS,
            "fwd_tflops": summ["nominal_tflops"]["fwd"],
            "bwd_tflops": summ["nominal_tflops"]["bwd"],
            "bwd_main_tflops": summ["nominal_tflops"]["bwd_main"],
            "pct_of_peak_fwd": summ["pct_of_peak"]["fwd"],
            "pct_of_peak_bwd_main": summ["pct_of_peak"]["bwd_main"],
            "pct_of_peak_bwd": summ["pct_of_peak"]["bwd"],
            "effective_pair_fraction": head_eff,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clocks, "device_status": status, "per_config": per_config or None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def time_e2e(case, fa, args, dev, world, flops):
    """The same step through the public Python API with the inputs copied in
    from pinned host memory and every output copied back, inside the timed
    region, as a user streaming batches would run it: two device buffer sets
    alternate, so that one step's Q, K, V, dO travel in (host-to-device copy
    engine) while the step before computes and has its O, LSE, dQ, dK, dV
    copied out (device-to-host engine).  Events order each buffer's reuse:
    its inputs are rewritten once the backward that read them has run, its
    outputs once the copies that read them are done.  One region over all steps is timed, from before the first
    copy in to after the last copy out; no L2 flush, since every step's inputs
    arrive from the host."""
    import torch
    import torch.distributed as dist
    hq, hk, hv, hdo = (case.inp[x].pin_memory() for x in ("q", "k", "v", "do"))
    ho, hdq, hdk, hdv = (torch.empty_like(hq).pin_memory() for _ in range(4))
    hlse = torch.empty(tuple(case.lse.shape), dtype=torch.float32).pin_memory()
    n_e2e = max(2, min(args.steps, 50))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_comp = torch.cuda.current_stream(dev)
    names = ("q", "k", "v", "do", "o", "lse", "dq", "dk", "dv")
    bufs = [{x: getattr(case, x) for x in names},
            {x: torch.empty_like(getattr(case, x)) for x in names}]
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, fwd_done, bwd_done, out_done = ([ev(), ev()] for _ in range(4))
    used = [False, False]

    def e2e_step(i):
        b = bufs[i % 2]
        j = i % 2
        with torch.cuda.stream(s_in):
            if used[j]:
                # the buffer's inputs are free once its last step's backward ran
                s_in.wait_event(bwd_done[j])
            b["q"].copy_(hq, non_blocking=True)
            b["k"].copy_(hk, non_blocking=True)
            b["v"].copy_(hv, non_blocking=True)
            b["do"].copy_(hdo, non_blocking=True)
            in_done[j].record(s_in)
        s_comp.wait_event(in_done[j])
        if used[j]:
            # its outputs are free once its last step's results are on the host
            s_comp.wait_event(out_done[j])
        fa.forward(b["q"], b["k"], b["v"], out=b["o"], lse=b["lse"], **case.fkw)
        fwd_done[j].record(s_comp)
        fa.backward(b["q"], b["k"], b["v"], b["o"], b["lse"], b["do"], workspace=case.ws,
                    dq=b["dq"], dk=b["dk"], dv=b["dv"], **case.fkw)
        bwd_done[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done[j])
            ho.copy_(b["o"], non_blocking=True)
            hlse.copy_(b["lse"], non_blocking=True)
            s_out.wait_event(bwd_done[j])
            hdq.copy_(b["dq"], non_blocking=True)
            hdk.copy_(b["dk"], non_blocking=True)
            hdv.copy_(b["dv"], non_blocking=True)
            out_done[j].record(s_out)
        used[j] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    end.record(s_out)  # the last copy out is the last work of the region
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    nb = case.q.numel() * case.q.element_size()
    # the pipelined steps must give the resident steps' results: dK and dV
    # are deterministic, so the last step's copies equal them bit for bit
    same = bool(torch.equal(hdk, case.dk.cpu()) and torch.equal(hdv, case.dv.cpu()))
    del bufs
    return {"value": job_throughput(world, flops, n_e2e, e_ms), "unit": UNIT,
            "h2d_bytes_per_step": 4 * nb,
            "d2h_bytes_per_step": 4 * nb + case.lse.numel() * case.lse.element_size(),
            "steps": n_e2e, "ms_per_step": e_ms / n_e2e,
            "schedule": "two device buffer sets; copies in, compute and copies out of "
                        "consecutive steps overlap; every step copies all inputs in and "
                        "all outputs out",
            "dk_dv_equal_resident_step": same}


def measure_config(fa, w, args, rank, dev, flush, stream, world, local, peak):
    """One per_config entry: the workload timed for at least --min-seconds."""
    import torch
    case = Case(fa, w, rank, dev)
    for _ in range(args.warmup):
        flush.zero_()
        case.step(stream)
    torch.cuda.synchronize(dev)
    # estimate the step (with its flush) to size the timed region
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        flush.zero_()
        case.step(stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    est_ms = a.elapsed_time(b) / 3
    steps = int(min(5000, max(args.steps, math.ceil(args.min_seconds * 1e3 / max(est_ms, 1e-3)))))
    steps = int(max_over_ranks(steps, world, dev))  # every rank times the same count
    (fwd_ms, pre_ms, main_ms, post_ms), total_ms, clocks = timed_region(
        case, steps, flush, stream, dev, world, local)
    status = fa.last_device_status()
    entry = {"workload": describe(w), "steps": steps, "timed_s": total_ms * 1e-3,
             "clocks": clocks, "device_status": status}
    entry.update(kernel_summary(w, case.eff, fwd_ms, pre_ms, main_ms, post_ms, peak,
                                step_ms=total_ms / steps))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        entry["cpu_baseline"] = cpu_baseline(w, case.inp, args.cpu_seconds_per_config)
    if w.name == "tiny":
        # host cost of one fwd + bwd call pair through the Python API: wall time
        # of enqueueing 100 steps (no synchronisation inside the loop)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(100):
            case.step(stream)
        t1 = time.perf_counter()
        torch.cuda.synchronize(dev)
        entry["host_us_per_fwd_bwd_call"] = (t1 - t0) / 100 * 1e6
    if not args.no_unfused and w.name in UNFUSED_CONFIGS:
        un = time_unfused(case, dev, flush, stream, args.min_seconds, world)
        un["fused_extra_bytes"] = fused_extra_bytes(case)
        if "ms_per_step" in un:
            un["fused_speedup"] = un["ms_per_step"] / entry["ms"]["step"]
        entry["unfused"] = un
    del case
    torch.cuda.empty_cache()
    return entry


def run_unfused_sweep(args, fa, dev, flush, stream, world, rank):
    """Fused vs unfused standard attention: time and peak device memory
    against N (B=1, H=4, d=128, causal, no dropout)."""
    from dataclasses import replace

    import torch
    rows = []
    for N in (1024, 2048, 4096, 8192, 16384, 32768):
        w = replace(WORKLOADS["long128"], name=f"sweep{N}", B=1, H=4, N=N)
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        case = Case(fa, w, rank, dev)
        for _ in range(3):
            case.step(stream)
        (fwd_ms, pre_ms, main_ms, post_ms), total_ms, clocks = timed_region(
            case, 10, flush, stream, dev, world, 0)
        fused_peak = torch.cuda.max_memory_allocated(dev) - base
        un = time_unfused(case, dev, flush, stream, 0.2, world)
        f_fwd, f_bwd = attention_flops(w.B, w.H, w.N, w.d, w.causal)
        rows.append({"N": N, "fused_ms": total_ms / 10,
                     "fused_tflops": tflops(f_fwd + f_bwd, total_ms / 10),
                     "fused_peak_bytes_incl_inputs": int(fused_peak),
                     "fused_extra_bytes": fused_extra_bytes(case), "unfused": un})
        del case
    if rank == 0:
        print(json.dumps({"unfused_sweep": rows, "shape": "B=1 H=4 d=128 causal p=0"}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
