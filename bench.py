#!/usr/bin/env python
"""Throughput of exact attention (forward + backward) on B200.

One step = one forward (fa_fwd) and one backward (fa_bwd_prepare,
fa_bwd_main, fa_bwd_finish) over one batch of the workload, with every input
already resident in device memory.  Timing: W untimed warm-up steps, then K
steps, each bracketed by CUDA events on the launching stream, with a 256 MiB
write between steps so that no step finds its inputs in the 126 MB L2.  A
barrier and a device synchronisation bracket the K steps; the reported time is
the maximum over ranks.

Rank r of an N-rank run (torchrun, one process per GPU) processes its own
batch of the workload (independent (b, h) problems, no collective on the data
path): weak scaling.  ``value`` is the FLOPs of all ranks divided by that time.

FLOPs are counted as 4 B H N^2 d for the forward, 2.5 times that for the
backward, both halved under a causal mask.

``--impl reference`` times the float64 CPU oracle instead (on rank 0 only):
each step is one (b, h) head of the same workload, forward and backward.
"""

from __future__ import annotations

import argparse
import hashlib
import json
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
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "fwd_kernel": ["fa_fwd.cu", "ptx.cuh", "philox.cuh"],
    "bwd_main_kernel": ["fa_bwd.cu", "ptx.cuh", "philox.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="gpt2")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (profiling / scaling studies)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (profiling / scaling studies)")
    ap.add_argument("--dropout", type=float, default=None,
                    help="override the workload's dropout probability (ablation studies)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="bound on the CPU-oracle sample timed beside the GPU run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def workload_config(w, rank_batch=None):
    cfg = {
        "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d}"
                    + (" causal" if w.causal else "")
                    + (f" dropout={w.dropout_p}" if w.dropout_p else "")
                    + (f" key-lengths U[{w.seqlen_range[0]},{w.seqlen_range[1]}]"
                       if w.seqlen_range else "")
                    + (f" block-mask diag+{w.block_density:g}" if w.block_density else ""),
        "B": w.B if rank_batch is None else rank_batch, "H": w.H, "N": w.N, "d": w.d,
        "causal": w.causal, "dropout_p": w.dropout_p, "scale": w.scale,
        "seqlen_range": w.seqlen_range, "block_density": w.block_density,
        "l2": "flushed: 256 MiB write before every timed step",
        "flops": "fwd 4*B*H*N^2*d, bwd 2.5x, halved if causal (nominal count)",
    }
    return cfg


def effective_fraction(inp, w):
    """Share of the nominal (query, key) pairs the masks leave (for context)."""
    import numpy as np
    N = w.N
    frac = 1.0
    if inp["seqlens"] is not None:
        frac *= float(np.mean(inp["seqlens"])) / N
    if inp["block_mask"] is not None:
        frac *= float(inp["block_mask"].mean())
    return frac


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "io_aware_exact_20_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
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


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
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
            time.sleep(0.02)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "source": "nvml"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


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


def time_oracle_heads(w, inp, seconds=None, heads=None):
    """Runs the oracle forward + backward head by head.  Stops after ``seconds``
    (at least one head) or after the listed heads.  Returns (flops, elapsed,
    heads done)."""
    import numpy as np
    from oracle import attention_backward, attention_forward

    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    q, k, v, do = (f64(inp[x]) for x in ("q", "k", "v", "do"))
    B, H = q.shape[0], q.shape[1]
    order = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    ff, fb = attention_flops(1, 1, w.N, w.d, w.causal)
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    for bh in order:
        kw = dict(causal=w.causal, seqlens=inp["seqlens"], dropout_p=w.dropout_p,
                  seed=w.dropout_seed, block_mask=inp["block_mask"], heads=[bh])
        attention_forward(q, k, v, w.scale, **kw)
        attention_backward(q, k, v, do, w.scale, **kw)
        done += 1
        flops += ff + fb
        if seconds is not None and time.perf_counter() - t0 >= seconds:
            break
    return flops, time.perf_counter() - t0, done


# ---------------------------------------------------------------------------
# reference arm: the oracle as it stands, on the host cores
# ---------------------------------------------------------------------------

def selected_workload(args):
    from dataclasses import replace
    w = WORKLOADS[args.workload]
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


def rank_workload(w, rank):
    """The workload one rank runs: the same shape, its own batch of data (the
    data seed is shifted by the rank), so ranks share no (b, h) problem."""
    from dataclasses import replace
    return replace(w, data_seed=w.data_seed + 7919 * rank)


def max_over_ranks(x, world, device):
    """Largest value of x over all ranks (the whole job ends with the slowest)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, flops_per_step, steps, total_ms):
    """Whole-job TFLOP/s: every rank ran `steps` steps of `flops_per_step`."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = selected_workload(args)
    inp = make_inputs(w, B=1)
    heads = [(0, h % w.H) for h in range(max(1, args.warmup + args.steps))]
    for i in range(args.warmup):
        time_oracle_heads(w, inp, heads=[heads[i]])
    fl, el, n = time_oracle_heads(w, inp, heads=heads[args.warmup:args.warmup + args.steps])
    value = fl / el / 1e12
    cores = oracle_threads()
    sample = "one (b, h) head of the workload per step, forward + backward, float64 numpy"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / max(n, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, rank_batch=1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

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

    w = selected_workload(args)
    inp = make_inputs(rank_workload(w, rank))
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))
    B, H, N, d = q.shape
    kw = dict(scale=w.scale, causal=w.causal, seqlens=inp["seqlens"], dropout_p=w.dropout_p,
              seed=w.dropout_seed, block_mask=inp["block_mask"])
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    (prep, main, fin), (dq, dk, dv), keep = fa.backward_phases(q, k, v, o, lse, do, **kw)
    sl, bm, ws = keep
    fkw = dict(kw, seqlens=sl, block_mask=bm)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.forward(q, k, v, out=o, lse=lse, **fkw)
        if ev is not None:
            ev[1].record(stream)
        prep()
        if ev is not None:
            ev[2].record(stream)
        main()
        if ev is not None:
            ev[3].record(stream)
        fin()
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    st = fa.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up is {st}, not ok")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(events[i])
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    status = fa.last_device_status()
    launches = 4 * args.steps

    step_ms = [e[0].elapsed_time(e[4]) for e in events]
    fwd_ms = [e[0].elapsed_time(e[1]) for e in events]
    pre_ms = [e[1].elapsed_time(e[2]) for e in events]
    main_ms = [e[2].elapsed_time(e[3]) for e in events]
    post_ms = [e[3].elapsed_time(e[4]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    f_fwd, f_bwd = attention_flops(B, H, N, d, w.causal)
    value = job_throughput(world, f_fwd + f_bwd, args.steps, total_ms)
    peaks, peak_src = read_peaks()
    peak = float(peaks["bf16_tflops"])
    fwd_avg, main_avg = statistics.mean(fwd_ms), statistics.mean(main_ms)
    kern = {
        "fwd_kernel": {"ms": fwd_avg, "tflops": f_fwd / (fwd_avg * 1e-3) / 1e12,
                       "flops_per_launch": f_fwd},
        "bwd_main_kernel": {"ms": main_avg, "tflops": f_bwd / (main_avg * 1e-3) / 1e12,
                            "flops_per_launch": f_bwd},
        "bwd_pre_kernel": {"ms": statistics.mean(pre_ms)},
        "bwd_post_kernel": {"ms": statistics.mean(post_ms)},
    }
    dom = "bwd_main_kernel" if main_avg >= fwd_avg else "fwd_kernel"
    ach = kern[dom]["tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak, "traffic": recorded_traffic(dom, w.name),
                "peak_source": f"{peak_src} bf16_tflops (burst; cuBLAS bf16 GEMM)",
                "per_kernel": kern}

    # ------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (inp[x].pin_memory() for x in ("q", "k", "v", "do"))
        ho, hdq, hdk, hdv = (torch.empty_like(hq).pin_memory() for _ in range(4))
        hlse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        n_e2e = max(1, min(args.steps, 50))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            do.copy_(hdo, non_blocking=True)
            fa.forward(q, k, v, out=o, lse=lse, **fkw)
            fa.backward(q, k, v, o, lse, do, workspace=ws, dq=dq, dk=dk, dv=dv, **fkw)
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
            hdq.copy_(dq, non_blocking=True)
            hdk.copy_(dk, non_blocking=True)
            hdv.copy_(dv, non_blocking=True)

        for _ in range(2):
            flush.zero_()
            e2e_step()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_e2e)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev)
        nb = q.numel() * q.element_size()
        e2e = {"value": job_throughput(world, f_fwd + f_bwd, n_e2e, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": 4 * nb,
               "d2h_bytes_per_step": 4 * nb + lse.numel() * lse.element_size(),
               "steps": n_e2e, "ms_per_step": e_ms / n_e2e}

    # ------------------------------------------------------ CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        fl, el, n = time_oracle_heads(w, inp, seconds=args.cpu_seconds)
        cpu = {"value": fl / el / 1e12, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{n} of {B * H} (b, h) heads of the workload, forward + backward, "
                         f"float64 numpy, {el:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(w),
            "pct_of_peak": 100.0 * value / peak,
            "fwd_tflops": kern["fwd_kernel"]["tflops"],
            "bwd_tflops": f_bwd / ((main_avg + statistics.mean(pre_ms)
                                    + statistics.mean(post_ms)) * 1e-3) / 1e12,
            "effective_pair_fraction": effective_fraction(inp, w),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk.summary(), "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
