#!/usr/bin/env python
"""Benchmark of the RACE attention hot path on B200; prints one JSON line.

A step is one pass of the whole hot path over one batch of synthetic input: the
forward (soft hash, sketch build, prefix scan, readout) and the backward (dq, dk, dv,
dW) of the causal 4M-token workload (8 heads, d = 64, L = 16, P = 8, tau = 0.25,
chunk 256, clustered q/k) unless --workload says otherwise.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU: heads are independent, so every rank
processes its own batch of heads (weak scaling) and the only exchange is the sum of
dW over ranks (NCCL all-reduce), as in data-parallel training of the layer.
Timing: CUDA events on the launching stream, barrier + synchronize on both sides,
max over ranks.  Inputs (12.9 GB of q, k, v) are far larger than L2.

--impl reference times the float64 CPU oracle (the reference arm of this repo) on a
bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_lsh_sketch_race_b200 import inputs as I  # noqa: E402

METRIC = "RACE attn tokens/s (fwd, fwd+bwd) at N=4M causal; % of tensor/HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


def flops_per_token_head(wl: I.Workload):
    """Algorithmic work of the method per token and head (chunk-independent):
    forward 4*LR*(d+1) + 4*d*L*P (state build, readout, q/k projections);
    backward 10*LR*(d+1) + 12*d*L*P."""
    LR = wl.L * wl.R
    fwd = 4 * LR * (wl.d + 1) + 4 * wl.d * wl.L * wl.P
    bwd = 10 * LR * (wl.d + 1) + 12 * wl.d * wl.L * wl.P
    return fwd, bwd


def bytes_per_token_head(wl: I.Workload):
    """HBM bytes the method must move: read q, k, v, write o (forward); read q, k, v,
    o, dO, den, write dq, dk, dv (backward)."""
    es = 2 if wl.dtype == "bf16" else 4
    return 4 * wl.d * es, 8 * wl.d * es + 4


# Per-launch algorithmic flops of each kernel, as a multiple of (token-heads seen by
# one launch).  Kernels missing here are not candidates for the roofline line.
def kernel_work(name: str, wl: I.Workload):
    LR, d, L, P = wl.L * wl.R, wl.d, wl.L, wl.P
    th = wl.H * wl.N
    table = {
        "simt_readout_sweep": 4 * LR * (d + 1) + 4 * d * L * P if wl.causal else 2 * LR * (d + 1) + 2 * d * L * P,
        "simt_sketch_build": 2 * LR * (d + 1) + 2 * d * L * P,
        "simt_bwd_q": 4 * LR * (d + 1) + 8 * d * L * P,
        "simt_bwd_kv": 6 * LR * (d + 1) + 8 * d * L * P,
        "tc_causal_sweep": 4 * LR * (d + 1) + 4 * d * L * P,
        # q side: state of p(k)[v | 1] plus its readout by g'' (dP of p(q)); k side: the
        # same with the roles exchanged; both also project q and k
        "tc_bwd_q": 4 * LR * (d + 1) + 4 * d * L * P,
        "tc_bwd_k": 4 * LR * (d + 1) + 4 * d * L * P,
        "tc_sketch_build": 2 * LR * (d + 1) + 2 * d * L * P,
        "tc_readout": 2 * LR * (d + 1) + 2 * d * L * P,
    }
    if name not in table:
        return None
    return table[name] * th


# DRAM bytes (read + write) per token-head of a launch, from one ncu capture of a smaller
# launch of the same kernel and configuration (8 heads, N = 131,072, L = 16, P = 8,
# `dram__bytes_read.sum + dram__bytes_write.sum`): 946 MB per launch of the causal sweep
# (the mean of the forward's 80-column instantiation, 944 MB, and the dv pass's 64-column
# one, 948 MB: the bench's per-launch time of the sweep is the mean of the same two
# launches), 1,975 MB for the q side and 1,974 MB for the k side of the pipelined
# backward sweep.  The traffic grows in proportion to H x N.
DRAM_BYTES_PER_TOKEN_HEAD = {
    "tc_causal_sweep": (698.695e6 + 247.275e6) / (8 * 131072),
    "tc_bwd_q": (1442.38e6 + 532.65e6) / (8 * 131072),
    "tc_bwd_k": (1442.33e6 + 531.99e6) / (8 * 131072),
}


def kernel_traffic(name: str, wl: I.Workload):
    if wl.L != 16 or wl.P != 8 or name not in DRAM_BYTES_PER_TOKEN_HEAD:
        return None
    return DRAM_BYTES_PER_TOKEN_HEAD[name] * wl.H * wl.N


def roofline_lines(ktimes, wl: I.Workload, peaks, peak_src: str):
    """Roofline objects of the JSON line from the per-kernel CUDA-event totals
    ktimes = {name: (total_ms, launches)}: the dominant kernel of the step (the largest
    total among kernels with known algorithmic work) and, when that is not the forward
    sweep, the forward sweep as well; both against the sustained tensor peak."""
    def roofline_of(name):
        ms_launch = ktimes[name][0] / ktimes[name][1]
        work = kernel_work(name, wl)
        achieved = work / (ms_launch / 1000) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": kernel_traffic(name, wl),
                "peak_source": f"{peak_src} bf16_tflops_sustained",
                "ms_per_launch": ms_launch, "flops_per_launch": work,
                "share_of_step": ktimes[name][0] / sum(t[0] for t in ktimes.values())}

    roof = roof_fwd = None
    cands = [(t[0], n) for n, t in ktimes.items() if kernel_work(n, wl) is not None]
    if cands:
        roof = roofline_of(max(cands)[1])
    if "tc_causal_sweep" in ktimes and roof and roof["kernel"] != "tc_causal_sweep":
        roof_fwd = roofline_of("tc_causal_sweep")
    return roof, roof_fwd


def chunk_ran(wl: I.Workload, kernels: str) -> int:
    """Tokens per chunk of the kernels that run: the tensor-core sweeps use 128-token chunks
    (bf16, 6 <= P <= 8, L * 2^P a multiple of 128), the CUDA-core kernels 32-token tiles;
    the workload's requested chunk is advisory."""
    tensor = (wl.dtype == "bf16" and kernels != "simt" and 6 <= wl.P <= 8
              and (wl.L << wl.P) % 128 == 0)
    return 128 if tensor else 32


def rank_heads(rank: int, heads_per_rank: int):
    """Global head indices of one rank: heads are independent (W is shared), so with weak
    scaling rank r owns heads r*H .. r*H + H - 1 of the global batch of heads."""
    return [rank * heads_per_rank + h for h in range(heads_per_rank)]


def allreduce_dw(dW, world: int):
    """dW is a sum over all heads and tokens: the per-rank partial sums are added with one
    all-reduce (NCCL on GPUs; any backend of the default process group)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(dW, op=dist.ReduceOp.SUM)
    return dW


def max_over_ranks(ms: float, world: int, device) -> float:
    """Step time of the job = the slowest rank's device time."""
    if world <= 1:
        return ms
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- oracle arm
def oracle_rate(wl: I.Workload, n_tokens: int, backward: bool, seed_head: int = 0):
    """Time the float64 oracle on one head of n_tokens tokens; returns (tokens/s of the
    whole multi-head workload, seconds, threads)."""
    import numpy as np  # noqa: F401
    import oracle
    x = I.make_inputs(wl, "cpu", N=n_tokens, heads=[seed_head], with_dout=True)
    f = {k: v.double().numpy() for k, v in x.items()}
    t0 = time.perf_counter()
    if backward:
        oracle.backward(f["q"][0], f["k"][0], f["v"][0], f["W"], wl.tau, wl.causal,
                        f["dout"][0])
    else:
        oracle.forward(f["q"][0], f["k"][0], f["v"][0], f["W"], wl.tau, wl.causal)
    dt = time.perf_counter() - t0
    # one head of n tokens is 1/H of the per-token work of the full workload
    tokens_equiv = n_tokens * wl.batch / wl.H
    return tokens_equiv / dt, dt, os.cpu_count()


def run_reference(args, wl: I.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    backward = not args.fwd_only
    n = args.ref_tokens
    for _ in range(args.warmup):
        oracle_rate(wl, n, backward)
    times = []
    for s in range(args.steps):
        rate, dt, cores = oracle_rate(wl, n, backward, seed_head=s % wl.H)
        times.append(dt)
    ms = 1000 * statistics.mean(times)
    value = n * wl.batch / wl.H / (ms / 1000)
    unit = "tokens/s"
    sample = (f"one head of {n} tokens of the {wl.name} workload per step "
              f"({'forward+backward' if backward else 'forward'}), float64 numpy oracle; "
              f"tokens/s scaled by 1/{wl.H} heads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "H": wl.H, "N": wl.N, "d": wl.d, "L": wl.L,
                   "P": wl.P, "tau": wl.tau, "causal": wl.causal,
                   "step": "fwd+bwd" if backward else "fwd"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": os.cpu_count(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm
def run_ours(args, wl: I.Workload):
    import torch.distributed as dist

    from linear_lsh_sketch_race_b200 import race_attn as ra

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=dev)
    ra.load()
    backward = not args.fwd_only
    heads = rank_heads(rank, wl.H)
    x = I.make_inputs(wl, dev, heads=heads, with_dout=backward)
    q, k, v, W = x["q"], x["k"], x["v"], x["W"]
    dout = x.get("dout")
    out = torch.empty_like(q)
    den = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    a = ra.make_args(q, W, wl.tau, wl.causal, chunk=wl.chunk, impl=args.kernels, den=den)
    need = max(ra.race_workspace_size(a, False),
               ra.race_workspace_size(a, True) if backward else 0)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    a.workspace = ws.data_ptr()
    a.workspace_bytes = ws.numel()
    if backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dW = torch.empty_like(W)
    stream = torch.cuda.current_stream(dev)

    def fwd_only():
        ra.race_forward_ex(q, k, v, W, out, a, stream)

    def step():
        ra.race_forward_ex(q, k, v, W, out, a, stream)
        if backward:
            ra.race_backward_ex(q, k, v, W, out, dout, dq, dk, dv, dW, a, stream)
            allreduce_dw(dW, world)

    def timed(fn, n):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        return max_over_ranks(e0.elapsed_time(e1) / n, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert ra.race_device_status(stream) == 0

    sampler = ClockSampler(local)
    sampler.start()
    ra.race_timing_enable(True)
    n0 = ra.race_launch_count()
    ms = timed(step, args.steps)
    launches = ra.race_launch_count() - n0
    ktimes = ra.race_timing_report()
    ra.race_timing_enable(False)
    clocks = sampler.stop()
    if ra.race_device_status(stream) != 0:
        raise RuntimeError("device status flag raised during the timed region")
    fwd_ms = timed(fwd_only, args.steps) if backward else ms

    tokens = wl.batch * wl.N * world
    value = tokens / (ms / 1000)
    peaks, peak_src = load_peaks()
    f_fwd, f_bwd = flops_per_token_head(wl)

    roof, roof_fwd = roofline_lines(ktimes, wl, peaks, peak_src)

    ideal_ms = max(wl.H * wl.N * (f_fwd + (f_bwd if backward else 0)) /
                   (peaks["bf16_tflops"] * 1e12),
                   wl.H * wl.N * sum(bytes_per_token_head(wl)[: 2 if backward else 1]) /
                   (peaks["hbm_gbs"] * 1e9)) * 1000
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "H": wl.H, "N": wl.N, "d": wl.d, "L": wl.L,
                   "P": wl.P, "tau": wl.tau, "causal": wl.causal,
                   "chunk": chunk_ran(wl, args.kernels), "chunk_requested": wl.chunk,
                   "step": "fwd+bwd" if backward else "fwd", "kernels": args.kernels,
                   "l2": "inputs larger than L2 (q, k, v = %.1f GB per rank)" %
                         (3 * q.numel() * q.element_size() / 1e9),
                   "parallelism": f"heads sharded: {wl.H} heads per rank"},
        "fwd": {"value": tokens / (fwd_ms / 1000), "unit": "tokens/s",
                "ms_per_step": fwd_ms},
        "method_roofline": {"ideal_ms_per_step": ideal_ms, "frac": ideal_ms / ms,
                            "peak_source": f"{peak_src} bf16_tflops (burst) / hbm_gbs"},
        "roofline": roof,
        "roofline_fwd_sweep": roof_fwd,
        "kernel_ms_per_step": {n: t[0] / args.steps for n, t in ktimes.items()},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if not args.no_e2e:
        outs = {"out": out}
        if backward:
            outs.update(dq=dq, dk=dk, dv=dv, dW=dW)
        line["e2e"] = run_e2e(args, wl, x, outs, a, ra, dev, stream, world, backward)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_tokens
        rate, dt, cores = oracle_rate(wl, n, backward)
        line["cpu_baseline"] = {
            "value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"one head of {n} tokens ({'fwd+bwd' if backward else 'fwd'}), "
                      f"{dt:.1f} s of float64 numpy; tokens/s scaled by 1/{wl.H} heads"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(args, wl, x, outs, a, ra, dev, stream, world, backward):
    """Same step through the public API with host inputs: pinned host -> device copies
    of q, k, v (and dO), the step, device -> host copies of the results (o, and dq, dk,
    dv, dW for the backward), every step.

    Steps alternate between two device buffer sets (set 0 is the device-timed run's own
    tensors `x` and `outs`, set 1 is allocated here), so the inputs of step s + 1 upload
    on one copy stream while step s computes, and the results of step s - 1 download on
    another meanwhile (one cudaMemcpyAsync per tensor).  Every step computes all heads at
    once, which keeps the sweeps' grids as wide as in the device-timed run.  The timed
    region opens before the first upload and closes after the last download."""
    try:
        import torch.distributed as dist
        names = ["q", "k", "v"] + (["dout"] if backward else [])
        res = ["out"] + (["dq", "dk", "dv", "dW"] if backward else [])
        host = {n: torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=True) for n in names}
        for n in names:
            host[n].copy_(x[n])
        ins = [{n: x[n] for n in names}, {n: torch.empty_like(x[n]) for n in names}]
        res_sets = [{n: outs[n] for n in res}, {n: torch.empty_like(outs[n]) for n in res}]
        host_res = {n: torch.empty(outs[n].shape, dtype=outs[n].dtype, pin_memory=True)
                    for n in res}
        h2d = sum(host[n].numel() * host[n].element_size() for n in names)
        d2h = sum(host_res[n].numel() * host_res[n].element_size() for n in res)
        W = x["W"]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        fwd_in = [n for n in names if n != "dout"]
        grads = [n for n in res if n != "out"]
        # per buffer set: compute done reading its inputs; its o and its gradients copied out
        computed, out_read, grads_read = [None, None], [None, None], [None, None]

        def event(st):
            e = torch.cuda.Event()
            e.record(st)
            return e

        def step(s):
            # The forward needs q, k, v only and o is final after it: the forward starts
            # before dO has landed, and o downloads while the backward runs.
            b = s & 1
            d, r = ins[b], res_sets[b]
            with torch.cuda.stream(up):
                if computed[b] is not None:     # step s - 2 has read this input set
                    up.wait_event(computed[b])
                for n in fwd_in:
                    d[n].copy_(host[n], non_blocking=True)
                fwd_ready = event(up)
                if backward:
                    d["dout"].copy_(host["dout"], non_blocking=True)
                    bwd_ready = event(up)
            stream.wait_event(fwd_ready)
            if out_read[b] is not None:         # step s - 2's o has left this set
                stream.wait_event(out_read[b])
            ra.race_forward_ex(d["q"], d["k"], d["v"], W, r["out"], a, stream)
            fwd_done = event(stream)
            with torch.cuda.stream(down):
                down.wait_event(fwd_done)
                host_res["out"].copy_(r["out"], non_blocking=True)
                out_read[b] = event(down)
            if backward:
                stream.wait_event(bwd_ready)
                if grads_read[b] is not None:   # step s - 2's gradients have left this set
                    stream.wait_event(grads_read[b])
                ra.race_backward_ex(d["q"], d["k"], d["v"], W, r["out"], d["dout"],
                                    r["dq"], r["dk"], r["dv"], r["dW"], a, stream)
                allreduce_dw(r["dW"], world)
            computed[b] = event(stream)
            if not backward:
                return out_read[b]
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                for n in grads:
                    host_res[n].copy_(r[n], non_blocking=True)
                grads_read[b] = event(down)
            return grads_read[b]

        n = max(1, min(args.steps, args.e2e_steps) if args.e2e_steps > 0 else args.steps)
        for s in range(2):                      # warm-up: both buffer sets once
            step(s)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        for s in range(n):
            last = step(s)
        stream.wait_event(last)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(e0.elapsed_time(e1) / n, world, dev)
        tokens = wl.batch * wl.N * world
        return {"value": tokens / (ms / 1000), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms, "steps": n, "buffer_sets": 2}
    except Exception as e:  # pinned host memory can be short on some hosts
        return {"value": None, "unit": "tokens/s", "error": repr(e)[:200]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=I.HEADLINE, choices=sorted(I.WORKLOADS))
    ap.add_argument("--N", type=int, default=0, help="override sequence length")
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--kernels", choices=["auto", "simt", "tensor"], default="auto")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="steps of the end-to-end leg (0: the same as --steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=8192)
    ap.add_argument("--ref-tokens", type=int, default=2048)
    args = ap.parse_args()
    wl = I.WORKLOADS[args.workload]
    if args.N:
        wl = wl.replace(N=args.N, name=f"{wl.name}_N{args.N}")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
