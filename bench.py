#!/usr/bin/env python
"""Benchmark of the LM-head loss path: one step = the five calls
lmhead_fwd -> ce_fwd -> ce_bwd (BF16 dlogits) -> lmhead_bwd_dx -> lmhead_bwd_dw
on one synthetic batch (default: M=4096 tokens, K=4096, V=128256; X ~ N(0,1),
W ~ N(0,0.02^2) in BF16, 1% of targets ignored, grad_loss = 1/num_valid; the
FP32 logits take 2.1 GB).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload lmhead_4096x4096x128256 | lmhead_1024x4096x32768 |
                                lmhead_<M>x<K>x<V> | ce_8192x151936_outliers | sweep |
                                bitexact_16x512x32768]

The default workload is the largest LM-head configuration of the method that
fits one GPU.  The mid-size LM head (and any lmhead_<M>x<K>x<V> shape, N(0,1) x
N(0,0.02^2) operands with 1% of rows ignored, used for scaled profiles) and the
wide-row cross-entropy workload print the same kind of line;
"sweep" runs the FP32-versus-BF16 output comparison of the GEMM (15 shapes,
N = 32768, 10 warm-up pairs, 30 alternating-order samples, medians);
"bitexact_16x512x32768" times the latency-bound smoke workload (lmhead_fwd,
ce_fwd, ce_bwd) in microseconds.

Prints one JSON line on rank 0.  Timing: CUDA events on the launching stream
around every step (and every call inside it), L2 flushed by a 512 MiB write
between steps outside the timed events, device time summed over the K steps
and the maximum taken over ranks.  With N > 1 (torchrun) every rank runs an
independent replica of the step on its own batch (weak scaling, no
collective on the data path).

--impl reference times the CPU oracle (FP64, all host cores) on a bounded
sample of the same workload; it is the deliberately slow baseline, not a
competitor.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LM-head+CE fwd+bwd tokens/s; GEMM TFLOP/s and CE GB/s as % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ("lm_head_fp32_b200/csrc/gemm_tc.cuh", "lm_head_fp32_b200/csrc/ce_kernels.cuh",
                  "lm_head_fp32_b200/csrc/ptx.cuh", "lm_head_fp32_b200/csrc/lmhead.cu",
                  "lm_head_fp32_b200/csrc/softmax_merge.cuh")
FLUSH_BYTES = 512 << 20
L2_NOTE = ("flushed between steps outside the timed events: a 512 MiB write, then a read of "
           "it, so that no dirty line of the flush is left for the step to write back")


def flush_l2(buf):
    """Evict the L2 (126 MB) between timed steps: write a buffer four times
    its size, then read it back, which also writes back the dirty lines of
    the write before the next step starts."""
    buf.zero_()
    return buf.sum()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample", type=int, default=256,
                    help="tokens of the workload the CPU oracle baseline processes")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--step", choices=["separate", "fused"], default="separate",
                    help="separate: the five calls; fused: lmhead_fwd_ce (logits and CE "
                         "statistics in one pass) then ce_bwd, dX, dW")
    ap.add_argument("--parallel", choices=["replicas", "vocab"], default="replicas",
                    help="N > 1: replicas = every rank runs its own batch (weak scaling); "
                         "vocab = the vocabulary is split across the ranks, one batch in all "
                         "(strong scaling; NCCL all-gather of the per-row records and "
                         "all-reduce of dX)")
    ap.add_argument("--workload", default="lmhead_4096x4096x128256", type=workload_name,
                    help="lmhead_4096x4096x128256 (default), lmhead_1024x4096x32768, "
                         "lmhead_<M>x<K>x<V>, ce_8192x151936_outliers, sweep, "
                         "bitexact_16x512x32768")
    return ap.parse_args()


FIXED_WORKLOADS = ("ce_8192x151936_outliers", "sweep", "bitexact_16x512x32768")
_LMHEAD_RE = re.compile(r"lmhead_(\d+)x(\d+)x(\d+)$")


def workload_name(name: str) -> str:
    if name in FIXED_WORKLOADS or _LMHEAD_RE.match(name):
        return name
    raise argparse.ArgumentTypeError(f"unknown workload {name!r}")


def lmhead_config(name: str):
    """The LM-head workload of that name: the two named configurations keep
    their own seeds and ignore fractions; any other lmhead_<M>x<K>x<V> draws
    X ~ N(0,1), W ~ N(0,0.02^2) and ignores 1% of the rows."""
    from lm_head_fp32_b200 import synth
    for c in (synth.LARGEVOCAB, synth.MIDSIZE):
        if c.name == name:
            return c
    m = _LMHEAD_RE.match(name)
    if not m:
        raise ValueError(f"not an LM-head workload: {name}")
    M, K, V = (int(v) for v in m.groups())
    return synth.GemmConfig(name, M, K, V, "normal", ignore_frac=0.01)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, clocks):
    """Dense-BF16 denominator for the GEMMs: the sustained figure when the
    power cap throttled the timed steps (sw_power_cap seen by the clock
    sampler: the kernels ran inside a long power-limited stretch, as the
    sustained cuBLAS loop did), else the burst figure."""
    if "sw_power_cap" in (clocks or {}).get("reasons", []):
        return peaks["bf16_tflops_sustained"], "sustained: sw_power_cap active in the timed steps"
    return peaks["bf16_tflops"], "burst"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """Per-launch DRAM bytes of each kernel from the committed ncu summary of
    this workload, or {} when there is none or it was taken on different
    kernel sources."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.md")
    if not os.path.exists(p):
        return {}
    txt = open(p).read()
    m = re.search(r"kernel-source-hash:\s*([0-9a-f]+)", txt)
    if not m or m.group(1) != kernel_source_hash():
        return {}
    out = {}
    for name, val in re.findall(r"^\|\s*(\w+)\s*\|\s*([0-9.eE+]+)\s*\|", txt, flags=re.M):
        try:
            out[name] = float(val)
        except ValueError:
            pass
    return out


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(x: float, pg, device) -> float:
    """Maximum of a per-rank float across all ranks (the job's device time)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ----------------------------------------------------------------------------
# CPU oracle baseline (the reference arm of this path)
# ----------------------------------------------------------------------------

def oracle_step(X, W, t, g, rows):
    """The whole path on the CPU oracle for the given token rows: logits,
    CE forward, CE backward (BF16 round), dX rows and those tokens' share of dW."""
    import numpy as np
    import oracle
    from lm_head_fp32_b200 import synth
    xb, wb = synth.bf16_bits(X), synth.bf16_bits(W)
    L = oracle.round_f32(oracle.logits(xb, wb, rows=rows))
    tt = t.numpy()[rows]
    oracle.ce_fwd(L, tt)
    dl = oracle.round_bf16(oracle.ce_bwd(L, tt, g))
    oracle.dx(dl, wb)                       # dX for the sampled rows
    oracle.dw(dl, xb[rows])                 # their contribution to dW (all V rows)


def cpu_baseline(cfg, X, W, t, g, tokens: int):
    import numpy as np
    import oracle
    rows = np.arange(tokens, dtype=np.int64)
    t0 = time.perf_counter()
    oracle_step(X, W, t, g, rows)
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{tokens} of {cfg.M} tokens of {cfg.name} through all five steps "
                      f"(logits, CE fwd, CE bwd, dX rows, their dW share), FP64, {dt:.1f} s"}


def reference_tokens_per_step(steps: int, warmup: int, cap: int, K: int = 4096,
                              V: int = 32768) -> int:
    """Tokens of the oracle's sample per reference step: 1 to min(cap, 16),
    sized so that the whole run stays near a minute and a half of host time
    (about 0.1 s per token on 16 cores at K = 4096, V = 32768; the cost of a
    token grows with K * V)."""
    budget = int(900 * (4096 * 32768) / (K * V))
    return max(1, min(cap, 16, budget // max(1, steps + warmup)))


def run_reference(args):
    world, rank, local, pg = dist_setup(args)
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    name = args.workload if _LMHEAD_RE.match(args.workload) else "lmhead_4096x4096x128256"
    cfg = lmhead_config(name)
    X, W, t = cfg.make()
    g = cfg.grad_scalar(t)
    import numpy as np
    import oracle
    per_step = reference_tokens_per_step(args.steps, args.warmup, args.cpu_sample, cfg.K, cfg.V)
    for i in range(args.warmup):
        oracle_step(X, W, t, g, np.arange(per_step, dtype=np.int64) + (i * per_step) % cfg.M)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_step(X, W, t, g, (np.arange(per_step, dtype=np.int64) + i * per_step) % cfg.M)
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "V": cfg.V,
                       "tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"{per_step} tokens of {cfg.name} per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def gpu_setup(args):
    import torch
    world, rank, local, pg = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    return world, rank, local, pg, dev


def run_ours(args, cfg):
    import torch
    from lm_head_fp32_b200 import lmhead, synth

    world, rank, local, pg, dev = gpu_setup(args)
    M, K, V = cfg.M, cfg.K, cfg.V
    # every rank draws its own batch (replica r uses seed + 7919 r)
    rcfg = synth.GemmConfig(cfg.name, M, K, V, cfg.dist, cfg.x_std, cfg.w_std, cfg.ignore_frac,
                            cfg.grad, cfg.seed + 7919 * rank)
    X, W, t = rcfg.make()
    g = rcfg.grad_scalar(t)
    Xd, Wd, td = X.to(dev), W.to(dev), t.to(dev)
    gd = torch.tensor([g], dtype=torch.float32, device=dev)
    logits = torch.empty((M, V), dtype=torch.float32, device=dev)
    stats = torch.empty((M, 4), dtype=torch.float32, device=dev)
    dl = torch.empty((M, V), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.float32, device=dev)
    dW = torch.empty((V, K), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    fused = args.step == "fused"
    ws = torch.empty(lmhead.lmhead_fwd_ce_workspace_bytes(M, V), dtype=torch.uint8, device=dev)
    variants = {
        "fused": (["lmhead_fwd_ce", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw"], [
            lambda: lmhead.lmhead_fwd_ce(Xd, Wd, td, logits, stats, ws, -100, status),
            lambda: lmhead.ce_bwd(logits, td, stats, gd, dl, -100, status),
            lambda: lmhead.lmhead_bwd_dx(dl, Wd, dX, status),
            lambda: lmhead.lmhead_bwd_dw(dl, Xd, dW, status),
        ]),
        "separate": (["lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw"], [
            lambda: lmhead.lmhead_fwd(Xd, Wd, logits, status),
            lambda: lmhead.ce_fwd(logits, td, stats, -100, status),
            lambda: lmhead.ce_bwd(logits, td, stats, gd, dl, -100, status),
            lambda: lmhead.lmhead_bwd_dx(dl, Wd, dX, status),
            lambda: lmhead.lmhead_bwd_dw(dl, Xd, dW, status),
        ]),
    }
    names, calls = variants["fused" if fused else "separate"]
    K_steps = args.steps

    def timed_loop(calls, per_kernel):
        """W warm-up steps, then K timed steps.  per_kernel: an event after
        every call as well (the per-kernel times); otherwise events only
        around each step, so that nothing sits between the calls and each
        kernel's programmatic dependent launch overlaps the previous one's
        tail as in an untimed step.  Returns the per-call times (or None), the
        job time (max over ranks) and the clock record."""
        for _ in range(max(args.warmup, 3)):
            flush_l2(flush)
            for c in calls:
                c()
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"device status {int(status.item())}"
        n_ev = len(calls) + 1 if per_kernel else 2
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K_steps)]
        sampler = ClockSampler(dev.index)
        barrier(pg)
        torch.cuda.synchronize()
        sampler.start()
        time.sleep(0.25)                      # let the sampler attach
        for i in range(K_steps):
            flush_l2(flush)                   # L2 flush, outside the timed events
            e = ev[i]
            e[0].record(stream)
            for j, c in enumerate(calls):
                c()
                if per_kernel:
                    e[j + 1].record(stream)
            if not per_kernel:
                e[1].record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        barrier(pg)
        assert int(status.item()) == 0, f"device status {int(status.item())}"
        per_call = ([[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K_steps)]
                     for j in range(len(calls))] if per_kernel else None)
        step_ms = [ev[i][0].elapsed_time(ev[i][-1]) for i in range(K_steps)]
        return per_call, max_over_ranks(sum(step_ms), pg, dev), clocks

    # the headline: the step timed as a whole
    _, total_ms, clocks = timed_loop(calls, per_kernel=False)
    value = world * M * K_steps / (total_ms / 1e3)
    # each kernel's time, from a second loop with an event after every call
    per_call, kernel_loop_ms, kclocks = timed_loop(calls, per_kernel=True)
    # the other form of the step, for comparison: the fused forward
    # (lmhead_fwd_ce: logits and CE statistics in one pass) or the five calls
    alt_key = "separate" if fused else "fused"
    alt_names, alt_calls = variants[alt_key]
    _, alt_total_ms, _ = timed_loop(alt_calls, per_kernel=False)
    alt_per_call, _, _ = timed_loop(alt_calls, per_kernel=True)
    alt = {"value": world * M * K_steps / (alt_total_ms / 1e3), "unit": "tokens/s",
           "ms_per_step": alt_total_ms / K_steps, "step": ", ".join(alt_names),
           "kernels_ms": {n: round(statistics.mean(alt_per_call[j]), 5)
                          for j, n in enumerate(alt_names)}}

    # end to end through the public API: every step copies its X and targets
    # from pinned host memory, and its per-row statistics (the loss) and dX
    # (the gradient handed back to the layer below) to pinned host memory.
    # Inputs and outputs are double-buffered; inputs are copied on one side
    # stream and outputs on another, so step i+1's input copy and step i-1's
    # output copy run under step i's kernels, as in a training loop with a
    # prefetching loader.  dW stays on the device with W.
    Xh = X.pin_memory()
    th = t.pin_memory()
    outh = [(torch.empty((M, 4), dtype=torch.float32).pin_memory(),
             torch.empty((M, K), dtype=torch.float32).pin_memory()) for _ in range(2)]
    Xb = [Xd, torch.empty_like(Xd)]
    tb = [td, torch.empty_like(td)]
    sb = [stats, torch.empty_like(stats)]
    dXb = [dX, torch.empty_like(dX)]
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_copied = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        if i >= 2:
            h2d_s.wait_event(done[b])       # step i-2 has finished with input buffer b
        with torch.cuda.stream(h2d_s):
            Xb[b].copy_(Xh, non_blocking=True)
            tb[b].copy_(th, non_blocking=True)
            copied[b].record(h2d_s)
        stream.wait_event(copied[b])
        if i >= 2:
            stream.wait_event(out_copied[b])  # step i-2's outputs have left buffer b
        if fused:
            lmhead.lmhead_fwd_ce(Xb[b], Wd, tb[b], logits, sb[b], ws, -100, status)
        else:
            lmhead.lmhead_fwd(Xb[b], Wd, logits, status)
            lmhead.ce_fwd(logits, tb[b], sb[b], -100, status)
        lmhead.ce_bwd(logits, tb[b], sb[b], gd, dl, -100, status)
        lmhead.lmhead_bwd_dx(dl, Wd, dXb[b], status)
        lmhead.lmhead_bwd_dw(dl, Xb[b], dW, status)
        done[b].record(stream)
        d2h_s.wait_event(done[b])
        with torch.cuda.stream(d2h_s):
            outh[b][0].copy_(sb[b], non_blocking=True)
            outh[b][1].copy_(dXb[b], non_blocking=True)
            out_copied[b].record(d2h_s)

    e2e_steps = max(10, min(K_steps, 100))
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_s.wait_event(a)
    d2h_s.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    for b in range(2):
        stream.wait_event(out_copied[b])    # the last results are on the host
    z.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(z), pg, dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    h2d = Xh.numel() * Xh.element_size() + th.numel() * th.element_size()
    d2h = sum(o.numel() * o.element_size() for o in outh[0])

    # roofline of every kernel; the dominant one goes in "roofline"
    peaks, peak_src = load_peaks()
    peak_t, peak_kind = tensor_peak(peaks, kclocks)
    flop = 2.0 * M * K * V
    nv = int((t != -100).sum())
    ce_fwd_bytes = nv * V * 4 + M * (8 + 16)
    ce_bwd_bytes = nv * V * 4 + M * V * 2 + M * (8 + 16)
    algo = {"lmhead_fwd": ("tensor", flop), "lmhead_fwd_ce": ("tensor", flop),
            "ce_fwd": ("hbm", ce_fwd_bytes),
            "ce_bwd": ("hbm", ce_bwd_bytes), "lmhead_bwd_dx": ("tensor", flop),
            "lmhead_bwd_dw": ("tensor", flop)}
    traffic = committed_traffic(cfg.name)
    kernels = {}
    for j, n in enumerate(names):
        ms = statistics.mean(per_call[j])
        bound, work = algo[n]
        if bound == "tensor":
            ach, peak, unit = work / (ms / 1e3) / 1e12, peak_t, "TFLOP/s"
        else:
            ach, peak, unit = work / (ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
        kernels[n] = {"ms": round(ms, 5), "bound": bound, "achieved": round(ach, 1), "unit": unit,
                      "frac": round(ach / peak, 4), "algorithmic": work}
        if bound == "tensor":
            kernels[n]["frac_of_burst"] = round(ach / peaks["bf16_tflops"], 4)
    dom = max(names, key=lambda n: kernels[n]["ms"])
    kd = kernels[dom]
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"],
                "peak": peak_t if kd["bound"] == "tensor" else peaks["hbm_gbs"],
                "unit": kd["unit"], "frac": kd["frac"],
                "peak_source": f"{peak_src} ({peak_kind if kd['bound'] == 'tensor' else 'copy'})",
                "traffic": traffic.get(dom)}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K_steps, "warmup": args.warmup, "ms_per_step": total_ms / K_steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": cfg.name, "M": M, "K": K, "V": V, "logits": "fp32",
                       "dlogits": "bf16", "dX_dW": "fp32", "accumulate": "fp32",
                       "ignored_rows": M - nv, "grad_loss": "1/num_valid",
                       "l2": L2_NOTE,
                       "parallelism": f"replicas x{world}",
                       "step": ("lmhead_fwd_ce, ce_bwd, lmhead_bwd_dx, lmhead_bwd_dw" if fused else
                                "lmhead_fwd, ce_fwd, ce_bwd, lmhead_bwd_dx, lmhead_bwd_dw")},
            "roofline": roofline, "kernels": kernels,
            "e2e": {"value": world * M * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "note": "X and targets in, stats and dX out, pinned host memory, "
                            "double-buffered on two side streams; no L2 flush (the step's "
                            "working set is far larger than L2)"},
            "gpu_launches": sum(2 if n == "lmhead_fwd_ce" else 1 for n in names) * K_steps,
            "clocks": clocks, f"{alt_key}_step": alt,
            "kernel_timing": {"ms_per_step": kernel_loop_ms / K_steps, "clocks": kclocks,
                              "note": "per-kernel times come from a second loop of the same "
                                      "steps with an event after every call"}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # about 10-30 s of oracle work: the sample shrinks as the vocabulary grows
        sample = max(8, int(args.cpu_sample * 32768 * 4096 / (cfg.V * cfg.K)))
        line["cpu_baseline"] = cpu_baseline(cfg, X, W, t, g, sample)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def vocab_shard_inputs(cfg, world: int, rank: int):
    """This rank's inputs of a vocabulary-parallel step: the whole batch (the
    same X and targets on every rank) and rows [off, off + n) of W."""
    from lm_head_fp32_b200 import vocab_parallel
    X, W, t = cfg.make()
    off, n = vocab_parallel.shard_bounds(cfg.V, world, rank)
    return X, W[off:off + n].contiguous(), t, off, n


def vocab_line(cfg, world: int, steps: int, warmup: int, total_ms: float, stage_ms: dict,
               clocks, nv: int, peaks, peak_src: str, shard_rows: int) -> dict:
    """The JSON line of a vocabulary-parallel run: every rank works on the same
    M tokens, so the job processes M tokens per step whatever the rank count
    (strong scaling); total_ms is the maximum over ranks of the summed step
    times, stage_ms this rank's mean time per stage."""
    M, K = cfg.M, cfg.K
    peak_t, peak_kind = tensor_peak(peaks, clocks)
    flop = 2.0 * M * K * shard_rows
    work = {"lmhead_fwd": ("tensor", flop), "lmhead_bwd_dx": ("tensor", flop),
            "lmhead_bwd_dw": ("tensor", flop),
            "ce_fwd_shard": ("hbm", nv * shard_rows * 4 + M * 24),
            "ce_bwd_shard": ("hbm", nv * shard_rows * 4 + M * shard_rows * 2 + M * 24)}
    kernels = {}
    for n, ms in stage_ms.items():
        if n not in work or ms <= 0:
            kernels[n] = {"ms": round(ms, 5)}
            continue
        bound, w = work[n]
        if bound == "tensor":
            ach, peak, unit = w / (ms / 1e3) / 1e12, peak_t, "TFLOP/s"
        else:
            ach, peak, unit = w / (ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
        kernels[n] = {"ms": round(ms, 5), "bound": bound, "achieved": round(ach, 1), "unit": unit,
                      "frac": round(ach / peak, 4), "algorithmic": w}
        if bound == "tensor":
            kernels[n]["frac_of_burst"] = round(ach / peaks["bf16_tflops"], 4)
    dom = max((n for n in kernels if "bound" in kernels[n]), key=lambda n: kernels[n]["ms"])
    kd = kernels[dom]
    return {"metric": METRIC, "value": M * steps / (total_ms / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": total_ms / steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": cfg.name, "M": M, "K": K, "V": cfg.V, "logits": "fp32",
                       "dlogits": "bf16", "dX_dW": "fp32", "ignored_rows": M - nv,
                       "grad_loss": "1/num_valid", "parallelism": f"vocab{world}",
                       "nccl_ranks": world, "vocab_rows_per_rank": shard_rows,
                       "l2": L2_NOTE,
                       "step": "lmhead_fwd, ce_fwd_shard, all-gather [M,4], ce_merge_shards, "
                               "ce_bwd_shard, lmhead_bwd_dx, all-reduce dX, lmhead_bwd_dw"},
            "roofline": {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"],
                         "peak": peak_t if kd["bound"] == "tensor" else peaks["hbm_gbs"],
                         "unit": kd["unit"], "frac": kd["frac"],
                         "peak_source": f"{peak_src} ({peak_kind if kd['bound'] == 'tensor' else 'copy'})",
                         "traffic": None},
            "kernels": kernels, "clocks": clocks}


def run_vocab(args, cfg):
    """Vocabulary-parallel step across the ranks (strong scaling)."""
    import torch
    from lm_head_fp32_b200 import vocab_parallel

    world, rank, local, pg, dev = gpu_setup(args)
    X, Ws, t, off, n = vocab_shard_inputs(cfg, world, rank)
    g = cfg.grad_scalar(t)
    Xd, Wd, td = X.to(dev), Ws.to(dev), t.to(dev)
    gd = torch.tensor([g], dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        flush_l2(flush)
        vocab_parallel.step(Xd, Wd, td, off, cfg.V, gd, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    stages = vocab_parallel.STAGES
    ev = [{} for _ in range(args.steps)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    barrier(pg)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    for i in range(args.steps):
        flush_l2(flush)
        starts[i].record(stream)

        def mark(name, i=i):
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            ev[i][name] = e
        vocab_parallel.step(Xd, Wd, td, off, cfg.V, gd, status=status, mark=mark)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(pg)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    step_ms = [starts[i].elapsed_time(ev[i][stages[-1]]) for i in range(args.steps)]
    total_ms = max_over_ranks(sum(step_ms), pg, dev)
    stage_ms = {}
    for j, s in enumerate(stages):
        prev = [starts[i] if j == 0 else ev[i][stages[j - 1]] for i in range(args.steps)]
        stage_ms[s] = statistics.mean(prev[i].elapsed_time(ev[i][s]) for i in range(args.steps))
    peaks, peak_src = load_peaks()
    nv = int((t != -100).sum())
    line = vocab_line(cfg, world, args.steps, args.warmup, total_ms, stage_ms, clocks, nv, peaks,
                      peak_src, n)
    line["gpu_launches"] = (6 if n > 0 else 1) * args.steps

    # end to end: every step copies X and the targets in from pinned host
    # memory and the statistics and dX out, on the compute stream
    Xh, th = X.pin_memory(), t.pin_memory()
    sh = torch.empty((cfg.M, 4), dtype=torch.float32).pin_memory()
    dxh = torch.empty((cfg.M, cfg.K), dtype=torch.float32).pin_memory()
    e2e_steps = max(5, min(args.steps, 50))
    barrier(pg)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        Xd.copy_(Xh, non_blocking=True)
        td.copy_(th, non_blocking=True)
        stats, dX, _, _, _ = vocab_parallel.step(Xd, Wd, td, off, cfg.V, gd, status=status)
        sh.copy_(stats, non_blocking=True)
        dxh.copy_(dX, non_blocking=True)
    z.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(z), pg, dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    line["e2e"] = {"value": cfg.M * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": Xh.numel() * Xh.element_size() + th.numel() * 8,
                   "d2h_bytes_per_step": sh.numel() * 4 + dxh.numel() * 4,
                   "note": "copies on the compute stream, not overlapped"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_ce(args):
    """Wide-row cross-entropy workload: CE forward, CE backward with FP32
    dlogits, CE backward with BF16 dlogits (g = 1)."""
    import numpy as np
    import torch
    from lm_head_fp32_b200 import lmhead, synth

    world, rank, local, pg, dev = gpu_setup(args)
    cfg = synth.CE_WIDE
    R, Cc = cfg.rows, cfg.cols
    x, t, _ = cfg.make(device=dev)
    td = t.to(dev)
    st = torch.empty((R, 4), dtype=torch.float32, device=dev)
    g = torch.ones(1, dtype=torch.float32, device=dev)
    d32 = torch.empty((R, Cc), dtype=torch.float32, device=dev)
    d16 = torch.empty((R, Cc), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    names = ["ce_fwd", "ce_bwd_f32", "ce_bwd_bf16"]
    calls = [lambda: lmhead.ce_fwd(x, td, st, -100, status),
             lambda: lmhead.ce_bwd(x, td, st, g, d32, -100, status),
             lambda: lmhead.ce_bwd(x, td, st, g, d16, -100, status)]
    for _ in range(max(args.warmup, 3)):
        for c in calls:
            c()
    torch.cuda.synchronize()
    steps = min(args.steps, 30)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    sampler = ClockSampler(dev.index)
    barrier(pg)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    for i in range(steps):
        e = ev[i]
        e[0].record(stream)
        for j, c in enumerate(calls):
            c()
            e[j + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(pg)
    assert int(status.item()) == 0
    total_ms = max_over_ranks(sum(ev[i][0].elapsed_time(ev[i][-1]) for i in range(steps)), pg, dev)
    peaks, peak_src = load_peaks()
    nv = int((t != -100).sum())
    algo = {"ce_fwd": nv * Cc * 4 + R * 24, "ce_bwd_f32": nv * Cc * 4 + R * Cc * 4 + R * 24,
            "ce_bwd_bf16": nv * Cc * 4 + R * Cc * 2 + R * 24}
    kernels = {}
    for j, n in enumerate(names):
        ms = statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps))
        gbs = algo[n] / (ms / 1e3) / 1e9
        kernels[n] = {"ms": round(ms, 5), "bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s",
                      "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic": algo[n]}
    dom = max(names, key=lambda n: kernels[n]["ms"])
    line = {"metric": METRIC, "value": world * R * steps / (total_ms / 1e3), "unit": "rows/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": total_ms / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "rows": R, "cols": Cc, "ignored_rows": R - nv,
                       "outlier_rows": int(cfg.outlier_frac * R), "grad_loss": 1.0,
                       "l2": "inputs (5 GB) larger than L2"},
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": kernels[dom]["achieved"],
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": kernels[dom]["frac"],
                         "peak_source": f"{peak_src} (copy)", "traffic": committed_traffic(cfg.name).get(dom)},
            "kernels": kernels, "gpu_launches": len(calls) * steps, "clocks": clocks}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        rows = np.arange(512, dtype=np.int64)
        xs = x[:512].cpu().numpy()
        ts = t.numpy()[:512]
        t0 = time.perf_counter()
        oracle.ce_fwd(xs, ts)
        oracle.ce_bwd(xs, ts, 1.0)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": len(rows) / dt, "unit": "rows/s",
                                "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"512 of {R} rows, CE forward + backward, FP64, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_sweep(args):
    """FP32- versus BF16-output epilogue of the same GEMM over the 15 shapes
    M x K (N = 32768): 10 warm-up pairs, 30 alternating-order event-timed
    samples per kernel, medians (the protocol of the pages' GEMM benchmark)."""
    import torch
    from lm_head_fp32_b200 import lmhead, synth

    world, rank, local, pg, dev = gpu_setup(args)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    peaks, peak_src = load_peaks()
    rows = []
    for c in synth.sweep_configs():
        X = synth.normal_bf16((c.M, c.K), 1.0, c.seed, device=dev)
        W = synth.normal_bf16((c.V, c.K), 0.02, c.seed + 1, device=dev)
        o32 = torch.empty((c.M, c.V), dtype=torch.float32, device=dev)
        o16 = torch.empty((c.M, c.V), dtype=torch.bfloat16, device=dev)
        run = {"f32": lambda: lmhead.lmhead_fwd(X, W, o32, status),
               "bf16": lambda: lmhead.lmhead_fwd(X, W, o16, status)}

        def sample(k):
            flush_l2(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run[k]()
            b.record(stream)
            b.synchronize()
            return a.elapsed_time(b)

        for _ in range(10):
            sample("f32")
            sample("bf16")
        t = {"f32": [], "bf16": []}
        for i in range(30):
            order = ("f32", "bf16") if i % 2 == 0 else ("bf16", "f32")
            for k in order:
                t[k].append(sample(k))
        m32, m16 = statistics.median(t["f32"]), statistics.median(t["bf16"])
        flop = 2.0 * c.M * c.K * c.V
        bytes32 = 2.0 * c.V * c.K + 2.0 * c.M * c.K + 4.0 * c.M * c.V
        bound = "hbm" if c.M <= 128 else "tensor"
        ach = (bytes32 / (m32 / 1e3) / 1e9) if bound == "hbm" else (flop / (m32 / 1e3) / 1e12)
        peak = peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"]
        rows.append({"M": c.M, "K": c.K, "N": c.V, "f32_us": round(m32 * 1e3, 2),
                     "bf16_us": round(m16 * 1e3, 2),
                     "overhead_pct": round(100.0 * (m32 - m16) / m16, 2),
                     "f32_tflops": round(flop / (m32 / 1e3) / 1e12, 1), "bound": bound,
                     "f32_frac": round(ach / peak, 4)})
        del X, W, o32, o16
    assert int(status.item()) == 0
    ov = [r["overhead_pct"] for r in rows]
    ov4 = [r["overhead_pct"] for r in rows if r["K"] >= 4096]
    ov8 = [r["overhead_pct"] for r in rows if r["K"] >= 8192]
    line = {"metric": "FP32-output vs BF16-output GEMM overhead, same kernel", "unit": "%",
            "value": statistics.median(ov), "higher_is_better": False, "n_gpus": 1,
            "median_overhead_pct_K_ge_4096": statistics.median(ov4),
            "median_overhead_pct_K_ge_8192": statistics.median(ov8),
            "shapes_within_10pct": sum(1 for o in ov if o <= 10.0),
            "range_pct": [min(ov), max(ov)], "shapes": rows, "peak_source": peak_src,
            "protocol": "10 warm-up pairs, 30 alternating-order samples, medians, L2 flushed "
                        "(512 MiB write then read) before every sample"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_latency(args):
    """The bit-exact smoke workload (16 x 512 x 32768, integer BF16 operands):
    it fits in L2, so it is latency-bound and is reported in microseconds per
    step of lmhead_fwd, ce_fwd and ce_bwd (BF16 gradient), replayed from a
    CUDA graph (the eager step time and each call's eager time, means over
    the timed steps, are given too), with no roofline fraction."""
    import torch
    from lm_head_fp32_b200 import lmhead, synth

    world, rank, local, pg, dev = gpu_setup(args)
    cfg = synth.BITEXACT
    X, W, t = cfg.make()
    Xd, Wd, td = X.to(dev), W.to(dev), t.to(dev)
    M, V = cfg.M, cfg.V
    g = torch.full((1,), cfg.grad_scalar(t), dtype=torch.float32, device=dev)
    logits = torch.empty((M, V), dtype=torch.float32, device=dev)
    stats = torch.empty((M, 4), dtype=torch.float32, device=dev)
    dl = torch.empty((M, V), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    names = ["lmhead_fwd", "ce_fwd", "ce_bwd"]
    calls = [lambda: lmhead.lmhead_fwd(Xd, Wd, logits, status),
             lambda: lmhead.ce_fwd(logits, td, stats, -100, status),
             lambda: lmhead.ce_bwd(logits, td, stats, g, dl, -100, status)]
    for _ in range(max(args.warmup, 3)):
        for c in calls:
            c()
    torch.cuda.synchronize()
    K_steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
          for _ in range(K_steps)]
    sampler = ClockSampler(dev.index)
    barrier(pg)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)
    for i in range(K_steps):
        ev[i][0].record(stream)
        for j, c in enumerate(calls):
            c()
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(pg)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    per = {n: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K_steps)) * 1e3
           for j, n in enumerate(names)}
    step_ms = [ev[i][0].elapsed_time(ev[i][-1]) for i in range(K_steps)]
    eager_ms = max_over_ranks(sum(step_ms), pg, dev)

    # the same step captured once in a CUDA graph and replayed K times: at this
    # size the launches, not the kernels, set the step time
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph):
            for c in calls:
                c()
    stream.wait_stream(side)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    a.record(stream)
    for _ in range(K_steps):
        graph.replay()
    z.record(stream)
    torch.cuda.synchronize()
    total_ms = max_over_ranks(a.elapsed_time(z), pg, dev)
    del graph
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    line = {"metric": "latency of lmhead_fwd + ce_fwd + ce_bwd (us per step, CUDA graph replay)",
            "value": 1e3 * total_ms / K_steps, "unit": "us", "n_gpus": world, "steps": K_steps,
            "warmup": args.warmup, "ms_per_step": total_ms / K_steps, "higher_is_better": False,
            "eager_us_per_step": 1e3 * eager_ms / K_steps,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "M": M, "K": cfg.K, "V": V, "operands": "BF16 integers",
                       "l2": "inputs fit in L2 (latency-bound; no flush, no roofline fraction)"},
            "kernels_us": {n: round(v, 2) for n, v in per.items()},
            "gpu_launches": len(calls) * K_steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.workload == "sweep":
        run_sweep(args)
    elif args.workload == "bitexact_16x512x32768":
        run_latency(args)
    elif args.workload == "ce_8192x151936_outliers":
        run_ce(args)
    elif args.parallel == "vocab":
        run_vocab(args, lmhead_config(args.workload))
    else:
        run_ours(args, lmhead_config(args.workload))


if __name__ == "__main__":
    main()
