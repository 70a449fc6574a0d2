#!/usr/bin/env python
"""Throughput of the exact-attention hot path on B200 (libfa2).

One step = the whole path on one batch: fa2_fwd, fa2_bwd_preprocess and
fa2_bwd on B=8, H=16, N=2048, d=128, bf16, non-causal, synthetic N(0,1)
inputs.  FLOPs per step count 4*B*H*N^2*d for the forward and 2.5x that for
the backward (causal would halve both).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  With --gpus N > 1 it must be launched under
torchrun: every rank runs its own independent batch (the path shards over
independent (batch, head) problems with no data exchange), the timed region
is bracketed by barriers, and the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the plain definition of
attention) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd+bwd TFLOP/s (bf16, hd128) vs N and % of B200 dense BF16 peak"
WORKLOAD = dict(B=8, H=16, N=2048, d=128, causal=False)
REF_STEP_S = 1.0   # seconds of oracle work per reference-arm step
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def bench_config(w):
    """The workload description both arms print (the same dict)."""
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    return {"workload": "B=8 H=16 N=2048 d=128 bf16 non-causal fwd+bwd (per GPU)",
            "B": B, "H": H, "N": N, "d": d, "causal": causal,
            "l2": "inputs larger than L2 (q,k,v,o,dO,dq,dk,dv = 512 MiB + 128 MiB "
                  "fp32 dQ accumulator per GPU, vs 126 MB L2)",
            "flops_per_step": 3.5 * flops_fwd(B, H, N, d, causal)}


def flops_fwd(B, H, N, d, causal=False):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ traffic
KERNEL_SOURCES = {
    "fa2_fwd": ["sm100_ptx.cuh", "status.cuh", "philox.cuh", "attn_common.cuh", "fwd_sm100.cuh"],
    "fa2_bwd": ["sm100_ptx.cuh", "status.cuh", "philox.cuh", "attn_common.cuh", "bwd_sm100.cuh",
                "fwd_sm100.cuh"],
}


def sources_hash(call):
    """Hash of the kernel sources with their // comments and blank lines
    removed, so that a comment-only edit keeps a capture valid."""
    import hashlib
    import re
    m = hashlib.sha256()
    for f in sorted(KERNEL_SOURCES[call]):
        with open(os.path.join(ROOT, "exact_attention_147_b200", "csrc", f), encoding="utf-8") as fh:
            code = [re.sub(r"//.*$", "", ln).rstrip() for ln in fh.read().splitlines()]
        m.update("\n".join(ln for ln in code if ln).encode())
    return m.hexdigest()[:16]


def captured_traffic(call):
    """DRAM bytes per launch from the committed ncu capture, or None when the
    kernel sources changed since that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            t = json.load(fh).get(call)
        if t and t.get("sources_sha256") == sources_hash(call):
            return t["bytes"]
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ dist
def dist_setup(n_gpus):
    """One process per GPU over NCCL (see exact_attention_147_b200.ranks)."""
    from exact_attention_147_b200 import ranks
    if n_gpus <= 1 and "WORLD_SIZE" not in os.environ:
        return 0, 1, 0
    return ranks.init("nccl", timeout_s=120.0)


def barrier(world):
    from exact_attention_147_b200 import ranks
    ranks.barrier(world)


def max_over_ranks(x, world):
    from exact_attention_147_b200 import ranks
    return ranks.max_over_ranks(x, world, "cuda")


# ------------------------------------------------------------------ oracle arm
def oracle_sample(seconds: float, w):
    """Time the fp64 oracle (fwd + bwd of whole heads) for about `seconds`."""
    import numpy as np
    import torch

    from exact_attention_147_b200 import workloads as W
    from oracle import attention as oa

    wl = W.Workload("bench", B=1, N=w["N"], H=2, d=w["d"], causal=w["causal"], seed=100)
    q, k, v, do = W.make_inputs(wl, "cpu")
    heads = 0
    t0 = time.perf_counter()
    while True:
        h = heads % 2
        args = [t[0, :, h].to(torch.float64).numpy() for t in (q, k, v, do)]
        oa.head_forward(*args[:3], wl.softmax_scale, w["causal"])
        oa.head_backward(*args, wl.softmax_scale, w["causal"])
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per_head = flops_fwd(1, 1, w["N"], w["d"], w["causal"]) * 3.5
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        cores = os.cpu_count()
    return {"value": per_head * heads / el / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{heads} whole heads (N={w['N']}, d={w['d']}) fwd+bwd in fp64, "
                      f"{el:.1f} s", "seconds": el, "heads": heads}


def run_reference(args):
    """The oracle as the reference arm: each step times it on a bounded
    sample of the workload (whole heads, about one second); ms_per_step is
    that measured time and value the rate over the sampled heads."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = dict(WORKLOAD)
    for _ in range(args.warmup):
        oracle_sample(0.0, w)
    per_step = []
    for _ in range(args.steps):
        per_step.append(oracle_sample(REF_STEP_S, w))
    t_total = sum(r["seconds"] for r in per_step)
    heads_total = sum(r["heads"] for r in per_step)
    per_head = flops_fwd(1, 1, w["N"], w["d"]) * 3.5
    value = per_head * heads_total / t_total / 1e12
    full_step_flops = flops_fwd(w["B"], w["H"], w["N"], w["d"]) * 3.5
    cores = per_step[-1]["cores"]
    sample = (f"each step: whole heads (N={w['N']}, d={w['d']}) of the workload, fwd+bwd in "
              f"fp64, for about {REF_STEP_S:.0f} s; {heads_total} heads over {args.steps} steps")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(w),
        "impl": "reference",
        "sample_flops_per_step": per_head * heads_total / args.steps,
        "ms_per_full_step_extrapolated": full_step_flops / (value * 1e12) * 1e3,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    import torch

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    from exact_attention_147_b200 import fa2 as F
    from exact_attention_147_b200 import workloads as W

    F.load_library()
    w = dict(WORKLOAD)
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    from exact_attention_147_b200 import ranks
    wl = W.Workload("bench", B=B, N=N, H=H, d=d, causal=causal, seed=ranks.batch_seed(1000, rank))
    q, k, v, do = W.make_inputs(wl, "cuda")
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    D = torch.empty_like(lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(1, F.workspace_size(B, N, H, d, torch.bfloat16)), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        F.fwd(q, k, v, None, causal, (-1, -1), None, 0.0, out=out, lse=lse)
        if ev:
            ev[1].record(stream)
        F.bwd_preprocess(out, do, D)
        if ev:
            ev[2].record(stream)
        F.bwd(do, q, k, v, lse, D, None, causal, (-1, -1), None, 0.0, False, dq, dk, dv, ws)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert F.device_status() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    n0 = F.kernel_launches()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    n1 = F.kernel_launches()
    barrier(world)
    clk = clocks.stop()
    ms_total = max_over_ranks(start.elapsed_time(stop), world)
    status = F.device_status()
    assert status == 0, f"device status {status}"

    ms_fwd = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    ms_pre = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms_bwd = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    f_fwd = flops_fwd(B, H, N, d, causal)
    f_step = 3.5 * f_fwd
    ms_step = ms_total / args.steps
    value = ranks.whole_job_rate(f_step, world, ms_step * 1e-3) / 1e12

    # ---- end to end: pinned host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(F, args, world, f_step, (q, k, v, do), (out, lse, dq, dk, dv), D, ws,
                      causal)

    peaks, peak_src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    burst = float(peaks["bf16_tflops"])
    bwd_tflops = 2.5 * f_fwd / (ms_bwd * 1e-3) / 1e12
    fwd_tflops = f_fwd / (ms_fwd * 1e-3) / 1e12
    pre_bytes = 2 * B * N * H * d * 2 + B * H * N * 4
    pre_gbs = pre_bytes / (ms_pre * 1e-3) / 1e9
    dominant = "fa2_bwd" if ms_bwd >= ms_fwd else "fa2_fwd"
    achieved = bwd_tflops if dominant == "fa2_bwd" else fwd_tflops
    traffic = captured_traffic(dominant)
    # The kernels run in a timed region of a few tens of milliseconds at full
    # SM clock (see "clocks"), the condition of the burst GEMM measurement;
    # the sustained figure (seconds of GEMM under the power cap, lower clock)
    # is given beside it.
    roofline = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                "frac": achieved / burst, "traffic": traffic, "kernel": dominant,
                "peak_source": f"{peak_src} bf16_tflops (burst: the call is timed over a "
                               f"short region at full clock)",
                "frac_of_sustained_peak": achieved / sustained}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(w),
        "roofline": roofline,
        "calls": {"fa2_fwd": {"ms": ms_fwd, "tflops": fwd_tflops, "frac": fwd_tflops / burst},
                  "fa2_bwd_preprocess": {"ms": ms_pre, "GB/s": pre_gbs,
                                         "frac_hbm": pre_gbs / float(peaks["hbm_gbs"])},
                  "fa2_bwd": {"ms": ms_bwd, "tflops": bwd_tflops, "frac": bwd_tflops / burst}},
        "gpu_launches": int(n1 - n0),
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = {k2: v2 for k2, v2 in oracle_sample(12.0, w).items()
                                    if k2 in ("value", "unit", "cores", "kind", "sample")}
        except Exception as ex:  # pragma: no cover
            line["cpu_baseline"] = {"error": str(ex)}
    if world == 1 and not args.no_by_n:
        line["by_n"] = run_sweep(F, W, burst)
        line["dropout"] = run_dropout(F, W)
        line["packed"] = run_packed(F, W)
        line["blocksparse"] = run_blocksparse(F, W)
        line["fp8"] = run_fp8(F, W)
        line["long_local"] = run_long_local(F, W)
        line["alibi_det"] = run_alibi_det(F, W)
    if rank == 0:
        print(json.dumps(line), flush=True)
    ranks.finalize(world)
    return 0


def run_dropout(F, W, p=0.1):
    """The bench workload with attention dropout (fwd and bwd timed apart)."""
    import torch
    w = W.mid(False)
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd(q, k, v, dropout_p=p, dropout_seed=5)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, dropout_p=p, dropout_seed=5)
    ws = torch.empty(F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(3):
        F.fwd(q, k, v, dropout_p=p, dropout_seed=5, out=out, lse=lse)
        F.bwd(do, q, k, v, lse, D, dropout_p=p, dropout_seed=5, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.synchronize()
    reps = 10
    ev[0].record()
    for _ in range(reps):
        F.fwd(q, k, v, dropout_p=p, dropout_seed=5, out=out, lse=lse)
    ev[1].record()
    for _ in range(reps):
        F.bwd(do, q, k, v, lse, D, dropout_p=p, dropout_seed=5, dq=dq, dk=dk, dv=dv, workspace=ws)
    ev[2].record()
    torch.cuda.synchronize()
    ff = flops_fwd(w.B, w.H, w.N, w.d)
    tf = ev[0].elapsed_time(ev[1]) / reps
    tb = ev[1].elapsed_time(ev[2]) / reps
    return {"dropout_p": p, "workload": "B=8 H=16 N=2048 d=128", "fwd_ms": round(tf, 4),
            "fwd_tflops": round(ff / (tf * 1e-3) / 1e12, 1), "bwd_ms": round(tb, 4),
            "bwd_tflops": round(2.5 * ff / (tb * 1e-3) / 1e12, 1)}


def _time_pair(fwd_call, bwd_call, reps=10):
    """Mean ms of fwd_call and of bwd_call (CUDA events on the current stream)."""
    import torch
    for _ in range(3):
        fwd_call()
        bwd_call()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for _ in range(reps):
        fwd_call()
    ev[1].record()
    for _ in range(reps):
        bwd_call()
    ev[2].record()
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / reps, ev[1].elapsed_time(ev[2]) / reps


def run_packed(F, W):
    """A packed batch of mixed-length sequences (32768 tokens, lengths 128 to
    4096) against the same sequences padded to the longest one.  TFLOP/s
    count the useful work, sum over sequences of 4 L^2 d H (halved when
    causal); the padded times are for the same useful work."""
    import torch
    res = []
    for causal in (False, True):
        w = W.packed_mix(causal)
        q, k, v, do = W.make_inputs(w, "cuda")
        cu = w.cu_seqlens("cuda")
        out, lse = F.fwd_varlen(q, k, v, cu, w.N, causal=causal)
        D = F.bwd_preprocess(out, do)
        dq, dk, dv = F.bwd_varlen(do, q, k, v, lse, D, cu, w.N, causal=causal)
        ws = torch.empty(F.workspace_size(1, w.total, w.H, w.d, torch.bfloat16),
                         dtype=torch.uint8, device="cuda")
        tf, tb = _time_pair(
            lambda: F.fwd_varlen(q, k, v, cu, w.N, causal=causal, out=out, lse=lse),
            lambda: F.bwd_varlen(do, q, k, v, lse, D, cu, w.N, causal=causal, dq=dq, dk=dk,
                                 dv=dv, workspace=ws))
        ff = sum(flops_fwd(1, w.H, n, w.d, causal) for n in w.lengths)
        # the same sequences padded to the longest, as one padded call
        B, N = w.B, w.N
        qp, kp, vp, dop = (torch.zeros((B, N, w.H, w.d), dtype=t.dtype, device="cuda")
                           for t in (q, k, v, do))
        for b, n in enumerate(w.lengths):
            s = int(sum(w.lengths[:b]))
            for tp, t in ((qp, q), (kp, k), (vp, v), (dop, do)):
                tp[b, :n] = t[s:s + n]
        op_, lp = F.fwd(qp, kp, vp, causal=causal)
        Dp = F.bwd_preprocess(op_, dop)
        gp = F.bwd(dop, qp, kp, vp, lp, Dp, causal=causal)
        wsp = torch.empty(F.workspace_size(B, N, w.H, w.d, torch.bfloat16), dtype=torch.uint8,
                          device="cuda")
        pf, pb = _time_pair(
            lambda: F.fwd(qp, kp, vp, causal=causal, out=op_, lse=lp),
            lambda: F.bwd(dop, qp, kp, vp, lp, Dp, causal=causal, dq=gp[0], dk=gp[1], dv=gp[2],
                          workspace=wsp))
        res.append({"workload": w.name, "sequences": w.B, "max_len": w.N, "tokens": w.total,
                    "causal": causal, "fwd_ms": round(tf, 4),
                    "fwd_tflops": round(ff / (tf * 1e-3) / 1e12, 1), "bwd_ms": round(tb, 4),
                    "bwd_tflops": round(2.5 * ff / (tb * 1e-3) / 1e12, 1),
                    "padded_fwd_ms": round(pf, 4), "padded_bwd_ms": round(pb, 4)})
        del q, k, v, do, out, lse, D, dq, dk, dv, ws, qp, kp, vp, dop, op_, lp, Dp, gp, wsp
        torch.cuda.empty_cache()
    return res


def run_blocksparse(F, W):
    """The bench workload (B=8 H=16 N=2048 d=128) with a local + global
    block mask: a band of 3 blocks around the diagonal plus the first block
    column (60 of 256 blocks kept).  TFLOP/s count the kept blocks only
    (4 * 128 * 128 * d FLOPs each, forward); the dense times are for the
    whole 2048 x 2048 product."""
    import torch
    w = W.mid(False)
    nb = (w.N + 127) // 128
    qb = torch.arange(nb)[:, None]
    kb = torch.arange(nb)[None, :]
    one = (((qb - kb).abs() <= 1) | (kb == 0)).to(torch.uint8)
    mask = one.cuda()[None, None].expand(w.B, w.H, nb, nb)
    kept = int(one.sum())
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd_blocksparse(q, k, v, mask)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd_blocksparse(do, q, k, v, lse, D, mask)
    ws = torch.empty(F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    tf, tb = _time_pair(
        lambda: F.fwd_blocksparse(q, k, v, mask, out=out, lse=lse),
        lambda: F.bwd_blocksparse(do, q, k, v, lse, D, mask, dq=dq, dk=dk, dv=dv, workspace=ws))
    ff = 4.0 * 128 * 128 * w.d * kept * w.B * w.H
    return {"workload": "B=8 H=16 N=2048 d=128, band 3 + first column", "blocks_kept": kept,
            "blocks": nb * nb, "fwd_ms": round(tf, 4),
            "fwd_tflops": round(ff / (tf * 1e-3) / 1e12, 1), "bwd_ms": round(tb, 4),
            "bwd_tflops": round(2.5 * ff / (tb * 1e-3) / 1e12, 1)}


def run_fp8(F, W):
    """e4m3 forward of the bench workload (B=8 H=16 N=2048 d=128), causal and
    not, against the e4m3 dense peak taken as twice the measured bf16 burst
    peak (the nominal e4m3 : bf16 ratio of the tensor cores)."""
    import torch
    peaks, src = load_peaks()
    fp8_peak = 2.0 * float(peaks["bf16_tflops"])
    res = []
    for causal in (False, True):
        w = W.mid(causal)
        q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w, "cuda")
        out, lse = F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=causal)
        tf, _ = _time_pair(lambda: F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=causal, out=out, lse=lse),
                           lambda: None)
        tfl = flops_fwd(w.B, w.H, w.N, w.d, causal) / (tf * 1e-3) / 1e12
        res.append({"workload": "B=8 H=16 N=2048 d=128 e4m3", "causal": causal,
                    "fwd_ms": round(tf, 4), "fwd_tflops": round(tfl, 1),
                    "frac_of_e4m3_peak": round(tfl / fp8_peak, 3),
                    "e4m3_peak": f"2 x {src} bf16_tflops = {fp8_peak:.0f}"})
        del q8, k8, v8, out, lse
    return res


def allowed_pairs(N, causal, wl, wr):
    """Number of visible (query, key) pairs of one head: the FLOP count of a
    windowed call is 4 d per pair (x 2.5 for the backward)."""
    total = 0
    for i in range(N):
        lo = max(0, i - wl) if wl >= 0 else 0
        hi = i if causal else (min(N - 1, i + wr) if wr >= 0 else N - 1)
        total += hi - lo + 1
    return total


def run_long_local(F, W):
    """B=1, H=32, N=32768, d=128, causal, window (4096, 0): fwd and bwd timed
    apart; FLOPs count the visible pairs only."""
    import torch
    w = W.long_local()
    q, k, v, do = W.make_inputs(w, "cuda")
    win = (w.window_left, w.window_right)
    out, lse = F.fwd(q, k, v, causal=True, window_size=win)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, causal=True, window_size=win)
    ws = torch.empty(F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    tf, tb = _time_pair(lambda: F.fwd(q, k, v, causal=True, window_size=win, out=out, lse=lse),
                        lambda: F.bwd(do, q, k, v, lse, D, causal=True, window_size=win, dq=dq, dk=dk,
                                      dv=dv, workspace=ws), reps=5)
    ff = 4.0 * w.B * w.H * w.d * allowed_pairs(w.N, True, w.window_left, w.window_right)
    res = {"workload": "B=1 H=32 N=32768 d=128 causal window (4096, 0)", "flops_fwd": ff,
           "fwd_ms": round(tf, 4), "fwd_tflops": round(ff / (tf * 1e-3) / 1e12, 1),
           "bwd_ms": round(tb, 4), "bwd_tflops": round(2.5 * ff / (tb * 1e-3) / 1e12, 1)}
    del q, k, v, do, out, lse, D, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return res


def run_alibi_det(F, W):
    """B=4, H=16, N=4096, d=128, causal, ALiBi: forward, deterministic backward
    (whose ordered dQ pass recomputes S, P and dS: that work is not counted)
    and, beside it, the atomic backward; plus a bitwise repeat check."""
    import torch
    w = W.alibi_det()
    q, k, v, do = W.make_inputs(w, "cuda")
    sl = w.alibi_slopes().cuda()
    out, lse = F.fwd(q, k, v, causal=True, alibi_slopes=sl)
    D = F.bwd_preprocess(out, do)
    grads = [F.bwd(do, q, k, v, lse, D, causal=True, alibi_slopes=sl, deterministic=True) for _ in range(2)]
    repeat = all(torch.equal(a, b) for a, b in zip(grads[0], grads[1]))
    dq, dk, dv = grads[0]
    ws = {det: torch.empty(max(1, F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16, det)),
                           dtype=torch.uint8, device="cuda") for det in (False, True)}
    bwd = {det: (lambda det=det: F.bwd(do, q, k, v, lse, D, causal=True, alibi_slopes=sl, deterministic=det,
                                       dq=dq, dk=dk, dv=dv, workspace=ws[det])) for det in (False, True)}
    tf, tb_det = _time_pair(lambda: F.fwd(q, k, v, causal=True, alibi_slopes=sl, out=out, lse=lse), bwd[True])
    _, tb = _time_pair(lambda: None, bwd[False])
    ff = flops_fwd(w.B, w.H, w.N, w.d, True)
    res = {"workload": "B=4 H=16 N=4096 d=128 causal ALiBi", "fwd_ms": round(tf, 4),
           "fwd_tflops": round(ff / (tf * 1e-3) / 1e12, 1),
           "bwd_deterministic_ms": round(tb_det, 4),
           "bwd_deterministic_tflops": round(2.5 * ff / (tb_det * 1e-3) / 1e12, 1),
           "bwd_atomic_ms": round(tb, 4), "bwd_atomic_tflops": round(2.5 * ff / (tb * 1e-3) / 1e12, 1),
           "deterministic_bitwise_repeat": bool(repeat)}
    del q, k, v, do, out, lse, D, dq, dk, dv, ws, grads
    torch.cuda.empty_cache()
    return res


def run_sweep(F, W, peak):
    """TFLOP/s of fwd and bwd (timed separately) over the sequence-length
    sweep at 16384 tokens per batch, hidden 2048 as H=16 x d=128 and as
    H=32 x d=64, non-causal and causal; `frac` against the bf16 peak."""
    import torch
    res = []
    for d in (128, 64):
        for n in W.SWEEP_N:
            for causal in (False, True):
                w = W.sweep(n, d, causal)
                q, k, v, do = W.make_inputs(w, "cuda")
                out, lse = F.fwd(q, k, v, causal=causal)
                D = F.bwd_preprocess(out, do)
                dq, dk, dv = F.bwd(do, q, k, v, lse, D, causal=causal)
                ws = torch.empty(max(1, F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16)),
                                 dtype=torch.uint8, device="cuda")
                tf, tb = _time_pair(
                    lambda: F.fwd(q, k, v, causal=causal, out=out, lse=lse),
                    lambda: F.bwd(do, q, k, v, lse, D, causal=causal, dq=dq, dk=dk, dv=dv,
                                  workspace=ws))
                ff = flops_fwd(w.B, w.H, w.N, w.d, causal)
                tff, tfb = ff / (tf * 1e-3) / 1e12, 2.5 * ff / (tb * 1e-3) / 1e12
                res.append({"N": n, "d": d, "H": w.H, "B": w.B, "causal": causal,
                            "fwd_ms": round(tf, 4), "fwd_tflops": round(tff, 1),
                            "fwd_frac": round(tff / peak, 3),
                            "bwd_ms": round(tb, 4), "bwd_tflops": round(tfb, 1),
                            "bwd_frac": round(tfb / peak, 3)})
                del q, k, v, do, out, lse, D, dq, dk, dv, ws
                torch.cuda.empty_cache()
    return res


def run_e2e(F, args, world, f_step, inputs, outputs, D, ws, causal):
    """The step end to end through the public API: every step copies its
    inputs (q, k, v, dO) from pinned host memory and its results (o, lse, dq,
    dk, dv) back.  Copies in, the attention calls and copies out run on three
    streams with two device buffer sets, so step i+1's inputs arrive and step
    i-1's results leave while step i computes; every copy of every timed step
    is inside the timed region."""
    import torch
    from exact_attention_147_b200 import ranks
    hin = [t.cpu().pin_memory() for t in inputs]
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outputs]
    din = [inputs, [torch.empty_like(t) for t in inputs]]
    dout = [outputs, [torch.empty_like(t) for t in outputs]]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    computed = [None, None]   # step that last used buffer set b: its compute is done
    drained = [None, None]    # ... and its results have left

    def pipelined(n):
        for i in range(n):
            b = i % 2
            loaded = ev()
            with torch.cuda.stream(s_in):
                if computed[b] is not None:
                    s_in.wait_event(computed[b])        # step i-2 no longer reads set b
                for dst, src in zip(din[b], hin):
                    dst.copy_(src, non_blocking=True)
                loaded.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(loaded)
                if drained[b] is not None:
                    s_cmp.wait_event(drained[b])        # step i-2's results have left set b
                q, k, v, do = din[b]
                o, lse, dq, dk, dv = dout[b]
                F.fwd(q, k, v, None, causal, (-1, -1), None, 0.0, out=o, lse=lse, stream=s_cmp)
                F.bwd_preprocess(o, do, D, stream=s_cmp)
                F.bwd(do, q, k, v, lse, D, None, causal, (-1, -1), None, 0.0, False, dq, dk, dv,
                      ws, stream=s_cmp)
                computed[b] = ev()
                computed[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                for dst, src in zip(hout, dout[b]):
                    dst.copy_(src, non_blocking=True)
                drained[b] = ev()
                drained[b].record(s_out)

    pipelined(max(2, args.warmup // 2))
    torch.cuda.synchronize()
    ranks.barrier(world)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_cmp)
    s_in.wait_event(start)
    s_out.wait_event(start)
    pipelined(args.steps)
    s_cmp.wait_stream(s_in)
    s_cmp.wait_stream(s_out)
    stop.record(s_cmp)
    torch.cuda.synchronize()
    ranks.barrier(world)
    ms = ranks.max_over_ranks(start.elapsed_time(stop), world, "cuda") / args.steps
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return {"value": ranks.whole_job_rate(f_step, world, ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "pipeline": "copy-in, compute and copy-out streams, two device buffer sets"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libfa2", choices=["libfa2", "reference"])
    ap.add_argument("--no-by-n", action="store_true", help="skip the by-N table")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
