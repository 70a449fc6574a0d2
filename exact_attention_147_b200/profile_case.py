"""Run one attention problem a few times, untimed, so that a profiler can
capture its kernels on a case of chosen size.

    python -m exact_attention_147_b200.profile_case --B 4 --N 4096 --H 32 --d 64
        [--causal] [--alibi] [--deterministic] [--dropout P] [--fp8] [--reps 2]

Each repetition launches the forward, the backward preprocessing and the
backward once, in that order, on seeded N(0, 1) bf16 inputs (with --fp8: the
e4m3 forward only, on the same inputs quantised per tensor).  Nothing is
timed or checked against a reference here; the device status word is read at
the end and a non-zero status is an error.
"""

from __future__ import annotations

import argparse
import sys

import torch

from . import fa2 as F
from . import workloads as W


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=4)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--d", type=int, default=128, choices=[64, 128])
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--alibi", action="store_true")
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--dropout", type=float, default=0.0)
    ap.add_argument("--fp8", action="store_true", help="the e4m3 forward only (d = 128)")
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args(argv)
    w = W.Workload("profile-case", B=args.B, N=args.N, H=args.H, d=args.d, causal=args.causal,
                   alibi=args.alibi, deterministic=args.deterministic, seed=2)
    if args.fp8:
        q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w, "cuda")
        out, lse = F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=w.causal)
        for _ in range(args.reps - 1):
            F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=w.causal, out=out, lse=lse)
    else:
        q, k, v, do = W.make_inputs(w, "cuda")
        slopes = w.alibi_slopes()
        sl = None if slopes is None else slopes.cuda()
        kw = dict(causal=w.causal, alibi_slopes=sl, dropout_p=args.dropout, dropout_seed=3)
        out, lse = F.fwd(q, k, v, **kw)
        D = F.bwd_preprocess(out, do)
        dq, dk, dv = F.bwd(do, q, k, v, lse, D, deterministic=w.deterministic, **kw)
        ws = torch.empty(max(1, F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16,
                                                 w.deterministic)),
                         dtype=torch.uint8, device="cuda")
        for _ in range(args.reps - 1):
            F.fwd(q, k, v, out=out, lse=lse, **kw)
            D = F.bwd_preprocess(out, do)
            F.bwd(do, q, k, v, lse, D, deterministic=w.deterministic, dq=dq, dk=dk, dv=dv,
                  workspace=ws, **kw)
    torch.cuda.synchronize()
    status = F.device_status()
    if status != 0:
        print(f"device status {status:#x}", file=sys.stderr)
        return 1
    print(f"ok: B={w.B} N={w.N} H={w.H} d={w.d} causal={w.causal} alibi={w.alibi} "
          f"deterministic={w.deterministic} dropout={args.dropout} fp8={args.fp8} reps={args.reps}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
