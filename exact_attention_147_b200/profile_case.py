"""Run one attention problem a few times, untimed, so that a profiler can
capture its kernels on a case of chosen size.

    python -m exact_attention_147_b200.profile_case --B 4 --N 4096 --H 32 --d 64 [--causal] [--reps 2]

Each repetition launches the forward, the backward preprocessing and the
backward once, in that order, on seeded N(0, 1) bf16 inputs.  Nothing is
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
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args(argv)
    w = W.Workload("profile-case", B=args.B, N=args.N, H=args.H, d=args.d, causal=args.causal, seed=2)
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd(q, k, v, causal=w.causal)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, causal=w.causal)
    ws = torch.empty(F.workspace_size(w.B, w.N, w.H, w.d, torch.bfloat16), dtype=torch.uint8, device="cuda")
    for _ in range(args.reps - 1):
        F.fwd(q, k, v, causal=w.causal, out=out, lse=lse)
        D = F.bwd_preprocess(out, do)
        F.bwd(do, q, k, v, lse, D, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.synchronize()
    status = F.device_status()
    if status != 0:
        print(f"device status {status:#x}", file=sys.stderr)
        return 1
    print(f"ok: B={w.B} N={w.N} H={w.H} d={w.d} causal={w.causal} reps={args.reps}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
