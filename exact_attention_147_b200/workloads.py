"""Seeded synthetic inputs and the workload shapes they are drawn for.

This module holds no attention arithmetic: it only draws random tensors.
Both the CUDA path's tests/bench and the CPU oracle's tests take their
inputs from here, so the two sides see identical values.

Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws, in this order,
q, k, v and dO as float32 N(0, 1) tensors of shape [B, N, H, d]; each is
multiplied by its standard deviation and then cast to the compute dtype
(bf16 or fp32).  The values the GPU receives are therefore exactly the
values the oracle widens to float64.

Packed (variable-length) workloads list their sequence lengths; their
tensors are drawn the same way with shape [total, H, d], total = sum of the
lengths, and ``cu_seqlens`` holds the running sums (int32).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, mask options and input scales."""

    name: str
    B: int
    N: int
    H: int
    d: int
    dtype: torch.dtype = torch.bfloat16
    causal: bool = False
    window_left: int = -1
    window_right: int = -1
    alibi: bool = False
    deterministic: bool = False
    seed: int = 0
    q_std: float = 1.0
    k_std: float = 1.0
    v_std: float = 1.0
    do_std: float = 1.0
    scale: float | None = None
    tags: tuple = field(default_factory=tuple)
    lengths: tuple = ()        # packed workloads: one length per sequence

    @property
    def packed(self) -> bool:
        return len(self.lengths) > 0

    @property
    def total(self) -> int:
        return sum(self.lengths) if self.packed else self.B * self.N

    def cu_seqlens(self, device="cpu"):
        """Running sums [0, L_0, L_0 + L_1, ...] as int32."""
        cu = [0]
        for n in self.lengths:
            cu.append(cu[-1] + n)
        return torch.tensor(cu, dtype=torch.int32, device=device)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    def alibi_slopes(self):
        """slope_h = 2^(-8 (h + 1) / H) for the ALiBi workload (H = 16 gives
        2^(-(h+1)/2)); None when the workload has no ALiBi bias."""
        if not self.alibi:
            return None
        return torch.tensor([2.0 ** (-8.0 * (h + 1) / self.H)
                             for h in range(self.H)], dtype=torch.float32)

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


def make_inputs(w: Workload, device: str | torch.device = "cpu",
                with_grad_out: bool = True):
    """Draw (q, k, v, dO) for workload ``w`` (see the module docstring)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.total, w.H, w.d) if w.packed else (w.B, w.N, w.H, w.d)
    out = []
    stds = (w.q_std, w.k_std, w.v_std, w.do_std)
    for i, std in enumerate(stds):
        if i == 3 and not with_grad_out:
            out.append(None)
            continue
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out.append(t.to(w.dtype).to(device))
    return tuple(out)


def make_fp8_inputs(w: Workload, device: str | torch.device = "cpu"):
    """e4m3 inputs for workload ``w``: q, k, v drawn as in make_inputs (fp32,
    before any cast), each divided by its descale factor max|x| / 448 so that
    it spans the e4m3 range, then cast to torch.float8_e4m3fn.  Returns
    (q8, k8, v8, (q_descale, k_descale, v_descale)); the dequantised inputs
    are x8 * descale."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.N, w.H, w.d)
    out, scales = [], []
    for std in (w.q_std, w.k_std, w.v_std):
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        ds = float(t.abs().max()) / 448.0
        out.append((t / ds).to(torch.float8_e4m3fn).to(device))
        scales.append(ds)
    return out[0], out[1], out[2], tuple(scales)


# ---------------------------------------------------------------------------
# The five workload families.
# ---------------------------------------------------------------------------

def tiny(causal: bool = False, stress: bool = False) -> Workload:
    """B=1, H=2, N=256, d=64 in fp32, seed 0, scale 1/8.  The stress copy
    draws q and k with standard deviation 3 so that scaled logits have
    standard deviation ~9 and the running max is raised often."""
    return Workload(
        name="tiny-fp32" + ("-causal" if causal else "") + ("-stress" if stress else ""),
        B=1, N=256, H=2, d=64, dtype=torch.float32, causal=causal, seed=0,
        q_std=3.0 if stress else 1.0, k_std=3.0 if stress else 1.0,
        scale=1.0 / 8.0)


def mid(causal: bool = False) -> Workload:
    """B=8, H=16, N=2048, d=128, bf16 N(0,1)."""
    return Workload(name="b8-h16-n2048-d128" + ("-causal" if causal else ""),
                    B=8, N=2048, H=16, d=128, causal=causal, seed=1)


SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)


def sweep(n: int, d: int = 128, causal: bool = False) -> Workload:
    """16384 tokens per batch (B = 16384 / N); hidden 2048 as H=16 x d=128 or
    H=32 x d=64."""
    assert n in SWEEP_N and d in (64, 128)
    h = 2048 // d
    return Workload(name=f"sweep-n{n}-h{h}-d{d}" + ("-causal" if causal else ""),
                    B=16384 // n, N=n, H=h, d=d, causal=causal, seed=2)


def long_local() -> Workload:
    """B=1, H=32, N=32768, d=128, causal with window (4096, 0)."""
    return Workload(name="long-local-n32768-w4096", B=1, N=32768, H=32, d=128,
                    causal=True, window_left=4096, window_right=0, seed=3)


def alibi_det() -> Workload:
    """B=4, H=16, N=4096, d=128, causal, ALiBi, deterministic backward."""
    return Workload(name="alibi-det-b4-h16-n4096", B=4, N=4096, H=16, d=128,
                    causal=True, alibi=True, deterministic=True, seed=4)


def packed(name: str, lengths, H: int, d: int, **kw) -> Workload:
    """A packed batch of sequences of the given lengths (B = their number,
    N = the longest, which sizes the grids)."""
    lengths = tuple(int(n) for n in lengths)
    return Workload(name=name, B=len(lengths), N=max(max(lengths), 1), H=H, d=d,
                    lengths=lengths, **kw)


def length_mix(total: int, lo: int, hi: int, seed: int):
    """Sequence lengths drawn uniformly from [lo, hi] (seeded) until they sum
    to ``total`` (the last one is cut to fit)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out, left = [], total
    while left > 0:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        out.append(min(n, left))
        left -= out[-1]
    return tuple(out)


def packed_mix(causal: bool = False, total: int = 32768) -> Workload:
    """``total`` tokens in sequences of 128 to 4096 tokens (uniform, seed 5),
    H=16, d=128, bf16."""
    return packed(f"packed-mix-{total // 1024}k-h16-d128" + ("-causal" if causal else ""),
                  length_mix(total, 128, 4096, seed=5), H=16, d=128, causal=causal, seed=5)


def all_parity_workloads():
    """Every configured workload, in the order they are listed above."""
    ws = [tiny(False), tiny(True), tiny(False, True), tiny(True, True),
          mid(False), mid(True)]
    for d in (128, 64):
        for n in SWEEP_N:
            ws += [sweep(n, d, False), sweep(n, d, True)]
    ws += [long_local(), alibi_det()]
    return ws
