"""Forward parity: libfa2 against the fp64 oracle on the same seeded inputs.

Small shapes are compared element by element over whole tensors (several
128-row tiles, ragged tails, every mask); the full-size workloads are
compared on sampled heads (every element) and on sampled query rows of every
head.
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from tests.helpers import check_fwd, f64, logit_std, oracle_head_fwd, peaked_o_bound

pytestmark = pytest.mark.gpu


def run_fwd(w, q, k, v):
    slopes = w.alibi_slopes()
    out, lse = F.fwd(q, k, v, w.scale, w.causal, (w.window_left, w.window_right),
                     None if slopes is None else slopes.cuda())
    torch.cuda.synchronize()
    assert F.device_status() == 0
    return out, lse


def full_compare(w):
    q, k, v, _ = W.make_inputs(w, "cuda", with_grad_out=False)
    out, lse = run_fwd(w, q, k, v)
    peaked = logit_std(w) > 1.5
    for b in range(w.B):
        for h in range(w.H):
            o_ref, l_ref = oracle_head_fwd(w, q, k, v, b, h)
            o_max = peaked_o_bound(float(v[b, :, h].abs().max())) if peaked else None
            check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype,
                      f"{w.name} b={b} h={h}", o_max=o_max)


SMALL = []
for n in (1, 127, 129, 300, 513):
    for d in (64, 128):
        SMALL.append(W.Workload(f"small-n{n}-d{d}", B=2, N=n, H=2, d=d, seed=n + d))
        SMALL.append(W.Workload(f"small-n{n}-d{d}-causal", B=2, N=n, H=2, d=d, causal=True,
                                seed=n + d + 1))
SMALL += [
    W.Workload("win-130-0", B=1, N=700, H=2, d=128, causal=True, window_left=130,
               window_right=0, seed=11),
    W.Workload("win-5-7", B=1, N=600, H=2, d=64, window_left=5, window_right=7, seed=12),
    W.Workload("win-0-0", B=1, N=300, H=1, d=128, window_left=0, window_right=0, seed=13),
    W.Workload("win-wide", B=1, N=260, H=1, d=128, window_left=5000, window_right=5000, seed=14),
    W.Workload("win-300-left-only", B=1, N=900, H=2, d=128, window_left=300, seed=15),
    W.Workload("alibi-causal", B=2, N=520, H=4, d=128, causal=True, alibi=True, seed=16),
    W.Workload("alibi-noncausal", B=1, N=390, H=3, d=64, alibi=True, seed=17),
    W.Workload("alibi-window", B=1, N=700, H=2, d=128, causal=True, alibi=True,
               window_left=200, window_right=0, seed=18),
    W.Workload("big-logits", B=1, N=640, H=2, d=128, q_std=3.0, k_std=3.0, seed=19),
    W.Workload("big-logits-causal", B=1, N=640, H=2, d=64, causal=True, q_std=4.0, k_std=4.0,
               seed=20),
    W.Workload("scale-0.3", B=1, N=384, H=2, d=128, scale=0.3, seed=21),
    W.Workload("fp32-n300", B=1, N=300, H=2, d=128, dtype=torch.float32, causal=True, seed=22),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_full(w):
    full_compare(w)


@pytest.mark.parametrize("w", [W.tiny(False), W.tiny(True), W.tiny(False, True),
                               W.tiny(True, True)], ids=lambda w: w.name)
def test_tiny_fp32(w):
    full_compare(w)


def sampled_compare(w, heads, n_rows=48):
    q, k, v, _ = W.make_inputs(w, "cuda", with_grad_out=False)
    out, lse = run_fwd(w, q, k, v)
    for b, h in heads:
        o_ref, l_ref = oracle_head_fwd(w, q, k, v, b, h)
        check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype,
                  f"{w.name} head ({b},{h})")
    rng = np.random.default_rng(w.seed)
    rows = np.unique(np.concatenate([[0, w.N - 1, w.N // 2],
                                     rng.integers(0, w.N, size=n_rows)]))
    for b in range(w.B):
        for h in range(w.H):
            o_ref, l_ref = oracle_head_fwd(w, q, k, v, b, h, rows=rows)
            check_fwd(f64(out[b, rows, h]), f64(lse[b, h, rows]), o_ref, l_ref, w.dtype,
                      f"{w.name} rows of ({b},{h})")
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
def test_mid_sampled(causal):
    w = W.mid(causal)
    sampled_compare(w, [(0, 0), (w.B - 1, w.H - 1), (3, 7)])


@pytest.mark.parametrize("n", W.SWEEP_N)
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_sweep_sampled(n, d, causal):
    w = W.sweep(n, d, causal)
    sampled_compare(w, [(w.B - 1, w.H - 1)], n_rows=8)


def test_long_local_sampled():
    # one whole head (every row) and sampled rows of every head
    w = W.long_local()
    sampled_compare(w, [(0, 0)], n_rows=64)


@pytest.mark.parametrize("d,causal", [(128, False), (128, True), (64, True)])
def test_very_long_sequence_sampled(d, causal):
    # one head of 262144 tokens (2048 key blocks, 1024 units): unit counts,
    # TMA row coordinates and the statistics index reach far beyond the
    # workloads' sizes; sampled rows against the oracle
    w = W.Workload(f"long-{d}{'-causal' if causal else ''}", B=1, N=262144, H=1, d=d,
                   causal=causal, seed=140 + d)
    sampled_compare(w, [], n_rows=24)


def test_alibi_sampled():
    w = W.alibi_det()
    sampled_compare(w, [(1, 5)], n_rows=16)


def test_forward_is_bitwise_repeatable():
    w = W.Workload("repeat", B=2, N=1000, H=4, d=128, causal=True, alibi=True, seed=5)
    q, k, v, _ = W.make_inputs(w, "cuda", with_grad_out=False)
    o1, l1 = run_fwd(w, q, k, v)
    o2, l2 = run_fwd(w, q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_strided_inputs():
    """q, k, v as views into one packed [B, N, 3, H, d] buffer."""
    w = W.Workload("packed", B=2, N=333, H=3, d=128, seed=23)
    g = torch.Generator().manual_seed(23)
    qkv = torch.randn(w.B, w.N, 3, w.H, w.d, generator=g).to(torch.bfloat16).cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    out, lse = run_fwd(w, q, k, v)
    for b in range(w.B):
        for h in range(w.H):
            o_ref, l_ref = oa.head_forward(f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]),
                                           w.softmax_scale)
            check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype, "packed")
