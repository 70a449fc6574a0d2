"""Block-sparse masks: libfa2 against the fp64 oracle.

Random 128 x 128 block masks (ragged N, every mask option, dropout, the
deterministic backward, fp32), block rows the mask hides completely, masks
shared across batch and heads through zero strides, the all-ones mask bit
for bit against the padded kernels, and a local + global pattern on the
bench-sized workload (sampled heads).
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from oracle import philox
from tests.helpers import assert_same_sum_any_order, check_fwd, check_grad, d_rounding_bounds, f64

pytestmark = pytest.mark.gpu


def random_mask(B, H, N, density, seed, keep_diag=True):
    nb = (N + 127) // 128
    g = torch.Generator().manual_seed(seed)
    m = torch.rand((B, H, nb, nb), generator=g) < density
    if keep_diag:
        m |= torch.eye(nb, dtype=torch.bool)
    return m.to(torch.uint8)


def run(w, mask, dropout_p=0.0, seed=0):
    q, k, v, do = W.make_inputs(w, "cuda")
    slopes = w.alibi_slopes()
    sl = None if slopes is None else slopes.cuda()
    win = (w.window_left, w.window_right)
    m = mask.cuda()
    out, lse = F.fwd_blocksparse(q, k, v, m, w.scale, w.causal, win, sl, dropout_p,
                                 dropout_seed=seed)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd_blocksparse(do, q, k, v, lse, D, m, w.scale, w.causal, win, sl, dropout_p,
                                   w.deterministic, dropout_seed=seed)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    return (q, k, v, do), (out, lse, dq, dk, dv)


def compare(w, mask, ins, outs, heads=None, dropout_p=0.0, seed=0):
    q, k, v, do = ins
    out, lse, dq, dk, dv = outs
    slopes = w.alibi_slopes()
    ks = philox.keep_scale(dropout_p) if dropout_p > 0 else 1.0
    pairs = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in pairs:
        bm = mask[b, h].numpy().astype(bool)
        keep = (philox.keep_mask(b, h, np.arange(w.N), w.N, dropout_p, seed)
                if dropout_p > 0 else None)
        slope = None if slopes is None else float(slopes[h])
        args = (f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]))
        kw = dict(keep=keep, keep_scale=ks, block_mask=bm)
        o_ref, l_ref = oa.head_forward(*args, w.softmax_scale, w.causal, w.window_left,
                                       w.window_right, slope, **kw)
        tag = f"{w.name} ({b},{h})"
        dead = np.isneginf(l_ref)
        got_l = f64(lse[b, h])
        assert np.array_equal(np.isneginf(got_l), dead), tag + ": hidden rows differ"
        assert np.all(f64(out[b, dead, h]) == 0.0), tag + ": hidden rows must give O = 0"
        l_cmp = np.where(dead, 0.0, l_ref)
        o_max = None
        if dropout_p > 0 and w.dtype == torch.bfloat16:
            o_max = max(1e-2, ks * float(v[b, :, h].abs().max()) / 256.0)
        check_fwd(f64(out[b, :, h]), np.where(dead, 0.0, got_l), o_ref, l_cmp, w.dtype, tag,
                  o_max=o_max)
        rdq, rdk, rdv, _ = oa.head_backward(*args, f64(do[b, :, h]), w.softmax_scale, w.causal,
                                            w.window_left, w.window_right, slope, **kw)
        fq, fk = d_rounding_bounds(args[0], args[1], f64(do[b, :, h]), o_ref, w.softmax_scale,
                                   w.causal, w.window_left, w.window_right, slope, bm)
        check_grad(f64(dq[b, :, h]), rdq, w.dtype, tag + " dq", floor=fq)
        check_grad(f64(dk[b, :, h]), rdk, w.dtype, tag + " dk", floor=fk)
        check_grad(f64(dv[b, :, h]), rdv, w.dtype, tag + " dv")
        assert np.all(f64(dq[b, dead, h]) == 0.0), tag + ": hidden rows must give dQ = 0"


CASES = [
    (W.Workload("bs-n300-d128", B=2, N=300, H=2, d=128, seed=91), 0.5),
    (W.Workload("bs-n700-d64", B=1, N=700, H=2, d=64, seed=92), 0.4),
    (W.Workload("bs-n640-causal", B=1, N=640, H=3, d=128, causal=True, seed=93), 0.5),
    (W.Workload("bs-window", B=1, N=900, H=2, d=128, causal=True, window_left=300,
                window_right=0, seed=94), 0.6),
    (W.Workload("bs-alibi", B=1, N=520, H=2, d=128, causal=True, alibi=True, seed=95), 0.5),
    (W.Workload("bs-det", B=1, N=600, H=2, d=128, causal=True, deterministic=True, seed=96), 0.5),
    (W.Workload("bs-det-d64", B=2, N=384, H=1, d=64, deterministic=True, seed=97), 0.3),
    (W.Workload("bs-fp32", B=1, N=260, H=2, d=64, dtype=torch.float32, causal=True, seed=98,
                scale=1.0 / 8.0), 0.5),
]


@pytest.mark.parametrize("w,density", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_blocksparse_parity(w, density):
    mask = random_mask(w.B, w.H, w.N, density, w.seed)
    ins, outs = run(w, mask)
    compare(w, mask, ins, outs)


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_blocksparse_dropout(p):
    w = W.Workload("bs-drop", B=1, N=520, H=2, d=128, causal=True, seed=99)
    mask = random_mask(w.B, w.H, w.N, 0.5, 7)
    ins, outs = run(w, mask, p, 555)
    compare(w, mask, ins, outs, dropout_p=p, seed=555)


@pytest.mark.parametrize("det", [False, True])
def test_hidden_block_rows_and_columns(det):
    """Query block 1 sees nothing; key block 2 is seen by nobody."""
    w = W.Workload("bs-hidden", B=1, N=520, H=2, d=128, seed=100, deterministic=det)
    mask = torch.ones((1, 2, 5, 5), dtype=torch.uint8)
    mask[:, :, 1, :] = 0
    mask[:, :, :, 2] = 0
    ins, outs = run(w, mask)
    compare(w, mask, ins, outs)
    _, _, dq, dk, dv = outs
    assert torch.all(dk[0, 256:384] == 0) and torch.all(dv[0, 256:384] == 0)


def test_shared_mask_zero_strides():
    w = W.Workload("bs-shared", B=2, N=400, H=3, d=128, causal=True, seed=101)
    one = random_mask(1, 1, w.N, 0.5, 3)
    mask = one.expand(w.B, w.H, -1, -1)          # batch and head strides 0
    ins, outs = run(w, mask)
    compare(w, mask.contiguous(), ins, outs)


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_equals_padded_kernels_bitwise(causal):
    w = W.Workload("bs-ones", B=2, N=700, H=2, d=128, causal=causal, seed=102, deterministic=True)
    mask = torch.ones((w.B, w.H, 6, 6), dtype=torch.uint8)
    (q, k, v, do), (out, lse, dq, dk, dv) = run(w, mask)
    o2, l2 = F.fwd(q, k, v, causal=causal)
    D = F.bwd_preprocess(o2, do)
    g = F.bwd(do, q, k, v, l2, D, causal=causal, deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(out, o2) and torch.equal(lse, l2)
    assert torch.equal(dk, g[1]) and torch.equal(dv, g[2])
    if causal:
        # the padded causal call adds dQ in its in-kernel order (descending key
        # block), the block-sparse one in its second pass (ascending)
        assert_same_sum_any_order(dq, g[0], "dq")
    else:
        assert torch.equal(dq, g[0])


def test_local_global_pattern_bench_size():
    """B=8 H=16 N=2048 d=128 with a band of 3 blocks plus the first block
    column (a local + global pattern), sampled heads."""
    w = W.mid(False)
    nb = 16
    qb = torch.arange(nb)[:, None]
    kb = torch.arange(nb)[None, :]
    one = ((qb - kb).abs() <= 1) | (kb == 0)
    mask = one.to(torch.uint8)[None, None].expand(w.B, w.H, nb, nb)
    ins, outs = run(w, mask)
    compare(w, mask.contiguous(), ins, outs, heads=[(0, 0), (7, 15)])


def test_autograd_blocksparse():
    w = W.Workload("bs-ag", B=1, N=300, H=2, d=128, causal=True, seed=103)
    q, k, v, do = W.make_inputs(w, "cuda")
    mask = random_mask(1, 2, w.N, 0.5, 5).cuda()
    qg = q.clone().requires_grad_(True)
    out = F.flash_attention_v2_blocksparse(qg, k, v, mask.bool(), causal=True)
    out.backward(do)
    o_ref, _ = F.fwd_blocksparse(q, k, v, mask, causal=True)
    assert torch.equal(out.detach(), o_ref)
    assert torch.isfinite(qg.grad).all()
