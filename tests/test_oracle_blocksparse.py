"""Pins for the oracle's block-sparse masks.

The oracle ANDs an element mask expanded from the block mask into the causal
and window masks.  It is checked against scalar brute force on tiny heads
(block size 2), against PyTorch's float64 scaled_dot_product_attention with
an explicit boolean mask and its autograd, against the special cases that
reduce to the unmasked and causal definitions, and against the fully hidden
rows the block mask makes reachable.  A planted mistake (the block mask read
transposed) must fail the PyTorch pin.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa

RNG = np.random.default_rng(4242)


def brute(q, k, v, scale, bm, block, causal=False, wl=-1, wr=-1, slope=None):
    n, d = q.shape
    o = np.zeros_like(v)
    lse = np.full(n, -math.inf)
    for i in range(n):
        vis = []
        for j in range(n):
            if not bm[i // block][j // block]:
                continue
            if causal and j > i:
                continue
            if wl >= 0 and j < i - wl:
                continue
            if wr >= 0 and j > i + wr:
                continue
            s = scale * sum(q[i, c] * k[j, c] for c in range(d))
            if slope is not None:
                s -= slope * abs(i - j)
            vis.append((j, s))
        if not vis:
            continue
        m = max(s for _, s in vis)
        z = sum(math.exp(s - m) for _, s in vis)
        for j, s in vis:
            o[i] += math.exp(s - m) / z * v[j]
        lse[i] = m + math.log(z)
    return o, lse


@pytest.mark.parametrize("causal,wl,wr,slope", [(False, -1, -1, None), (True, -1, -1, None),
                                                (False, 3, 1, None), (True, 4, 0, 0.3)])
def test_brute_force_block2(causal, wl, wr, slope):
    n, d, block = 9, 3, 2
    nb = (n + block - 1) // block
    q, k, v = (RNG.standard_normal((n, d)) for _ in range(3))
    bm = RNG.random((nb, nb)) < 0.6
    bm[0, 0] = True
    o, lse = oa.head_forward(q, k, v, 0.7, causal, wl, wr, slope, block_mask=bm, block=block)
    ob, lb = brute(q, k, v, 0.7, bm, block, causal, wl, wr, slope)
    assert np.allclose(o, ob, atol=1e-13)
    assert np.array_equal(np.isinf(lse), np.isinf(lb))
    fin = np.isfinite(lb)
    assert np.allclose(lse[fin], lb[fin], atol=1e-13)


def test_all_true_block_mask_is_the_unmasked_definition():
    n, d = 300, 16
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    nb = (n + 127) // 128
    bm = np.ones((nb, nb), dtype=bool)
    o1, l1 = oa.head_forward(q, k, v, 0.25, True, block_mask=bm)
    o2, l2 = oa.head_forward(q, k, v, 0.25, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    g1 = oa.head_backward(q, k, v, do, 0.25, True, block_mask=bm)
    g2 = oa.head_backward(q, k, v, do, 0.25, True)
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)


def test_lower_triangular_blocks_with_causal_is_causal():
    n, d = 400, 8
    q, k, v = (RNG.standard_normal((n, d)) for _ in range(3))
    nb = (n + 127) // 128
    bm = np.tril(np.ones((nb, nb), dtype=bool))
    o1, l1 = oa.head_forward(q, k, v, 0.3, True, block_mask=bm)
    o2, l2 = oa.head_forward(q, k, v, 0.3, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_fully_hidden_block_row():
    n, d = 260, 8
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    bm = np.ones((3, 3), dtype=bool)
    bm[1, :] = False                      # queries 128..255 see nothing
    o, lse = oa.head_forward(q, k, v, 0.3, False, block_mask=bm)
    assert np.all(o[128:256] == 0) and np.all(np.isneginf(lse[128:256]))
    assert np.all(np.isfinite(lse[:128])) and np.all(np.isfinite(lse[256:]))
    dq, dk, dv, dvec = oa.head_backward(q, k, v, do, 0.3, False, block_mask=bm)
    assert np.all(dq[128:256] == 0) and np.all(dvec[128:256] == 0)
    # those queries contribute nothing to dK / dV
    do2 = do.copy()
    do2[128:256] = 0
    _, dk2, dv2, _ = oa.head_backward(q, k, v, do2, 0.3, False, block_mask=bm)
    assert np.allclose(dk, dk2, atol=1e-14) and np.allclose(dv, dv2, atol=1e-14)


def torch_masked(q, k, v, do, scale, mask):
    """float64 SDPA with an explicit boolean mask, and its gradients."""
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt[None, None], kt[None, None], vt[None, None], attn_mask=torch.tensor(mask)[None, None],
        scale=scale)[0, 0]
    (o * torch.tensor(do)).sum().backward()
    return o.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_with_explicit_mask(causal):
    n, d, block = 37, 6, 8
    nb = (n + block - 1) // block
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    bm = RNG.random((nb, nb)) < 0.5
    np.fill_diagonal(bm, True)            # every row keeps its diagonal block
    mask = oa.allowed_mask(np.arange(n), n, causal, -1, -1) & np.kron(
        bm, np.ones((block, block), dtype=bool))[:n, :n]
    o_t, dq_t, dk_t, dv_t = torch_masked(q, k, v, do, 0.4, mask)
    o, _ = oa.head_forward(q, k, v, 0.4, causal, block_mask=bm, block=block)
    dq, dk, dv, _ = oa.head_backward(q, k, v, do, 0.4, causal, block_mask=bm, block=block)
    assert np.allclose(o, o_t, atol=1e-12)
    for a, b in ((dq, dq_t), (dk, dk_t), (dv, dv_t)):
        assert np.allclose(a, b, atol=1e-12)


def test_planted_transposed_block_mask_fails_the_torch_pin():
    n, d, block = 40, 6, 8
    nb = n // block
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    bm = np.tril(RNG.random((nb, nb)) < 0.7) | np.eye(nb, dtype=bool)
    bm[4, 0] = True
    bm[0, 4] = False
    mask = np.kron(bm, np.ones((block, block), dtype=bool))
    o_t = torch_masked(q, k, v, do, 0.4, mask)[0]
    o_bad, _ = oa.head_forward(q, k, v, 0.4, False, block_mask=bm.T, block=block)
    assert not np.allclose(o_bad, o_t, atol=1e-6)
    o_ok, _ = oa.head_forward(q, k, v, 0.4, False, block_mask=bm, block=block)
    assert np.allclose(o_ok, o_t, atol=1e-12)
