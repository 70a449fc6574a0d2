"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a hand-
worked example, closed forms at Q = 0, invariants of softmax attention,
an independent online-softmax implementation, PyTorch's own attention and
autograd in float64, and central finite differences.  The last test plants
plausible mistakes in copies of the oracle and checks that some pin fails.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# --------------------------------------------------------------------------
# Hand-worked golden example
# --------------------------------------------------------------------------

def test_golden_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_softmax.json")))
    q, k, v = (np.array(g[x], dtype=np.float64) for x in ("q", "k", "v"))
    o, lse = oa.head_forward(q, k, v, g["scale"])
    assert np.allclose(o[0], g["expect_O"], atol=1e-14)
    assert abs(lse[0] - g["expect_LSE"]) < 1e-14
    c = g["causal_query_1"]
    o2, lse2 = oa.head_forward(np.array(c["q"]), k, v, g["scale"], causal=True)
    assert np.allclose(o2, c["expect_O"], atol=1e-14)
    assert np.allclose(lse2, c["expect_LSE"], atol=1e-14)
    bw = g["backward"]
    # one query, two keys: pad q/do to the two-row shape head_backward takes
    # by giving the second query a zero upstream gradient.
    q2 = np.vstack([q, q])
    do2 = np.vstack([np.array(bw["do"]), np.zeros((1, 1))])
    dq, dk, dv, _ = oa.head_backward(q2, k, v, do2, g["scale"])
    assert np.allclose(dq[0], bw["expect_dq"], atol=1e-14)
    assert np.allclose(dk, bw["expect_dk"], atol=1e-14)
    assert np.allclose(dv, bw["expect_dv"], atol=1e-14)


# --------------------------------------------------------------------------
# Brute force with scalar Python loops on tiny heads
# --------------------------------------------------------------------------

def brute_head(q, k, v, scale, causal, wl, wr, slope):
    n, d = q.shape
    o = np.zeros_like(v)
    lse = np.zeros(n)
    for i in range(n):
        s = []
        for j in range(n):
            ok = (not causal or j <= i) and (wl < 0 or j >= i - wl) and \
                 (wr < 0 or j <= i + wr)
            if ok:
                x = scale * sum(q[i, c] * k[j, c] for c in range(d))
                if slope is not None:
                    x -= slope * abs(i - j)
                s.append((j, x))
        mx = max(x for _, x in s)
        den = sum(math.exp(x - mx) for _, x in s)
        for j, x in s:
            o[i] += math.exp(x - mx) / den * v[j]
        lse[i] = mx + math.log(den)
    return o, lse


@pytest.mark.parametrize("causal,wl,wr,slope", [
    (False, -1, -1, None), (True, -1, -1, None), (False, 2, 1, None),
    (True, 3, 0, None), (True, -1, -1, 0.5), (False, 1, 2, 0.25),
])
def test_brute_force_tiny(causal, wl, wr, slope):
    n, d = 7, 3
    q, k, v = rand(n, d), rand(n, d), rand(n, d)
    o, lse = oa.head_forward(q, k, v, 0.7, causal, wl, wr, slope)
    ob, lb = brute_head(q, k, v, 0.7, causal, wl, wr, slope)
    assert np.abs(o - ob).max() < 1e-13
    assert np.abs(lse - lb).max() < 1e-13


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1),
                                          (True, 5, 0), (False, 3, 3)])
def test_rows_sum_to_one_and_constant_v(causal, wl, wr):
    n, d = 40, 8
    q, k = rand(n, d, scale=2), rand(n, d, scale=2)
    s = oa.head_scores(q, k, np.arange(n), 0.5, causal, wl, wr, 0.1)
    p, _, _ = oa._softmax_rows(s)
    assert np.abs(p.sum(1) - 1).max() < 1e-13
    assert (p[~oa.allowed_mask(np.arange(n), n, causal, wl, wr)] == 0).all()
    vconst = np.tile(rand(1, d), (n, 1))
    o, _ = oa.head_forward(q, k, vconst, 0.5, causal, wl, wr, 0.1)
    assert np.abs(o - vconst).max() < 1e-13


def test_row_shift_invariance():
    """k_j -> k_j + u adds scale <q_i, u> to every score of row i: O is
    unchanged and LSE_i moves by exactly that amount."""
    n, d = 33, 6
    q, k, v, u = rand(n, d), rand(n, d), rand(n, d), rand(1, d)
    for causal in (False, True):
        o1, l1 = oa.head_forward(q, k, v, 0.9, causal)
        o2, l2 = oa.head_forward(q, k + u, v, 0.9, causal)
        assert np.abs(o1 - o2).max() < 1e-12
        assert np.abs((l2 - l1) - 0.9 * (q @ u[0])).max() < 1e-12


def test_causal_row_zero():
    n, d = 17, 5
    q, k, v = rand(n, d), rand(n, d), rand(n, d)
    o, lse = oa.head_forward(q, k, v, 0.3, causal=True)
    assert np.abs(o[0] - v[0]).max() < 1e-15
    assert abs(lse[0] - 0.3 * q[0] @ k[0]) < 1e-14


# --------------------------------------------------------------------------
# Closed forms at Q = 0
# --------------------------------------------------------------------------

def test_q_zero_closed_forms():
    n, d = 50, 4
    q = np.zeros((n, d))
    k, v = rand(n, d), rand(n, d)
    # non-causal: uniform weights
    o, lse = oa.head_forward(q, k, v, 1.0)
    assert np.abs(o - v.mean(0)).max() < 1e-13
    assert np.abs(lse - math.log(n)).max() < 1e-13
    # causal: mean of the prefix
    o, lse = oa.head_forward(q, k, v, 1.0, causal=True)
    pref = np.cumsum(v, 0) / np.arange(1, n + 1)[:, None]
    assert np.abs(o - pref).max() < 1e-13
    assert np.abs(lse - np.log(np.arange(1, n + 1))).max() < 1e-13
    # causal window (L, 0): mean of the last min(i, L) + 1 rows
    L = 6
    o, lse = oa.head_forward(q, k, v, 1.0, causal=True, window_left=L,
                             window_right=0)
    for i in range(n):
        lo = max(0, i - L)
        assert np.abs(o[i] - v[lo:i + 1].mean(0)).max() < 1e-13
        assert abs(lse[i] - math.log(i - lo + 1)) < 1e-13
    # ALiBi causal: weights r^(i-j), r = exp(-slope)
    slope = 0.3
    r = math.exp(-slope)
    o, lse = oa.head_forward(q, k, v, 1.0, causal=True, slope=slope)
    for i in range(n):
        w = r ** (i - np.arange(i + 1))
        assert np.abs(o[i] - (w[:, None] * v[:i + 1]).sum(0) / w.sum()).max() < 1e-13
        assert abs(lse[i] - math.log((1 - r ** (i + 1)) / (1 - r))) < 1e-12


# --------------------------------------------------------------------------
# Online softmax (the explainer's running max / running sum / running output)
# --------------------------------------------------------------------------

def online_head(q, k, v, scale, causal, wl, wr, slope, block):
    """Independent block-by-block online softmax, written from the
    explainer's description: keep a running max, a running sum of
    exp(score - max) and a running weighted V; rescale both when a block
    raises the max."""
    n, d = q.shape
    o = np.zeros((n, v.shape[1]))
    lse = np.zeros(n)
    for i in range(n):
        m, l, acc = -np.inf, 0.0, np.zeros(v.shape[1])
        for j0 in range(0, n, block):
            js = np.arange(j0, min(n, j0 + block))
            x = scale * (k[js] @ q[i])
            if slope is not None:
                x = x - slope * np.abs(i - js)
            ok = np.ones(len(js), bool)
            if causal:
                ok &= js <= i
            if wl >= 0:
                ok &= js >= i - wl
            if wr >= 0:
                ok &= js <= i + wr
            if not ok.any():
                continue
            x = x[ok]
            m_new = max(m, x.max())
            alpha = math.exp(m - m_new) if np.isfinite(m) else 0.0
            pj = np.exp(x - m_new)
            l = alpha * l + pj.sum()
            acc = alpha * acc + pj @ v[js[ok]]
            m = m_new
        o[i] = acc / l
        lse[i] = m + math.log(l)
    return o, lse


@pytest.mark.parametrize("causal,wl,wr,slope,std", [
    (False, -1, -1, None, 1.0), (True, -1, -1, None, 3.0),
    (True, 20, 0, None, 1.0), (True, -1, -1, 0.2, 1.0), (False, 9, 4, 0.1, 3.0)])
def test_online_equals_two_pass(causal, wl, wr, slope, std):
    n, d = 70, 8
    q, k, v = rand(n, d, scale=std), rand(n, d, scale=std), rand(n, d)
    o, lse = oa.head_forward(q, k, v, 0.35, causal, wl, wr, slope)
    o2, l2 = online_head(q, k, v, 0.35, causal, wl, wr, slope, block=16)
    assert np.abs(o - o2).max() < 1e-12
    assert np.abs(lse - l2).max() < 1e-12


# --------------------------------------------------------------------------
# PyTorch float64 attention and autograd as an outside check
# --------------------------------------------------------------------------

def torch_reference(q, k, v, do, scale, causal, wl, wr, slope):
    n = q.shape[0]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    ok = torch.tensor(oa.allowed_mask(np.arange(n), n, causal, wl, wr))
    bias = torch.zeros(n, n, dtype=torch.float64)
    if slope is not None:
        idx = torch.arange(n, dtype=torch.float64)
        bias = -slope * (idx[:, None] - idx[None, :]).abs()
    bias = bias.masked_fill(~ok, float("-inf"))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt[None, None], kt[None, None], vt[None, None], attn_mask=bias,
        scale=scale)[0, 0]
    o.backward(torch.tensor(do, dtype=torch.float64))
    lse = torch.logsumexp(scale * qt.detach() @ kt.detach().T + bias, dim=1)
    return (o.detach().numpy(), lse.numpy(), qt.grad.numpy(),
            kt.grad.numpy(), vt.grad.numpy())


@pytest.mark.parametrize("causal,wl,wr,slope", [
    (False, -1, -1, None), (True, -1, -1, None), (True, 11, 0, None),
    (True, -1, -1, 0.35), (False, 7, 3, 0.1)])
def test_against_torch_fp64(causal, wl, wr, slope):
    n, d = 48, 16
    q, k, v, do = rand(n, d, scale=2), rand(n, d, scale=2), rand(n, d), rand(n, d)
    o, lse = oa.head_forward(q, k, v, 0.25, causal, wl, wr, slope)
    dq, dk, dv, dvec = oa.head_backward(q, k, v, do, 0.25, causal, wl, wr, slope)
    ro, rl, rdq, rdk, rdv = torch_reference(q, k, v, do, 0.25, causal, wl, wr, slope)
    assert np.abs(o - ro).max() < 1e-12
    assert np.abs(lse - rl).max() < 1e-12
    assert np.abs(dq - rdq).max() < 1e-11
    assert np.abs(dk - rdk).max() < 1e-11
    assert np.abs(dv - rdv).max() < 1e-11


# --------------------------------------------------------------------------
# Central finite differences of L = sum(O * dO)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal,wl,wr,slope", [
    (False, -1, -1, None), (True, -1, -1, 0.3), (True, 4, 0, None)])
def test_finite_differences(causal, wl, wr, slope):
    n, d, scale, h = 12, 4, 0.6, 1e-6
    q, k, v, do = rand(n, d), rand(n, d), rand(n, d), rand(n, d)
    grads = oa.head_backward(q, k, v, do, scale, causal, wl, wr, slope)[:3]

    def loss(qq, kk, vv):
        o, _ = oa.head_forward(qq, kk, vv, scale, causal, wl, wr, slope)
        return float((o * do).sum())

    for which, g in enumerate(grads):
        fd = np.zeros((n, d))
        for i in range(n):
            for c in range(d):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][i, c] += h
                args_m[which][i, c] -= h
                fd[i, c] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        rel = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert rel < 1e-6, (which, rel)


# --------------------------------------------------------------------------
# Gradient invariants
# --------------------------------------------------------------------------

def test_gradient_invariants():
    n, d = 37, 8
    q, k, v, do = rand(n, d), rand(n, d), rand(n, d), rand(n, d)
    for causal, slope in ((False, None), (True, 0.2)):
        dq, dk, dv, dvec = oa.head_backward(q, k, v, do, 0.4, causal,
                                            slope=slope)
        # sum_j dS_ij = 0  =>  sum_j dK_j = 0
        assert np.abs(dk.sum(0)).max() < 1e-12
        # D_i = sum_j P_ij dP_ij
        s = oa.head_scores(q, k, np.arange(n), 0.4, causal, -1, -1, slope)
        p, _, _ = oa._softmax_rows(s)
        assert np.abs(dvec - (p * (do @ v.T)).sum(1)).max() < 1e-12
        # zero upstream gradient gives zero gradients
        z = oa.head_backward(q, k, v, np.zeros_like(do), 0.4, causal,
                             slope=slope)
        assert all(np.abs(t).max() == 0 for t in z)


def test_fully_hidden_row_is_zero():
    s = np.array([[-np.inf, -np.inf], [0.0, 1.0]])
    p, m, l = oa._softmax_rows(s)
    assert (p[0] == 0).all() and m[0] == -np.inf and l[0] == 0
    assert abs(p[1].sum() - 1) < 1e-15


def test_batched_layout_and_rows():
    b, n, h, d = 2, 20, 3, 4
    q, k, v, do = (rand(b, n, h, d) for _ in range(4))
    slopes = [0.1, 0.2, 0.3]
    o, lse = oracle.attention_forward(q, k, v, 0.5, True, alibi_slopes=slopes)
    for bb in range(b):
        for hh in range(h):
            oh, lh = oa.head_forward(q[bb, :, hh], k[bb, :, hh], v[bb, :, hh],
                                     0.5, True, slope=slopes[hh])
            assert np.array_equal(o[bb, :, hh], oh)
            assert np.array_equal(lse[bb, hh], lh)
    rows = [0, 7, 19]
    orow, lrow = oracle.attention_forward_rows(q, k, v, 1, 2, rows, 0.5, True,
                                               alibi_slopes=slopes)
    assert np.abs(orow - o[1, rows, 2]).max() < 1e-14
    assert np.abs(lrow - lse[1, 2, rows]).max() < 1e-14
    dvec_full = oracle.attention_backward(q, k, v, do, 0.5, True,
                                          alibi_slopes=slopes)[3]
    assert np.abs(oracle.bwd_preprocess(o, do) - dvec_full).max() < 1e-13


def test_row_chunking_matches(monkeypatch):
    n, d = 64, 4
    q, k, v, do = rand(n, d), rand(n, d), rand(n, d), rand(n, d)
    full_f = oa.head_forward(q, k, v, 0.5, True)
    full_b = oa.head_backward(q, k, v, do, 0.5, True)
    monkeypatch.setattr(oa, "_MAX_SCORE_ELEMS", 64 * 5)
    ch_f = oa.head_forward(q, k, v, 0.5, True)
    ch_b = oa.head_backward(q, k, v, do, 0.5, True)
    for a, c in zip(full_f + full_b, ch_f + ch_b):
        assert np.abs(a - c).max() < 1e-13


# --------------------------------------------------------------------------
# Planted mistakes: each must be caught by at least one pin above
# --------------------------------------------------------------------------

def _mutants():
    def no_d_term(q, k, v, do, scale, causal=False, wl=-1, wr=-1, slope=None):
        n = q.shape[0]
        s = oa.head_scores(q, k, np.arange(n), scale, causal, wl, wr, slope)
        p, _, _ = oa._softmax_rows(s)
        dp = do @ v.T
        ds = p * dp                                  # dropped "- D"
        return scale * ds @ k, scale * ds.T @ q, p.T @ do, None

    def transposed_dk(q, k, v, do, scale, causal=False, wl=-1, wr=-1, slope=None):
        n = q.shape[0]
        s = oa.head_scores(q, k, np.arange(n), scale, causal, wl, wr, slope)
        p, _, _ = oa._softmax_rows(s)
        o = p @ v
        dp = do @ v.T
        ds = p * (dp - (do * o).sum(1)[:, None])
        return scale * ds @ k, scale * ds @ q, p.T @ do, None   # ds, not ds.T

    return {"no_d_term": no_d_term, "transposed_dk": transposed_dk}


@pytest.mark.parametrize("name", ["no_d_term", "transposed_dk"])
def test_planted_gradient_mistakes_are_caught(name):
    mut = _mutants()[name]
    n, d = 12, 4
    q, k, v, do = rand(n, d), rand(n, d), rand(n, d), rand(n, d)
    ro, rl, rdq, rdk, rdv = torch_reference(q, k, v, do, 0.6, True, -1, -1, None)
    dq, dk, dv, _ = mut(q, k, v, do, 0.6, True)
    assert max(np.abs(dq - rdq).max(), np.abs(dk - rdk).max(),
               np.abs(dv - rdv).max()) > 1e-3


def test_planted_mask_mistake_is_caught(monkeypatch):
    """An off-by-one causal mask (j < i instead of j <= i) breaks the
    causal-row-0 and Q = 0 closed-form pins."""
    real = oa.allowed_mask

    def wrong(rows, n_keys, causal, wl, wr):
        ok = real(rows, n_keys, False, wl, wr)
        if causal:
            i = np.asarray(rows)[:, None]
            j = np.arange(n_keys)[None, :]
            ok &= j < i
            ok[:, 0] = True      # keep row 0 finite
        return ok

    monkeypatch.setattr(oa, "allowed_mask", wrong)
    n, d = 10, 3
    q = np.zeros((n, d))
    v = rand(n, d)
    o, lse = oa.head_forward(q, rand(n, d), v, 1.0, causal=True)
    pref = np.cumsum(v, 0) / np.arange(1, n + 1)[:, None]
    assert np.abs(o - pref).max() > 1e-3
