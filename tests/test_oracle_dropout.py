"""Pins for the oracle's dropout: the counter-based generator and the way a
dropout mask enters attention and its gradient.

The generator is checked for what a counter-based RNG must give (a
deterministic function of (counter, key), distinct outputs for distinct
counters, uniform bytes, the kept fraction the threshold promises); the
dropout arithmetic is checked against unbiasedness (the mean over masks is
the un-dropped output), PyTorch float64 autograd and finite differences.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import philox

RNG = np.random.default_rng(777)


# Known-answer vectors of Philox4x32-10 published with the generator's
# reference implementation (Random123, the "kat_vectors" file that
# accompanies Salmon et al., SC 2011): (counter c0..c3, key k0, k1) ->
# output words.  A wrong multiplier, Weyl constant, round count or word
# order changes every one of them.
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF), (0xFFFFFFFF, 0xFFFFFFFF),
     (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,expect", PHILOX_KAT)
def test_philox_known_answers(ctr, key, expect):
    got = philox.philox4x32_10(*[np.uint32(c) for c in ctr], *key)
    assert tuple(int(x) for x in got) == expect


def test_philox_known_answers_vectorised():
    # the same vectors through the broadcasting path the mask generator uses
    c = np.array([v[0] for v in PHILOX_KAT], dtype=np.uint32).T
    for (ctr, key, expect), col in zip(PHILOX_KAT, range(c.shape[1])):
        got = philox.philox4x32_10(c[0], c[1], c[2], c[3], *key)
        assert tuple(int(w[col]) for w in got) == expect


def test_philox_is_a_deterministic_function_of_counter_and_key():
    c = RNG.integers(0, 2**32, size=(4, 1000), dtype=np.uint64).astype(np.uint32)
    a = philox.philox4x32_10(*c, 123, 456)
    b = philox.philox4x32_10(*c, 123, 456)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    d = philox.philox4x32_10(*c, 124, 456)
    assert not np.array_equal(a[0], d[0])


def test_philox_distinct_counters_give_distinct_blocks():
    n = 200000
    c0 = np.arange(n, dtype=np.uint32)
    out = philox.philox4x32_10(c0, 0, 0, 0, 7, 9)
    blocks = np.stack(out, axis=1).view(np.dtype((np.void, 16)))
    assert len(np.unique(blocks)) == n


def test_random_bytes_uniform_and_keep_fraction():
    bytes_ = philox.random_bytes(1, 3, np.arange(512), 512, seed=2024).ravel()
    counts = np.bincount(bytes_, minlength=256)
    expect = bytes_.size / 256
    chi2 = ((counts - expect) ** 2 / expect).sum()
    # 255 degrees of freedom: mean 255, sd ~22.6; 8 sd margin
    assert chi2 < 255 + 8 * math.sqrt(2 * 255)
    for p in (0.1, 0.25, 0.5, 0.9):
        keep = philox.keep_mask(0, 0, np.arange(512), 512, p, seed=5)
        t = philox.dropout_threshold(p)
        q = (256 - t) / 256
        sd = math.sqrt(q * (1 - q) / keep.size)
        assert abs(keep.mean() - q) < 6 * sd


def test_neighbouring_elements_uncorrelated():
    b = philox.random_bytes(0, 0, np.arange(256), 256, seed=99).astype(np.float64)
    x = (b - b.mean()) / b.std()
    for ax in (0, 1):
        r = (x * np.roll(x, 1, axis=ax)).mean()
        assert abs(r) < 6 / math.sqrt(x.size)


def test_threshold_and_scale():
    assert philox.dropout_threshold(0.0) == 0 and philox.keep_scale(0.0) == 1.0
    assert philox.dropout_threshold(0.5) == 128 and philox.keep_scale(0.5) == 2.0
    assert philox.dropout_threshold(0.1) == 26
    assert abs(philox.keep_scale(0.1) - 256 / 230) < 1e-15
    with pytest.raises(ValueError):
        philox.dropout_threshold(0.999)


def test_zero_dropout_keeps_everything():
    keep = philox.keep_mask(1, 1, np.arange(64), 64, 0.0, seed=1)
    assert keep.all()


def test_dropout_is_unbiased():
    """The mean of the dropped output over many masks is the un-dropped
    output (kept probabilities are scaled by 1 / keep probability)."""
    n, d, p = 12, 3, 0.3
    q, k, v = RNG.standard_normal((n, d)), RNG.standard_normal((n, d)), RNG.standard_normal((n, d))
    o_ref, lse_ref = oa.head_forward(q, k, v, 0.5, causal=True)
    acc = np.zeros_like(o_ref)
    n_masks = 4000
    for seed in range(n_masks):
        keep = philox.keep_mask(0, 0, np.arange(n), n, p, seed)
        o, lse = oa.head_forward(q, k, v, 0.5, causal=True, keep=keep,
                                 keep_scale=philox.keep_scale(p))
        assert np.array_equal(lse, lse_ref)      # LSE ignores dropout
        acc += o
    mean = acc / n_masks
    # per-element standard error is at most ~ max|v| * sqrt(s-1) / sqrt(n_masks)
    se = np.abs(v).max() * math.sqrt(philox.keep_scale(p) - 1) / math.sqrt(n_masks)
    assert np.abs(mean - o_ref).max() < 6 * se


def torch_dropout_reference(q, k, v, do, scale, causal, keep, ks):
    n = q.shape[0]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = scale * qt @ kt.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    pr = torch.softmax(s, dim=1)
    o = (pr * torch.tensor(keep, dtype=torch.float64) * ks) @ vt
    o.backward(torch.tensor(do, dtype=torch.float64))
    return o.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("p,causal", [(0.1, False), (0.5, True), (0.25, True)])
def test_dropout_against_torch_autograd(p, causal):
    n, d = 40, 8
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    keep = philox.keep_mask(1, 2, np.arange(n), n, p, seed=31)
    ks = philox.keep_scale(p)
    o, _ = oa.head_forward(q, k, v, 0.4, causal, keep=keep, keep_scale=ks)
    dq, dk, dv, dvec = oa.head_backward(q, k, v, do, 0.4, causal, keep=keep, keep_scale=ks)
    ro, rdq, rdk, rdv = torch_dropout_reference(q, k, v, do, 0.4, causal, keep, ks)
    assert np.abs(o - ro).max() < 1e-12
    assert np.abs(dq - rdq).max() < 1e-11
    assert np.abs(dk - rdk).max() < 1e-11
    assert np.abs(dv - rdv).max() < 1e-11
    assert np.abs(dvec - (do * o).sum(1)).max() < 1e-12


def test_dropout_finite_differences():
    n, d, scale, h, p = 10, 3, 0.7, 1e-6, 0.4
    q, k, v, do = (RNG.standard_normal((n, d)) for _ in range(4))
    keep = philox.keep_mask(0, 1, np.arange(n), n, p, seed=8)
    ks = philox.keep_scale(p)
    grads = oa.head_backward(q, k, v, do, scale, True, keep=keep, keep_scale=ks)[:3]

    def loss(qq, kk, vv):
        o, _ = oa.head_forward(qq, kk, vv, scale, True, keep=keep, keep_scale=ks)
        return float((o * do).sum())

    for which, g in enumerate(grads):
        fd = np.zeros((n, d))
        for i in range(n):
            for c in range(d):
                a_p = [q.copy(), k.copy(), v.copy()]
                a_m = [q.copy(), k.copy(), v.copy()]
                a_p[which][i, c] += h
                a_m[which][i, c] -= h
                fd[i, c] = (loss(*a_p) - loss(*a_m)) / (2 * h)
        assert np.abs(fd - g).max() / max(1.0, np.abs(g).max()) < 1e-6


def test_planted_missing_rescale_is_caught():
    """Forgetting the 1 / keep-probability factor biases the output."""
    n, d, p = 12, 3, 0.5
    q, k, v = RNG.standard_normal((n, d)), RNG.standard_normal((n, d)), RNG.standard_normal((n, d)) + 3
    o_ref, _ = oa.head_forward(q, k, v, 0.5)
    acc = np.zeros_like(o_ref)
    for seed in range(500):
        keep = philox.keep_mask(0, 0, np.arange(n), n, p, seed)
        acc += oa.head_forward(q, k, v, 0.5, keep=keep, keep_scale=1.0)[0]   # planted mistake
    assert np.abs(acc / 500 - o_ref).max() > 0.5
