"""Shared helpers for the parity tests: oracle calls on sampled heads/rows
and the tolerance checks stated for this library."""

from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oa


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def head(t: torch.Tensor, b: int, h: int) -> np.ndarray:
    return f64(t[b, :, h])


def slope_of(w, h):
    s = w.alibi_slopes()
    return None if s is None else float(s[h])


def oracle_head_fwd(w, q, k, v, b, h, rows=None):
    qh = head(q, b, h) if rows is None else f64(q[b, rows, h])
    return oa.head_forward(qh, head(k, b, h), head(v, b, h), w.softmax_scale, w.causal,
                           w.window_left, w.window_right, slope_of(w, h),
                           rows=None if rows is None else np.asarray(rows))


def oracle_head_bwd(w, q, k, v, do, b, h):
    return oa.head_backward(head(q, b, h), head(k, b, h), head(v, b, h), head(do, b, h),
                            w.softmax_scale, w.causal, w.window_left, w.window_right,
                            slope_of(w, h))


# Tolerances (fp32 accumulation of bf16 inputs, and fp32 inputs).
BF16_O_MAX, BF16_O_MEAN, BF16_LSE_MAX, BF16_GRAD_REL = 1e-2, 1e-3, 1e-3, 5e-2
BF16_GRAD_FLOOR = 1e-4
F32_TOL = 1e-4


def logit_std(w) -> float:
    """Standard deviation of the scaled logits for the workload's inputs."""
    return w.q_std * w.k_std * w.softmax_scale * (w.d ** 0.5)


def peaked_o_bound(v_max: float) -> float:
    """O error bound when logits are far from N(0,1) (a peaked softmax).

    P enters the PV product as bf16: each weight carries a relative rounding
    error of at most 2^-9, so sum_j p_j d_j v_j / l is at most 2^-9 max|v|;
    rounding O itself to bf16 adds at most 2^-9 |O| <= 2^-9 max|v|.  Total:
    2^-8 max|v|.  (For N(0,1) logits the weights are spread out, the errors
    average, and the fixed 1e-2 bound holds with a wide margin.)  The mean
    bound used with it is a quarter of this maximum."""
    return max(BF16_O_MAX, v_max / 256.0)


def check_fwd(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what="", o_max=None):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite O"
    err = np.abs(o_gpu - o_ref)
    lerr = np.abs(lse_gpu - lse_ref)
    if dtype == torch.float32:
        assert err.max() <= F32_TOL, f"{what}: O max err {err.max():.3e}"
        assert lerr.max() <= F32_TOL, f"{what}: LSE max err {lerr.max():.3e}"
    else:
        bound = BF16_O_MAX if o_max is None else o_max
        assert err.max() <= bound, f"{what}: O max err {err.max():.3e} > {bound:.3e}"
        mean_bound = BF16_O_MEAN if o_max is None else max(BF16_O_MEAN, o_max / 4)
        assert err.mean() <= mean_bound, f"{what}: O mean err {err.mean():.3e}"
        assert lerr.max() <= BF16_LSE_MAX, f"{what}: LSE max err {lerr.max():.3e}"
    return float(err.max()), float(lerr.max())


def d_rounding_bounds(q, k, do, o, scale, causal=False, wl=-1, wr=-1, slope=None,
                      block_mask=None):
    """Per-element bounds on the error a bf16 dQ and dK carry because
    D = rowsum(dO o O) is formed from the bf16-rounded O (the backward pass
    takes O as an input), for one head.

    bf16 keeps 8 significant bits, so |O - bf16(O)| <= 2^-8 |O| and
    |dD_i| <= delta_i = 2^-8 sum_c |dO_ic O_ic|.  dS_ij = P_ij (dP_ij - D_i)
    then carries P_ij dD_i, so
        |err dQ_ic| <= scale delta_i sum_j P_ij |k_jc|,
        |err dK_jc| <= scale sum_i P_ij delta_i |q_ic|.
    These matter where the exact gradient cancels to zero: a query that sees
    a single key has dS = dP - D = 0 exactly, and with dropout O = v / (1-p)
    is no longer exact in bf16.  P comes from the oracle's scores and O is
    the oracle's output."""
    q, k, do, o = (np.asarray(x, dtype=np.float64) for x in (q, k, do, o))
    s = oa.head_scores(q, k, np.arange(q.shape[0]), scale, causal, wl, wr, slope, block_mask)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - np.where(np.isfinite(m), m, 0.0))
    p /= np.maximum(p.sum(axis=1, keepdims=True), 1e-300)
    delta = 2.0 ** -8 * np.abs(do * o).sum(axis=1)
    e_q = scale * delta[:, None] * (p @ np.abs(k))
    e_k = scale * (p.T @ (delta[:, None] * np.abs(q)))
    return e_q, e_k


def check_grad(g_gpu, g_ref, dtype, what="", floor=0.0):
    g_gpu = np.asarray(g_gpu, dtype=np.float64)
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite gradient"
    diff = np.abs(g_gpu - g_ref)
    err = diff.max()
    scale = np.abs(g_ref).max()
    if dtype == torch.float32:
        bound = F32_TOL * max(1.0, scale)
    else:
        # relative to the largest reference gradient, with an absolute floor
        # for gradients that vanish exactly (e.g. one visible key per row,
        # where dS = dP - D cancels to fp32 rounding noise), raised element
        # by element to the D-rounding bounds above where the caller passes them
        bound = np.maximum(max(BF16_GRAD_REL * scale, BF16_GRAD_FLOOR), floor)
    over = diff > bound
    assert not over.any(), (f"{what}: grad max err {err:.3e} > bound "
                            f"{np.max(bound):.3e} at {np.argwhere(over)[0]} (max|ref| {scale:.3e})")
    return float(err), float(scale)


def fp8_o_bound(q, k, v, scale, causal=False, wl=-1, wr=-1, slope=None):
    """Per-element bound on the O error of the e4m3 forward, for one head
    (q, k, v: the dequantised inputs in float64).

    The scores are exact (e4m3 products are exact in fp32).  P enters the
    PV product rounded to e4m3 as p = P_ij * c with P_ij = exp(s_ij - m_i)
    <= 1 and c >= 1 (the kernel's running max never exceeds the row max);
    the rounding error of p is at most max(2^-4 p, 2^-10) (3 mantissa bits;
    half the subnormal spacing), and dividing by l * c leaves at most
    sum_j max(2^-4 P_ij, 2^-10 [P_ij > 0]) |v_jc| / l_i, l_i = sum_j P_ij.
    O is then rounded to bf16: 2^-8 |O|.  A 1e-6 relative term covers the
    fp32 accumulation."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    s = oa.head_scores(q, k, np.arange(q.shape[0]), scale, causal, wl, wr, slope)
    m = s.max(axis=1, keepdims=True)
    P = np.exp(s - np.where(np.isfinite(m), m, 0.0))
    l = np.maximum(P.sum(axis=1, keepdims=True), 1e-300)
    err_p = np.where(P > 0, np.maximum(2.0 ** -4 * P, 2.0 ** -10), 0.0)
    o = (P @ v) / l
    return (err_p @ np.abs(v)) / l + 2.0 ** -8 * np.abs(o) + 1e-6 * (P @ np.abs(v)) / l


def assert_same_sum_any_order(a: torch.Tensor, b: torch.Tensor, what: str = ""):
    """a and b are bf16 roundings of fp32 sums of the same partial terms added
    in two different fixed orders (e.g. the deterministic dQ of the ordered
    in-kernel chain and of the second pass).  The fp32 sums differ only by
    reordering, far below one bf16 step, so the rounded values differ by at
    most one bf16 step (2^-7 relative) -- plus, where the sum cancels to near
    zero, a small absolute term (2^-12 of the largest value)."""
    a64, b64 = a.double(), b.double()
    bound = 2.0 ** -7 * b64.abs() + 2.0 ** -12 * float(b64.abs().max())
    diff = (a64 - b64).abs()
    assert bool((diff <= bound).all()), (
        f"{what}: max diff {float(diff.max()):.3e} beyond one bf16 step")
