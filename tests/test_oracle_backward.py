"""Pins of the oracle's attention gradients (oracle/backward.py) against
things other than its own formulas: torch's autograd through its scaled-dot-
product attention in fp64 (a library routine that derives the gradient from
the forward alone), central finite differences of the pinned forward oracle,
the textbook special cases k = 1 (token-causal) and k >= n (bidirectional),
and two invariants of the softmax Jacobian.

Source: papernotes.org note "DiT as Real-Time Rerenderer", Method > Key
Designs 2 (the attention equation and mask M) and Key Designs 3 (the student
is trained by gradient descent -- Self Forcing, DMD -- through it).
"""
import math

import numpy as np
import pytest
import torch

import oracle


def inputs(n, H, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((n, H, d)) * scale for _ in range(4)]


def autograd_grads(q, k, v, do, mask):
    """dQ, dK, dV of sum(dO * O) by torch autograd through F.sdpa in fp64."""
    tq, tk, tv = (torch.tensor(a.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.tensor(mask) if mask is not None else None)
    out.backward(torch.tensor(do.transpose(1, 0, 2)))
    return [t.grad.numpy().transpose(1, 0, 2) for t in (tq, tk, tv)]


def frame_mask(n, k):
    f = np.arange(n) // k
    return f[None, :] <= f[:, None]


@pytest.mark.parametrize("n,k,H,d", [(12, 3, 2, 8), (17, 4, 1, 16), (9, 2, 3, 4), (40, 7, 2, 32)])
def test_backward_matches_autograd(n, k, H, d):
    q, kk, v, do = inputs(n, H, d, n * 10 + k)
    got = oracle.prefill_backward(q, kk, v, do, k)
    want = autograd_grads(q, kk, v, do, frame_mask(n, k))
    for g, w, name in zip(got, want, "qkv"):
        assert np.allclose(g, w, rtol=1e-10, atol=1e-12), f"d{name}"


@pytest.mark.parametrize("n,H,d", [(11, 2, 8), (33, 1, 16)])
def test_textbook_reductions(n, H, d):
    """k = 1: token-causal (is_causal=True); k >= n: bidirectional."""
    q, kk, v, do = inputs(n, H, d, n)
    for k, causal in ((1, True), (n, False), (n + 5, False)):
        got = oracle.prefill_backward(q, kk, v, do, k)
        tq, tk, tv = (torch.tensor(a.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
                      for a in (q, kk, v))
        torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal).backward(
            torch.tensor(do.transpose(1, 0, 2)))
        for g, t in zip(got, (tq, tk, tv)):
            assert np.allclose(g, t.grad.numpy().transpose(1, 0, 2), rtol=1e-10, atol=1e-12), (k, causal)


def test_finite_differences_of_forward_oracle():
    """Central differences of L = sum(dO * O), O from the (separately pinned)
    C forward oracle, at a spread of entries of Q, K and V."""
    n, k, H, d = 7, 2, 1, 4
    q, kk, v, do = inputs(n, H, d, 3)
    dq, dk, dv = oracle.prefill_backward(q, kk, v, do, k)

    def loss(q_, k_, v_):
        return float(np.sum(do * oracle.prefill(q_, k_, v_, k)))

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for (i, hh, e) in [(0, 0, 0), (3, 0, 2), (6, 0, 3), (4, 0, 1)]:
            args = [q.copy(), kk.copy(), v.copy()]
            args[which][i, hh, e] += h
            lp = loss(*args)
            args[which][i, hh, e] -= 2 * h
            lm = loss(*args)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[i, hh, e]) <= 1e-6 * max(1.0, abs(fd)), (which, i, e, fd, grad[i, hh, e])


def test_softmax_jacobian_invariants():
    """Rows of dS sum to zero, so sum_j dK_j = 0; rows of P sum to one, so
    sum_j dV_j = sum_i dO_i (per head)."""
    n, k, H, d = 30, 4, 2, 8
    q, kk, v, do = inputs(n, H, d, 8)
    dq, dk, dv = oracle.prefill_backward(q, kk, v, do, k)
    assert np.allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    assert np.allclose(dv.sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)


def test_blocking_and_key_row_selection_agree():
    """The query-row blocking does not change the result, and the key-row and
    query-row variants return the same dK, dV and dQ rows."""
    n, k, H, d = 50, 6, 2, 8
    q, kk, v, do = inputs(n, H, d, 12)
    a = oracle.prefill_backward(q, kk, v, do, k, block=512)
    b = oracle.prefill_backward(q, kk, v, do, k, block=7)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-12, atol=1e-13)
    rows = np.array([0, 5, 6, 31, 49])
    dk, dv = oracle.prefill_backward_key_rows(q, kk, v, do, k, rows, block=11)
    assert np.allclose(dk, a[1][rows], rtol=1e-12, atol=1e-13)
    assert np.allclose(dv, a[2][rows], rtol=1e-12, atol=1e-13)
    dq = oracle.prefill_backward_query_rows(q, kk, v, do, k, rows)
    assert np.allclose(dq, a[0][rows], rtol=1e-12, atol=1e-13)


def test_lse_definition():
    """exp(lse) is the sum of exp(scaled score) over visible keys (brute force)."""
    n, k, H, d = 10, 3, 2, 4
    q, kk, _, _ = inputs(n, H, d, 5)
    lse = oracle.prefill_lse(q, kk, k)
    for i in range(n):
        for h in range(H):
            tot = sum(math.exp(float(q[i, h] @ kk[j, h]) / math.sqrt(d)) for j in range(n) if j // k <= i // k)
            assert abs(math.exp(lse[i, h]) - tot) <= 1e-12 * tot


@pytest.mark.parametrize("mistake", ["no_scale_dk", "no_rowsum", "dv_transposed_mask", "dq_sign"])
def test_pins_reject_plausible_mistakes(mistake):
    """Each plausible slip in a backward pass fails the autograd pin."""
    n, k, H, d = 12, 3, 2, 8
    q, kk, v, do = inputs(n, H, d, 4)
    dq, dk, dv = oracle.prefill_backward(q, kk, v, do, k)
    if mistake == "no_scale_dk":
        dk = dk * math.sqrt(d)
    elif mistake == "no_rowsum":
        # dS = P * dP (the -D_i term dropped): recompute dQ that way
        s = np.einsum("ihd,jhd->hij", q, kk) / math.sqrt(d)
        s[:, ~frame_mask(n, k)] = -np.inf
        p = np.exp(s - s.max(axis=2, keepdims=True))
        p /= p.sum(axis=2, keepdims=True)
        dp = np.einsum("ihd,jhd->hij", do, v)
        dq = np.einsum("hij,jhd->ihd", p * dp, kk) / math.sqrt(d)
    elif mistake == "dv_transposed_mask":
        s = np.einsum("ihd,jhd->hij", q, kk) / math.sqrt(d)
        s[:, ~frame_mask(n, k).T] = -np.inf
        p = np.exp(s - s.max(axis=2, keepdims=True))
        p /= p.sum(axis=2, keepdims=True)
        dv = np.einsum("hij,ihd->jhd", p, do)
    elif mistake == "dq_sign":
        dq = -dq
    want = autograd_grads(q, kk, v, do, frame_mask(n, k))
    assert not all(np.allclose(g, w, rtol=1e-10, atol=1e-12) for g, w in zip((dq, dk, dv), want))
