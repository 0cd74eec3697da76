"""Gradients of the block-causal attention, in fp64 (test infrastructure; see
the package doc).

The function differentiated is the attention of "DiT as Real-Time
Rerenderer" (papernotes note, Method > Key Designs 2) over one whole sequence,
the form training sees (Method > Key Designs 3: the student is trained with
Self Forcing and DMD, i.e. by gradient descent through this attention):

    O = softmax(S) V,   S = scale * Q K^T + M,
    M_ij = 0 if floor(j/k) <= floor(i/k) else -inf.

For an upstream gradient dO (= dL/dO) the chain rule gives, row by row with
P = softmax(S):

    dV = P^T dO
    dP = dO V^T
    dS_ij = P_ij * (dP_ij - sum_t P_it dP_it)      (softmax Jacobian)
    dQ = scale * dS K
    dK = scale * dS^T Q

Masked entries have P_ij = 0, so they carry no gradient.  The pages print no
backward; this is the plain derivative of their equation.  Everything runs in
float64 with numpy, per head, in blocks of query rows; nothing is fused or
reordered beyond summing the key-side gradients block by block.
"""
import math

import numpy as np


def _frame_mask(rows, n_keys, k_per_frame):
    """visible[r, j]: query row rows[r] sees key j (frame of j <= frame of row)."""
    kf = np.arange(n_keys, dtype=np.int64) // k_per_frame
    qf = np.asarray(rows, dtype=np.int64) // k_per_frame
    return kf[None, :] <= qf[:, None]


def _scores(qh, kh, rows, k_per_frame, scale):
    """Masked scaled scores S[rows, :] of one head (-inf where hidden)."""
    s = scale * (qh[rows] @ kh.T)
    s[~_frame_mask(rows, kh.shape[0], k_per_frame)] = -np.inf
    return s


def prefill_lse(q, k, k_per_frame, rows=None, scale=None):
    """Natural-log log-sum-exp of each row's visible scaled scores:
    lse[r, h] = log sum_{j visible} exp(scale * q_r . k_j).  Returns
    [len(rows), H] float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    n, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rows = np.arange(n, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    out = np.empty((rows.size, H))
    for h in range(H):
        s = _scores(q[:, h], k[:, h], rows, k_per_frame, scale)
        m = s.max(axis=1)
        out[:, h] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return out


def prefill_backward(q, k, v, do, k_per_frame, scale=None, block=512):
    """(dQ, dK, dV) of L = sum(dO * O) for the block-causal attention over one
    sequence; q, k, v, do: [n, H, d].  Returns three [n, H, d] float64."""
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    n, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = np.empty((n, H, d))
    dk = np.zeros((n, H, d))
    dv = np.zeros((n, H, d))
    for h in range(H):
        qh, kh, vh, doh = q[:, h], k[:, h], v[:, h], do[:, h]
        for r0 in range(0, n, block):
            rows = np.arange(r0, min(n, r0 + block))
            s = _scores(qh, kh, rows, k_per_frame, scale)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dp = doh[rows] @ vh.T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[rows, h] = scale * (ds @ kh)
            dk[:, h] += scale * (ds.T @ qh[rows])
            dv[:, h] += p.T @ doh[rows]
    return dq, dk, dv


def prefill_backward_key_rows(q, k, v, do, k_per_frame, key_rows, scale=None, block=2048):
    """dK and dV of selected key rows only (every query row still enters):
    the same formulas, with the gradient of each selected key summed over all
    query blocks.  Returns two [len(key_rows), H, d] float64."""
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    n, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    key_rows = np.asarray(key_rows, np.int64)
    dk = np.zeros((key_rows.size, H, d))
    dv = np.zeros((key_rows.size, H, d))
    for h in range(H):
        qh, kh, vh, doh = q[:, h], k[:, h], v[:, h], do[:, h]
        for r0 in range(0, n, block):
            rows = np.arange(r0, min(n, r0 + block))
            s = _scores(qh, kh, rows, k_per_frame, scale)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            dp = doh[rows] @ vh.T
            dsum = (p * dp).sum(axis=1, keepdims=True)
            ps, dps = p[:, key_rows], dp[:, key_rows]
            ds = ps * (dps - dsum)
            dk[:, h] += scale * (ds.T @ qh[rows])
            dv[:, h] += ps.T @ doh[rows]
    return dk, dv


def prefill_backward_query_rows(q, k, v, do, k_per_frame, rows, scale=None):
    """dQ of selected query rows only: each row's dQ needs only its own row of
    P and dP.  Returns [len(rows), H, d] float64."""
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    n, H, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rows = np.asarray(rows, np.int64)
    dq = np.empty((rows.size, H, d))
    for h in range(H):
        qh, kh, vh, doh = q[:, h], k[:, h], v[:, h], do[:, h]
        s = _scores(qh, kh, rows, k_per_frame, scale)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        dp = doh[rows] @ vh.T
        ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
        dq[:, h] = scale * (ds @ kh)
    return dq
