"""Gradients of exact attention in fp64: the plain derivative of the forward definition.

Test infrastructure only (see the package docstring).

What is differentiated.  The forward definition of attention.py (S = scale*Q*K^T with -inf at masked
positions, P = row softmax of S, O = P*V).  "轻松读懂FlashAttention 上", at the end of section
"Softmax求解重构", gives the reason the forward pass keeps the softmax statistics: with O and the
row statistics stored, S and P can be recomputed for the backward pass instead of being stored; the
Hugging Face page's parameter table (row ``training``) ties training mode to gradient computation.
Neither page prints the gradient formulas, so this module is the derivative itself, for an upstream
gradient dO of L = sum(dO * O):

    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - Drow),   Drow_i = sum_j P_ij dP_ij = sum_d dO_id O_id
    dQ = scale * dS K
    dK = scale * dS^T Q

A row without any visible key has O = 0 and contributes nothing (P = 0).  Every mask of the forward
oracle (none, causal bottom-right aligned, prefix-LM, key length) is accepted.  Pinned in the tests by
central finite differences of the forward oracle; the row-sampled form is pinned against the
whole-head form.
"""
from __future__ import annotations

import numpy as np

from .attention import _visible_mask


def attention_head_backward(q, k, v, do, scale: float, causal: bool = False, prefix: int = 0):
    """dQ [Nq,D], dK [Nk,D], dV [Nk,Dv] of one (batch, head), all float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    vis = _visible_mask(nq, nk, causal, None, prefix)
    s = np.where(vis, scale * (q @ k.T), -np.inf)
    p = np.zeros((nq, nk))
    live = vis.any(axis=1)
    if live.any():
        sl = s[live]
        e = np.exp(sl - sl.max(axis=1, keepdims=True))
        p[live] = e / e.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    drow = (do * o).sum(axis=1)
    ds = p * (dp - drow[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def attention_dense_backward(q, k, v, do, scale: float, causal: bool = False, prefix: int = 0):
    """Dense layout [B,N,H,D]: returns dQ, dK, dV in the layouts of q, k, v (float64)."""
    B, Nq, H, _ = q.shape
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = attention_head_backward(
                q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal, prefix)
    return dq, dk, dv


def attention_varlen_backward(q, k, v, do, cu_seqlens, scale: float, causal: bool = False, prefix: int = 0):
    """Packed varlen self-attention [total,H,D]: dQ, dK, dV per sequence (keys of its own sequence)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        for h in range(q.shape[1]):
            dq[s0:s1, h], dk[s0:s1, h], dv[s0:s1, h] = attention_head_backward(
                q[s0:s1, h], k[s0:s1, h], v[s0:s1, h], do[s0:s1, h], scale, causal, prefix)
    return dq, dk, dv


def attention_rows_backward(q, k, v, do, scale: float, rows, cols, causal: bool = False, prefix: int = 0,
                            chunk: int = 512):
    """dQ at query rows ``rows`` and dK, dV at key rows ``cols`` of one (batch, head), float64.

    For heads too long to differentiate whole: the same derivative as attention_head_backward, with
    the query rows visited ``chunk`` at a time.  Each visited block forms its scores against every
    key, its softmax P (hence its own O and Drow), and adds its share to the sampled dK/dV rows; the
    sampled dQ rows are finished inside the block that holds them.  Returns dQ [len(rows), D],
    dK [len(cols), D], dV [len(cols), Dv].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    dq = np.zeros((len(rows), q.shape[1]))
    dk = np.zeros((len(cols), q.shape[1]))
    dv = np.zeros((len(cols), v.shape[1]))
    for a in range(0, nq, chunk):
        e = min(nq, a + chunk)
        vis = _visible_mask(nq, nk, causal, None, prefix, row_lo=a, row_hi=e)
        s = np.where(vis, scale * (q[a:e] @ k.T), -np.inf)
        p = np.zeros((e - a, nk))
        live = vis.any(axis=1)
        if live.any():
            sl = s[live]
            w = np.exp(sl - sl.max(axis=1, keepdims=True))
            p[live] = w / w.sum(axis=1, keepdims=True)
        o = p @ v
        drow = (do[a:e] * o).sum(axis=1)
        # sampled query rows inside this block
        sel = np.nonzero((rows >= a) & (rows < e))[0]
        if len(sel):
            loc = rows[sel] - a
            ds = p[loc] * (do[rows[sel]] @ v.T - drow[loc, None])
            dq[sel] = scale * (ds @ k)
        # this block's share of the sampled key rows
        pc = p[:, cols]
        dsc = pc * (do[a:e] @ v[cols].T - drow[:, None])
        dk += scale * (dsc.T @ q[a:e])
        dv += pc.T @ do[a:e]
    return dq, dk, dv
