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

A row without any visible key has O = 0 and contributes nothing (P = 0).  Pinned in the tests by
central finite differences of the forward oracle.
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


def attention_dense_backward(q, k, v, do, scale: float, causal: bool = False):
    """Dense layout [B,N,H,D]: returns dQ, dK, dV in the layouts of q, k, v (float64)."""
    B, Nq, H, _ = q.shape
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = attention_head_backward(
                q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal)
    return dq, dk, dv


def backward_row_terms(do, o):
    """Drow = sum_d dO * O per row (the term the backward subtracts from dP), float64 [..., rows]."""
    return (np.asarray(do, dtype=np.float64) * np.asarray(o, dtype=np.float64)).sum(axis=-1)
