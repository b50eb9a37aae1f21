"""Tiled online-softmax attention and the merge of per-group softmax statistics, in fp64.

Test infrastructure only (see the package docstring).

1. ``tiled_online_attention`` follows the loop structure of the Ascend CANN ops-transformer
   FlashAttention article (zskr.cn), section "原理" steps 1-4 and its "代码讲解" walkthrough: the
   outer loop walks query blocks, the inner loop walks key/value blocks; each step forms the block
   scores scale*Q_i*K_j^T, masks them, and updates a running row max m, a running row sum l and an
   output accumulator that is rescaled by exp(m_old - m_new); the block output is divided by l at
   the end.  The walkthrough's code has defects that this restatement does not carry over (its
   causal mask ignores the block offsets, its matmul on [B,bs,H,D] tensors contracts over the wrong
   axes, and a row whose first block is fully masked would produce NaN); here the mask is the global
   one (key j visible to query i iff j <= i + Nk - Nq), the contraction is per (batch, head), and a
   running max of -inf leaves the state untouched.

2. ``group_stats`` / ``merge_groups`` / ``softmax_by_groups`` restate the section "Softmax求解重构"
   of the CSDN article "轻松读懂FlashAttention 上": a row x is cut into groups x(1), x(2), x(3);
   each group keeps m(x) (its max, a scalar), f(x) = exp(x - m(x)) (a vector) and l(x) = sum f(x);
   two groups merge as m = max(m1, m2), f = [e^(m1-m) f1, e^(m2-m) f2], l = e^(m1-m) l1 + e^(m2-m) l2,
   and softmax(x) = f(x) / l(x).  The article's formulas were lost in extraction; this is the
   standard reading of the surviving prose (groups merged two at a time, left to right).

3. ``split_kv_partials`` / ``combine_partials`` apply the same merge to single-query decode whose
   keys are cut into splits: each split yields a normalised partial output o_s and lse_s; a split's
   state is equivalent to (m = lse_s, l = 1, acc = o_s), and merging all of them gives the output.
"""
from __future__ import annotations

import math

import numpy as np


def tiled_online_attention(q, k, v, scale: float, causal: bool = False, block_q: int = 128,
                           block_k: int = 128, k_valid: int | None = None):
    """Blockwise online-softmax attention for one (batch, head): returns O [Nq,Dv], LSE [Nq]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    kv_len = nk if k_valid is None else k_valid
    out = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for i0 in range(0, nq, block_q):
        qi = q[i0:i0 + block_q]
        rows = np.arange(i0, i0 + qi.shape[0])
        acc = np.zeros((qi.shape[0], v.shape[1]))
        m = np.full(qi.shape[0], -np.inf)
        l = np.zeros(qi.shape[0])
        for j0 in range(0, nk, block_k):
            kj = k[j0:j0 + block_k]
            vj = v[j0:j0 + block_k]
            cols = np.arange(j0, j0 + kj.shape[0])
            s = scale * (qi @ kj.T)
            vis = np.broadcast_to(cols[None, :] < kv_len, s.shape)
            if causal:
                vis = vis & (cols[None, :] <= rows[:, None] + (nk - nq))
            s = np.where(vis, s, -np.inf)
            # statistics of this block (the "new" group) ...
            m_blk = s.max(axis=1)
            # ... merged into the running statistics
            m_new = np.maximum(m, m_blk)
            live = np.isfinite(m_new)
            ref = np.where(live, m_new, 0.0)
            alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
            p = np.exp(s - ref[:, None])  # exp(-inf) = 0 for masked entries
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ vj
            m = m_new
        ok = l > 0
        out[i0:i0 + qi.shape[0]][ok] = acc[ok] / l[ok, None]
        lse[i0:i0 + qi.shape[0]] = np.where(ok, m + np.log(np.where(ok, l, 1.0)), -np.inf)
    return out, lse


def group_stats(x):
    """(m(x), f(x), l(x)) of one group of a row."""
    x = np.asarray(x, dtype=np.float64)
    m = float(np.max(x))
    f = np.exp(x - m)
    return m, f, float(np.sum(f))


def merge_groups(a, b):
    """Merge the statistics of two adjacent groups (a left of b)."""
    m1, f1, l1 = a
    m2, f2, l2 = b
    m = max(m1, m2)
    e1, e2 = math.exp(m1 - m), math.exp(m2 - m)
    return m, np.concatenate([e1 * f1, e2 * f2]), e1 * l1 + e2 * l2


def softmax_by_groups(x, n_groups: int = 3):
    """softmax(x) computed by cutting x into ``n_groups`` groups and merging them in order."""
    parts = np.array_split(np.asarray(x, dtype=np.float64), n_groups)
    state = group_stats(parts[0])
    for p in parts[1:]:
        state = merge_groups(state, group_stats(p))
    m, f, l = state
    return f / l, m, l


def split_bounds(nk: int, num_splits: int):
    """Key range [lo, hi) of each split: splits of ceil(nk / num_splits) keys, the last ones may be
    shorter or empty."""
    per = -(-nk // num_splits)
    return [(min(nk, s * per), min(nk, (s + 1) * per)) for s in range(num_splits)]


def split_kv_partials(q_vec, k, v, scale: float, num_splits: int):
    """Per-split normalised partial outputs o_s [S,Dv] and lse_s [S] for one query vector."""
    q_vec = np.asarray(q_vec, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    o = np.zeros((num_splits, v.shape[1]))
    lse = np.full(num_splits, -np.inf)
    for s, (lo, hi) in enumerate(split_bounds(k.shape[0], num_splits)):
        if hi <= lo:
            continue
        sc = scale * (k[lo:hi] @ q_vec)
        m, f, l = group_stats(sc)
        o[s] = (f @ v[lo:hi]) / l
        lse[s] = m + math.log(l)
    return o, lse


def combine_partials(o_parts, lse_parts):
    """Merge split partials into the output and LSE of the whole key range.

    A split with normalised output o_s and log-sum-exp lse_s carries the state (m = lse_s, l = 1,
    acc = o_s); states merge as in ``merge_groups`` with acc playing the role of f @ V.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m, l, acc = -np.inf, 0.0, np.zeros(o_parts.shape[1])
    for o_s, lse_s in zip(o_parts, lse_parts):
        if not np.isfinite(lse_s):
            continue
        m_new = max(m, lse_s)
        e_old = math.exp(m - m_new) if np.isfinite(m) else 0.0
        e_s = math.exp(lse_s - m_new)
        acc = e_old * acc + e_s * o_s
        l = e_old * l + e_s
        m = m_new
    if l == 0.0:
        return np.zeros(o_parts.shape[1]), -np.inf
    return acc / l, m + math.log(l)
