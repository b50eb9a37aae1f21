"""Scalar pure-Python attention for tiny inputs (no numpy in the arithmetic).

Test infrastructure only (see the package docstring).  Every score, exponential and sum is formed
one element at a time with ``math.fsum`` (exactly rounded sums), so this evaluation shares no code
path with the numpy oracle.  It follows the same three-step definition (scores, safe row softmax,
weighted sum of values) of the Ascend CANN ops-transformer FlashAttention article, section "背景",
with the safe-softmax max subtraction of "轻松读懂FlashAttention 上" (the "小知识" note under
"内存卡点").  Meant for N <= 16.
"""
from __future__ import annotations

import math


def brute_attention_head(q, k, v, scale: float, causal: bool = False, k_valid=None, prefix: int = 0):
    """q: [Nq][D], k: [Nk][D], v: [Nk][Dv] nested sequences of floats -> (O rows, LSE list).

    With ``causal`` a key is visible when it is at or before the query's diagonal position or among
    the first ``prefix`` keys (prefix-LM mask; prefix = 0 is plain causal).
    """
    q = [[float(x) for x in row] for row in q]
    k = [[float(x) for x in row] for row in k]
    v = [[float(x) for x in row] for row in v]
    nq, nk, dv = len(q), len(k), len(v[0])
    kv_len = nk if k_valid is None else k_valid
    out, lse = [], []
    for i in range(nq):
        visible = [j for j in range(nk)
                   if j < kv_len and (not causal or j <= i + (nk - nq) or j < prefix)]
        if not visible:
            out.append([0.0] * dv)
            lse.append(-math.inf)
            continue
        scores = {j: scale * math.fsum(a * b for a, b in zip(q[i], k[j])) for j in visible}
        m = max(scores.values())
        w = {j: math.exp(scores[j] - m) for j in visible}
        l = math.fsum(w.values())
        out.append([math.fsum(w[j] * v[j][d] for j in visible) / l for d in range(dv)])
        lse.append(m + math.log(l))
    return out, lse
