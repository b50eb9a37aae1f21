"""Materialised fp64 attention: the plain definition the tiled method must reproduce exactly.

Test infrastructure only (see the package docstring).

Definition followed.  The Ascend CANN ops-transformer FlashAttention article (zskr.cn), section
"背景" (background), splits standard attention into three steps: the score matrix S = Q*K^T, a row
softmax of S, and the product of that softmax with V.  The CSDN article "轻松读懂FlashAttention 上",
section "内存卡点", names the same two N x N intermediates S and P.  "Was FlashAttention bei
Transformer-Inference verändert" states that the tiled method computes this exact result, not an
approximation.  The scale factor defaults to 1/sqrt(head_dim) ("如何为 Hugging Face Transformers
更多架构添加 Flash Attention 2 支持？", parameter table, row ``softmax_scale``); the causal mask keeps
the lower triangle (same table, row ``is_causal``); a 2-D key-padding mask marks valid keys per
batch item (same page, "常见错误排查", error 4).

Readings where the pages are silent:
  * causal with Nq != Nk is bottom-right aligned: query i sees key j iff j <= i + (Nk - Nq);
  * the prefix mask, which the same page names among the mask formats of other architectures
    ("原因分析", item 1) without defining it, is the prefix-LM mask: causal, except that the first
    ``prefix`` keys are visible to every query (query i sees key j iff j < prefix or
    j <= i + (Nk - Nq)); prefix = 0 is the causal mask;
  * a row with no visible key gets O = 0 and LSE = -inf;
  * LSE is the natural log-sum-exp of the scaled, masked scores of a row.

Everything is float64.  Inputs are the already-rounded 16-bit values widened exactly to float64.
S and P are formed for one (batch, head) at a time only.
"""
from __future__ import annotations

import numpy as np


def _visible_mask(nq: int, nk: int, causal: bool, k_valid: int | None, prefix: int = 0,
                  row_lo: int = 0, row_hi: int | None = None) -> np.ndarray:
    """Boolean [rows, nk]: True where query i (rows row_lo..row_hi-1, default all) may attend to key j."""
    row_hi = nq if row_hi is None else row_hi
    j = np.arange(nk)[None, :]
    vis = np.ones((row_hi - row_lo, nk), dtype=bool)
    if k_valid is not None:
        vis &= j < k_valid
    if causal:
        i = np.arange(row_lo, row_hi)[:, None]
        vis &= (j <= i + (nk - nq)) | (j < prefix)
    return vis


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, causal: bool = False,
                   k_valid: int | None = None, prefix: int = 0):
    """O [Nq, Dv] and LSE [Nq] for one (batch, head).

    q: [Nq, D], k: [Nk, D], v: [Nk, Dv], all float64.  ``k_valid`` (optional) masks keys j >= k_valid
    (key padding); ``prefix`` (causal only) makes the first ``prefix`` keys visible to every query.
    Step 1: S = scale * Q K^T.  Masked entries become -inf.  Step 2: row softmax with the row max m
    subtracted (safe softmax), P = exp(S - m), l = sum_j P.  Step 3: O = P V / l.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nk = q.shape[0], k.shape[0]
    s = scale * (q @ k.T)
    vis = _visible_mask(nq, nk, causal, k_valid, prefix)
    s = np.where(vis, s, -np.inf)
    o = np.zeros((nq, v.shape[1]), dtype=np.float64)
    lse = np.full(nq, -np.inf, dtype=np.float64)
    live = vis.any(axis=1)
    if live.any():
        sl = s[live]
        m = sl.max(axis=1)
        p = np.exp(sl - m[:, None])
        l = p.sum(axis=1)
        o[live] = (p @ v) / l[:, None]
        lse[live] = m + np.log(l)
    return o, lse


def attention_dense(q, k, v, scale: float, causal: bool = False, prefix: int = 0):
    """Dense layout: q [B,Nq,H,D], k/v [B,Nk,H,D] float64 -> O [B,Nq,H,Dv], LSE [B,H,Nq]."""
    B, Nq, H, _ = q.shape
    Dv = v.shape[3]
    o = np.zeros((B, Nq, H, Dv), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            o[b, :, h, :], lse[b, h, :] = attention_head(q[b, :, h, :], k[b, :, h, :], v[b, :, h, :],
                                                         scale, causal, prefix=prefix)
    return o, lse


def attention_varlen(q, k, v, cu_seqlens, scale: float, causal: bool = False, prefix: int = 0):
    """Packed varlen self-attention: q/k/v [total,H,D]; sequence b owns rows cu[b]:cu[b+1].

    Each query of sequence b attends to exactly the keys of sequence b (the packed form of the 2-D
    key-padding mask); with ``causal`` the prefix (same length for every sequence) is counted from the
    sequence's first key.  Returns O [total,H,Dv] and LSE [H,total].
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    total, H, _ = q.shape
    o = np.zeros((total, H, v.shape[2]), dtype=np.float64)
    lse = np.zeros((H, total), dtype=np.float64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        for h in range(H):
            o[s0:s1, h, :], lse[h, s0:s1] = attention_head(q[s0:s1, h, :], k[s0:s1, h, :],
                                                           v[s0:s1, h, :], scale, causal, prefix=prefix)
    return o, lse


def padded_key_mask_attention(q, k, v, key_mask, scale: float):
    """Padded form: q/k/v [B,Nmax,H,D] with a 2-D key mask [B,Nmax] (True = real token).

    The 2-D mask is read as the (batch, 1, 1, seq_len) broadcast of "常见错误排查", error 4: it hides
    padded keys from every query row.  Returns O [B,Nmax,H,Dv] and LSE [B,H,Nmax].
    """
    B, N, H, _ = q.shape
    o = np.zeros((B, N, H, v.shape[3]), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        kv = np.asarray(key_mask[b], dtype=bool)
        for h in range(H):
            s = scale * (q[b, :, h, :] @ k[b, :, h, :].T)
            s = np.where(kv[None, :], s, -np.inf)
            m = s.max(axis=1)
            ok = np.isfinite(m)
            p = np.zeros_like(s)
            p[ok] = np.exp(s[ok] - m[ok, None])
            l = p.sum(axis=1)
            res = np.zeros((N, v.shape[3]))
            res[ok] = (p[ok] @ v[b, :, h, :]) / l[ok, None]
            o[b, :, h, :] = res
            lse[b, h, :] = np.where(ok, m + np.log(np.where(ok, l, 1.0)), -np.inf)
    return o, lse


def attention_rows(q_head, k_head, v_head, rows, scale: float, causal: bool = False,
                   k_valid: int | None = None, prefix: int = 0):
    """O and LSE of selected query rows of one (batch, head), each row evaluated on its own.

    q_head [Nq,D]; ``rows`` are query indices.  Used to check full-size runs on sampled outputs.
    """
    q_head = np.asarray(q_head, dtype=np.float64)
    k_head = np.asarray(k_head, dtype=np.float64)
    v_head = np.asarray(v_head, dtype=np.float64)
    nq, nk = q_head.shape[0], k_head.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((len(rows), v_head.shape[1]))
    lse = np.full(len(rows), -np.inf)
    for r, i in enumerate(rows):
        last = nk if k_valid is None else k_valid
        if causal:  # visible keys form the prefix [0, last) of the row
            last = min(last, max(prefix, int(i) + (nk - nq) + 1))
        if last <= 0:
            continue
        s = scale * (k_head[:last] @ q_head[i])
        m = s.max()
        p = np.exp(s - m)
        l = p.sum()
        o[r] = (p @ v_head[:last]) / l
        lse[r] = m + np.log(l)
    return o, lse


def attention_decode(q, k_cache, v_cache, scale: float):
    """Single-token decode: q [B,1,H,D], cache [B,Nk,H,D] -> O [B,1,H,Dv], LSE [B,H,1].

    The one query attends to every cached key ("Was FlashAttention bei Transformer-Inference
    verändert": prefill versus single-token decode differ only in the available parallelism).
    """
    return attention_dense(q, k_cache, v_cache, scale, causal=False)


def attention_decode_gqa(q, k_cache, v_cache, scale: float, seqlens_k=None):
    """Single-token decode with grouped KV heads and per-sequence cache lengths.

    q [B,1,Hq,D]; k_cache/v_cache [B,Nk,Hkv,D] with Hq a multiple of Hkv; query head h reads KV head
    h // (Hq // Hkv).  ``seqlens_k`` (optional, length B) gives the valid cache length of each batch
    item: its query sees keys [0, seqlens_k[b]) (all Nk when omitted); a zero length gives O = 0 and
    LSE = -inf.  Returns O [B,1,Hq,Dv] and LSE [B,Hq].

    Reading: "Was FlashAttention bei Transformer-Inference verändert" asks whether a backend supports
    the head dim, mask and cache layout and separates prefill from single-token decode, without
    fixing a layout; grouped KV heads and per-sequence lengths are the plainest cache layout with
    those two properties.
    """
    B, _, Hq, _ = q.shape
    Nk, Hkv = k_cache.shape[1], k_cache.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    o = np.zeros((B, 1, Hq, v_cache.shape[3]), dtype=np.float64)
    lse = np.full((B, Hq), -np.inf, dtype=np.float64)
    for b in range(B):
        L = Nk if seqlens_k is None else int(seqlens_k[b])
        if L <= 0:
            continue
        for h in range(Hq):
            ob, lb = attention_head(q[b, :, h, :], k_cache[b, :L, h // G, :], v_cache[b, :L, h // G, :], scale)
            o[b, :, h, :], lse[b, h] = ob, lb[0]
    return o, lse



def attention_decode_shard(q, k_shard, v_shard, scale: float, key_offset: int, seqlens_k=None):
    """Decode over one key shard of a longer cache: O [B,1,Hq,Dv] and LSE [B,Hq] of the shard alone.

    k_shard/v_shard [B,Nk_shard,Hkv,D] hold keys [key_offset, key_offset + Nk_shard) of the whole
    cache; ``seqlens_k`` (optional) counts valid keys of the whole cache, so the shard sees its keys
    below seqlens_k[b].  The result is the definition restricted to those keys (O = 0, LSE = -inf
    where there are none): the softmax statistics of one key group in the sense of
    "轻松读懂FlashAttention 上", section "Softmax求解重构", which merge into the whole cache's
    result.
    """
    nk = k_shard.shape[1]
    lens = None
    if seqlens_k is not None:
        lens = [min(max(int(L) - key_offset, 0), nk) for L in seqlens_k]
    return attention_decode_gqa(q, k_shard, v_shard, scale, lens)


def attention_decode_paged(q, k_pages, v_pages, block_table, scale: float, seqlens_k):
    """Single-token decode over a paged cache: O [B,1,Hq,Dv] and LSE [B,Hq].

    k_pages/v_pages [P, page_size, Hkv, D] are pools of fixed-size pages of cache rows (row r of page
    p is one key).  ``block_table`` [B, pages_per_seq] lists, for each batch item, the pool pages that
    hold its keys in order: entry i holds keys [i * page_size, (i + 1) * page_size).  Batch item b
    sees its first seqlens_k[b] keys, so only its first ceil(seqlens_k[b] / page_size) entries are
    read; the rest of the row (and any page no entry names) is never looked at.  The query then
    attends to the keys gathered in that order exactly as over a contiguous cache with grouped KV
    heads (query head h reads KV head h // (Hq // Hkv)).

    Reading: "Was FlashAttention bei Transformer-Inference verändert" lists the cache layout among
    the properties a backend must support without fixing one; a pool of fixed-size pages addressed
    through a per-sequence table is the plainest layout beside the contiguous one, and it changes
    only where each key row is read from, not what is computed.
    """
    B = q.shape[0]
    ps = k_pages.shape[1]
    seqlens_k = [int(L) for L in seqlens_k]
    lmax = max(seqlens_k + [1])
    cap = -(-lmax // ps) * ps
    k_g = np.zeros((B, cap) + k_pages.shape[2:], dtype=np.float64)
    v_g = np.zeros((B, cap) + v_pages.shape[2:], dtype=np.float64)
    for b, L in enumerate(seqlens_k):
        for i in range(-(-L // ps)):
            page = int(block_table[b][i])
            k_g[b, i * ps:(i + 1) * ps] = k_pages[page]
            v_g[b, i * ps:(i + 1) * ps] = v_pages[page]
    return attention_decode_gqa(q, k_g, v_g, scale, seqlens_k)
