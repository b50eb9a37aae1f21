"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and bench.py.

This module only draws random numbers and rounds them to 16-bit storage.  It holds none of the
attention arithmetic, so the CPU oracle and the CUDA path can both consume its output without
sharing any code with each other.

Recipe (the same on every machine):
  * generator: numpy ``default_rng`` (PCG64), float32 standard normal;
  * seeding: one independent stream per (config seed, tensor id, batch item), tensor ids Q=0, K=1, V=2,
    so that any batch item can be regenerated on its own and host memory stays bounded;
  * rounding: bf16 by round-to-nearest-even on the float32 bit pattern, fp16 by numpy's ``astype``
    (also round-to-nearest-even).  Values are handed out as raw 16-bit patterns (``uint16``), so the
    oracle and the GPU see identical bits;
  * varlen lengths: integers uniform on [lo, hi] inclusive, drawn first from ``default_rng(seed)``.

Tensors use the layout [B, N, H, D] of the tiling sketch on the Ascend FlashAttention page
("FlashAttention核心逻辑", the ``flash_attention_forward`` docstring); varlen tensors are packed as
[total_tokens, H, D] with ``cu_seqlens`` prefix sums.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

Q_ID, K_ID, V_ID = 0, 1, 2

# Synthetic workloads: shapes, dtypes, scales and seeds of the five configurations the method is
# measured on.  ``scale`` defaults to 1/sqrt(D) where the workload does not fix one.
CONFIGS = {
    "tiny": dict(B=2, Nq=512, Nk=512, H=8, D=64, dtype="bf16", scale=1.0 / math.sqrt(64), seed=1),
    "prefill_d64": dict(B=4, Nq=8192, Nk=8192, H=16, D=64, dtype="bf16", scale=1.0 / math.sqrt(64),
                        causal=True, seed=2),
    "prefill_d128": dict(B=8, Nq=4096, Nk=4096, H=32, D=128, dtype="bf16",
                         scale=1.0 / math.sqrt(128), causal=True, seed=3),
    "varlen": dict(nseq=64, len_lo=128, len_hi=2048, H=16, D=64, dtype="fp16", scale=0.1,
                   causal=False, seed=4),
    "decode": dict(B=64, Nk=8192, H=32, D=128, dtype="bf16", scale=1.0 / math.sqrt(128),
                   num_splits=16, seed=5),
    # grouped KV heads (4 query heads per KV head) and per-sequence cache lengths U{1024..8192}
    "decode_gqa": dict(B=64, Nk=8192, H=32, Hkv=8, D=128, dtype="bf16", scale=1.0 / math.sqrt(128),
                       num_splits=16, seed=6, len_lo=1024, len_hi=8192),
    # long-context decode, cut along the key axis over the ranks: the "decode" cache read as 4
    # sequences of 131072 keys (sequence b is batch items 16b .. 16b+15 of "decode" laid end to end,
    # the same bytes), with its own queries; splits are per key shard
    "decode_long": dict(B=4, Nk=131072, H=32, D=128, dtype="bf16", scale=1.0 / math.sqrt(128),
                        num_splits=64, seed=7, cache_of="decode"),
    # the grouped decode workload with its cache in a paged pool: pages of 16 rows at positions of
    # a seeded permutation of the pool, one block-table row per sequence
    "decode_paged": dict(page_size=16, seed=8, cache_of="decode_gqa"),
}


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(16, os.cpu_count() or 1))


def round_to_bits(x: np.ndarray, dtype: str, out: np.ndarray | None = None) -> np.ndarray:
    """Round float32 values to bf16 or fp16 and return the 16-bit patterns as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if out is None:
        out = np.empty(x.shape, dtype=np.uint16)
    if dtype == "bf16":
        b = x.view(np.uint32)
        bias = (b >> np.uint32(16)) & np.uint32(1)
        bias += np.uint32(0x7FFF)
        bias += b
        bias >>= np.uint32(16)
        out[...] = bias
    elif dtype == "fp16":
        out[...] = x.astype(np.float16).view(np.uint16)
    else:
        raise ValueError(f"unsupported storage dtype {dtype!r}")
    return out


def bits_to_float(bits: np.ndarray, dtype: str, as_type=np.float64) -> np.ndarray:
    """Exact widening of 16-bit patterns to float32/float64 values."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        f = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    elif dtype == "fp16":
        f = bits.view(np.float16)
    else:
        raise ValueError(f"unsupported storage dtype {dtype!r}")
    return f.astype(as_type)


def normal_bits(seed, n: int, dtype: str, std: float = 1.0) -> np.ndarray:
    """``n`` standard-normal draws (times ``std``) from ``default_rng(seed)``, rounded to 16 bits."""
    rng = np.random.default_rng(seed)
    x = np.empty(n, dtype=np.float32)
    rng.standard_normal(out=x, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return round_to_bits(x, dtype)


def batch_item(seed: int, tensor_id: int, b: int, shape, dtype: str, std: float = 1.0) -> np.ndarray:
    """One batch item (or one varlen sequence) of a tensor, as uint16 bits of the given shape."""
    n = int(np.prod(shape))
    return normal_bits([seed, tensor_id, b], n, dtype, std).reshape(shape)


def batched(seed: int, tensor_id: int, B: int, shape, dtype: str, std: float = 1.0,
            out: np.ndarray | None = None) -> np.ndarray:
    """A [B, *shape] uint16 tensor, one independent stream per batch item (threaded)."""
    shape = tuple(shape)
    if out is None:
        out = np.empty((B,) + shape, dtype=np.uint16)

    def fill(b):
        out[b] = batch_item(seed, tensor_id, b, shape, dtype, std)

    if B == 1 or out.nbytes < (8 << 20):
        for b in range(B):
            fill(b)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(B)))
    return out


def dense_qkv(seed: int, B: int, Nq: int, Nk: int, H: int, D: int, dtype: str, std: float = 1.0):
    """Q [B,Nq,H,D], K and V [B,Nk,H,D] as uint16 bits."""
    q = batched(seed, Q_ID, B, (Nq, H, D), dtype, std)
    k = batched(seed, K_ID, B, (Nk, H, D), dtype, std)
    v = batched(seed, V_ID, B, (Nk, H, D), dtype, std)
    return q, k, v


def varlen_lengths(seed: int, nseq: int, lo: int, hi: int) -> np.ndarray:
    """Sequence lengths uniform on [lo, hi] inclusive, the first draws of ``default_rng(seed)``."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=nseq).astype(np.int64)


def cu_seqlens_of(lengths) -> np.ndarray:
    """int32 prefix sums [0, l0, l0+l1, ...] of length nseq+1."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu.astype(np.int32)


def varlen_qkv(seed: int, lengths, H: int, D: int, dtype: str, std: float = 1.0):
    """Packed Q, K, V [total, H, D] (uint16 bits) and cu_seqlens (int32)."""
    lengths = [int(x) for x in lengths]
    cu = cu_seqlens_of(lengths)
    total = int(cu[-1])
    outs = []
    for tid in (Q_ID, K_ID, V_ID):
        t = np.empty((total, H, D), dtype=np.uint16)

        def fill(b, t=t, tid=tid):
            t[cu[b]:cu[b + 1]] = batch_item(seed, tid, b, (lengths[b], H, D), dtype, std)

        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(len(lengths))))
        outs.append(t)
    return outs[0], outs[1], outs[2], cu


def decode_inputs(seed: int, B: int, Nk: int, H: int, D: int, dtype: str, std: float = 1.0):
    """Single-query Q [B,1,H,D] and a K/V cache [B,Nk,H,D], uint16 bits."""
    return dense_qkv(seed, B, 1, Nk, H, D, dtype, std)


def decode_gqa_inputs(seed: int, B: int, Nk: int, Hq: int, Hkv: int, D: int, dtype: str, std: float = 1.0):
    """Single-query Q [B,1,Hq,D] and a K/V cache [B,Nk,Hkv,D], uint16 bits."""
    q = batched(seed, Q_ID, B, (1, Hq, D), dtype, std)
    k = batched(seed, K_ID, B, (Nk, Hkv, D), dtype, std)
    v = batched(seed, V_ID, B, (Nk, Hkv, D), dtype, std)
    return q, k, v


def key_ramp(q: np.ndarray, k: np.ndarray, dtype: str, q_value: float, top: float, key_axis: int,
             cu_seqlens=None):
    """Copies of Q and K (uint16 bits) with channel 0 replaced to give scores that rise along the keys.

    Channel 0 of every query becomes ``q_value`` and channel 0 of key j becomes ``top * j / (n - 1)``,
    j counted along ``key_axis`` of K (from the start of each packed sequence when ``cu_seqlens`` is
    given, the key axis being axis 0 then).  Only the inputs' structure changes: the last channel
    index is the head dimension, all other channels keep their random values.
    """
    q2, k2 = q.copy(), k.copy()
    q2[..., 0] = round_to_bits(np.full(q2.shape[:-1], q_value, dtype=np.float32), dtype)
    kc = np.moveaxis(k2[..., 0], key_axis, 0)  # view: keys first
    if cu_seqlens is None:
        spans = [(0, kc.shape[0])]
    else:
        spans = [(int(a), int(b)) for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:])]
    for a, b in spans:
        n = b - a
        if n <= 0:
            continue
        ramp = (np.arange(n, dtype=np.float32) * np.float32(top / max(n - 1, 1))).astype(np.float32)
        vals = np.broadcast_to(ramp.reshape((n,) + (1,) * (kc.ndim - 1)), (n,) + kc.shape[1:])
        kc[a:b] = round_to_bits(np.ascontiguousarray(vals), dtype)
    return q2, k2


def config_inputs(name: str, **overrides):
    """Inputs of one named workload (optionally with smaller sizes for the oracle)."""
    c = dict(CONFIGS[name])
    c.update(overrides)
    if name == "varlen":
        lengths = c.get("lengths")
        if lengths is None:
            lengths = varlen_lengths(c["seed"], c["nseq"], c["len_lo"], c["len_hi"])
        q, k, v, cu = varlen_qkv(c["seed"], lengths, c["H"], c["D"], c["dtype"])
        return dict(cfg=c, q=q, k=k, v=v, cu_seqlens=cu, lengths=np.asarray(lengths))
    if name == "decode":
        q, k, v = decode_inputs(c["seed"], c["B"], c["Nk"], c["H"], c["D"], c["dtype"])
        return dict(cfg=c, q=q, k=k, v=v)
    q, k, v = dense_qkv(c["seed"], c["B"], c["Nq"], c["Nk"], c["H"], c["D"], c["dtype"])
    return dict(cfg=c, q=q, k=k, v=v)
