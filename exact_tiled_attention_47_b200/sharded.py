"""Key-sharded single-token decode: a KV cache cut along the key axis, one shard per rank.

"轻松读懂FlashAttention 上", section "内存卡点", notes that contexts reach 64k to 128k tokens and more;
such a cache can be spread over the GPUs of a node along its key axis.  Each rank then runs the
split-KV decode kernels on its own shard (``fa_decode_splitkv_shard``), which leave the shard's fp32
(O, LSE) -- the softmax statistics of one key group -- and the ranks exchange these small results
with one all-gather.  Each rank finally merges all shards' results (``fa_decode_merge``) by the
group-statistics merge of the same page's section "Softmax求解重构", so every rank holds the exact
output over the whole cache.

Bytes crossing the interconnect per step: world * B * H * (D + 1) * 4 (about 1 MiB per rank for
B = 64, H = 32, D = 128), against B * Nk * Hkv * D * 4 bytes of K and V read from HBM: the exchange
is a small fraction of the step, so it is a plain NCCL all-gather between two kernels.

Host logic only (shard ranges, the exchange, buffer sizes); all arithmetic runs in the library.
"""
from __future__ import annotations

import math


def shard_range(Nk_total: int, world: int, rank: int):
    """(key_offset, Nk_shard) of rank ``rank``: contiguous ranges of floor or ceil(Nk_total / world)
    keys in rank order, the longer ones first, covering [0, Nk_total) exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside [0, world)")
    if Nk_total < world:
        raise ValueError("every rank needs at least one key")
    base, extra = divmod(Nk_total, world)
    offset = rank * base + min(rank, extra)
    return offset, base + (1 if rank < extra else 0)


def part_floats(B: int, H: int, D: int) -> int:
    """fp32 words of one shard's packed result: O [B,H,D], LSE [B,H], padded to 16 bytes (the
    layout and size ``fa_decode_part_bytes`` defines)."""
    n = B * H * (D + 1)
    return (n + 3) // 4 * 4


def gather_parts(part, world: int, group=None):
    """All ranks' packed shard results laid end to end in rank order: [world * len(part)] fp32.

    With world == 1 the local buffer is returned as it is.  Works with any torch.distributed backend
    (NCCL on the GPUs, gloo on CPU tensors).
    """
    if world == 1:
        return part
    import torch
    import torch.distributed as dist
    out = torch.empty(world * part.numel(), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, part, group=group)
    return out


def _stream_handle(s):
    return s if isinstance(s, int) else s.cuda_stream


def decode_sharded(q, k_shard, v_shard, key_offset: int, Nk_total: int, scale=None, num_splits: int = 16,
                   seqlens_k=None, out_dtype=None, group=None, workspace=None, stream=None):
    """O [B,1,Hq,D], LSE [B,Hq] of single-token decode over a cache whose keys [key_offset,
    key_offset + Nk_shard) this rank holds in k_shard / v_shard [B, Nk_shard, Hkv, D].

    Every rank of ``group`` (default: the world, or a single process without torch.distributed)
    calls this with its own shard; ``seqlens_k`` (int32 [B] on the device, optional) counts keys of
    the whole cache.  All ranks return the same result.
    """
    import torch
    from . import FAError, FA_OK, fa_decode_merge, fa_decode_part_bytes, fa_decode_splitkv_shard, \
        fa_decode_workspace_bytes
    world = 1
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            world = dist.get_world_size(group)
    except ImportError:
        pass
    if world > 1 and stream is not None and _stream_handle(stream) != torch.cuda.current_stream().cuda_stream:
        raise ValueError("the exchange runs on the current stream: call with stream=None")
    B, _, Hq, D = q.shape
    Nk_shard, Hkv = k_shard.shape[1], k_shard.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if workspace is None:
        workspace = torch.empty(fa_decode_workspace_bytes(B, Hq, D, num_splits), dtype=torch.uint8,
                                device=q.device)
    nf = fa_decode_part_bytes(B, Hq, D) // 4
    if nf != part_floats(B, Hq, D):
        raise RuntimeError("packed shard result size disagrees with the library")
    part = torch.empty(nf, dtype=torch.float32, device=q.device)
    st = fa_decode_splitkv_shard(q, k_shard, v_shard, part, B, Hq, Hkv, Nk_shard, key_offset, Nk_total, D, scale,
                                 num_splits, seqlens_k, workspace, stream=stream)
    if st != FA_OK:
        raise FAError(st, "fa_decode_splitkv_shard")
    parts = gather_parts(part, world, group)
    o = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    st = fa_decode_merge(parts, world, B, Hq, D, o, lse, stream=stream)
    if st != FA_OK:
        raise FAError(st, "fa_decode_merge")
    return o, lse
