"""Exact tiled attention for NVIDIA B200 (sm_100a): Python binding of libfa_sm100.so.

The functions named like the C entry points (``fa_fwd``, ``fa_decode_splitkv``, ...) only marshal
arguments -- tensors become device pointers, torch streams become ``cudaStream_t`` -- and return the
C status code.  ``attention`` and ``decode`` additionally allocate the outputs with torch and raise
``FAError`` on a non-zero status.  All arithmetic runs in the library's CUDA kernels; there is no
CPU path.  PyTorch supplies device memory and streams only.
"""
from __future__ import annotations

import ctypes
import math

from ._lib import DEBUG_LIB_PATH, LIB_PATH, LibraryMissing, SIGNATURES, load

FA_BF16, FA_FP16, FA_FP32 = 0, 1, 2
(FA_OK, FA_ERR_NULL, FA_ERR_DTYPE, FA_ERR_HEADDIM, FA_ERR_SHAPE, FA_ERR_ALIGN, FA_ERR_CU_SEQLENS,
 FA_ERR_WORKSPACE, FA_ERR_DEVICE, FA_ERR_LAUNCH, FA_ERR_TIMEOUT, FA_ERR_BOUNDS, FA_ERR_PAGE_TABLE) = range(13)
FA_BUILD_DEBUG = 1

__all__ = [
    "fa_fwd", "fa_fwd_prefix", "fa_bwd", "fa_bwd_masked", "fa_bwd_workspace_bytes", "attention_backward", "fa_decode_workspace_bytes", "fa_decode_splitkv", "fa_decode_splitkv_gqa", "fa_decode_splitkv_paged", "decode_paged", "fa_status_string",
    "fa_device_status", "fa_abi_version", "fa_build_flags", "fa_selftest_wait_timeout", "fa_decode_splitkv_noalloc", "FA_NOALLOC_SCRATCH_BYTES",
    "fa_decode_part_bytes", "fa_decode_splitkv_shard", "fa_decode_merge", "decode_sharded", "shard_range", "attention", "decode", "FAError", "LibraryMissing",
    "LIB_PATH", "DEBUG_LIB_PATH", "FA_BF16", "FA_FP16", "FA_FP32", "FA_BUILD_DEBUG",
]


class FAError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: status {status} ({fa_status_string(status)})")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _dtype_code(t):
    import torch
    return {torch.bfloat16: FA_BF16, torch.float16: FA_FP16, torch.float32: FA_FP32}.get(t.dtype, -1)


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, D, scale, causal, cu_seqlens=None, stream=None,
           in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_fwd``; returns its status.  Dtypes default to those of q and o."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    return lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(H), int(Nq), int(Nk),
                      int(D), float(scale), int(bool(causal)), _ptr(cu_seqlens), _stream(stream),
                      int(in_dtype), int(o_dtype))


def fa_fwd_prefix(q, k, v, o, lse, B, H, Nq, Nk, D, scale, prefix_len, cu_seqlens=None, stream=None,
                  in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_fwd_prefix`` (causal with a bidirectional key prefix); returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    return lib.fa_fwd_prefix(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(H), int(Nq), int(Nk),
                             int(D), float(scale), int(prefix_len), _ptr(cu_seqlens), _stream(stream),
                             int(in_dtype), int(o_dtype))


def fa_bwd_workspace_bytes(B, H, Nq) -> int:
    return int(load().fa_bwd_workspace_bytes(int(B), int(H), int(Nq)))


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, D, scale, causal, workspace, workspace_bytes=None,
           stream=None, in_dtype=None, grad_dtype=None) -> int:
    """Marshal to the C ``fa_bwd``; returns its status.  Dtypes default to those of q and dq."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if grad_dtype is None:
        grad_dtype = _dtype_code(dq)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                      int(B), int(H), int(Nq), int(Nk), int(D), float(scale), int(bool(causal)), _ptr(workspace),
                      int(workspace_bytes), _stream(stream), int(in_dtype), int(grad_dtype))


def fa_bwd_masked(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, D, scale, causal, prefix_len, cu_seqlens,
                  workspace, workspace_bytes=None, stream=None, in_dtype=None, grad_dtype=None) -> int:
    """Marshal to the C ``fa_bwd_masked`` (prefix mask, packed varlen); returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if grad_dtype is None:
        grad_dtype = _dtype_code(dq)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                             _ptr(dv), int(B), int(H), int(Nq), int(Nk), int(D), float(scale), int(bool(causal)),
                             int(prefix_len), _ptr(cu_seqlens), _ptr(workspace), int(workspace_bytes),
                             _stream(stream), int(in_dtype), int(grad_dtype))


def fa_decode_workspace_bytes(B, H, D, num_splits) -> int:
    return int(load().fa_decode_workspace_bytes(int(B), int(H), int(D), int(num_splits)))


def fa_decode_splitkv_gqa(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nk, D, scale, num_splits, seqlens_k,
                          workspace, workspace_bytes=None, stream=None, in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_decode_splitkv_gqa``; returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_decode_splitkv_gqa(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), int(B), int(Hq),
                                     int(Hkv), int(Nk), int(D), float(scale), int(num_splits), _ptr(seqlens_k),
                                     _ptr(workspace), int(workspace_bytes), _stream(stream), int(in_dtype),
                                     int(o_dtype))


def fa_decode_splitkv_paged(q, k_pages, v_pages, block_table, o, lse, B, Hq, Hkv, num_pages, page_size,
                            pages_per_seq, D, scale, num_splits, seqlens_k, workspace, workspace_bytes=None,
                            stream=None, in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_decode_splitkv_paged``; returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_decode_splitkv_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(o),
                                       _ptr(lse), int(B), int(Hq), int(Hkv), int(num_pages), int(page_size),
                                       int(pages_per_seq), int(D), float(scale), int(num_splits), _ptr(seqlens_k),
                                       _ptr(workspace), int(workspace_bytes), _stream(stream), int(in_dtype),
                                       int(o_dtype))


def fa_decode_part_bytes(B, H, D) -> int:
    return int(load().fa_decode_part_bytes(int(B), int(H), int(D)))


def fa_decode_splitkv_shard(q, k_shard, v_shard, part, B, Hq, Hkv, Nk_shard, key_offset, Nk_total, D, scale,
                            num_splits, seqlens_k, workspace, workspace_bytes=None, stream=None,
                            in_dtype=None) -> int:
    """Marshal to the C ``fa_decode_splitkv_shard``; returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_decode_splitkv_shard(_ptr(q), _ptr(k_shard), _ptr(v_shard), _ptr(part), int(B), int(Hq),
                                       int(Hkv), int(Nk_shard), int(key_offset), int(Nk_total), int(D),
                                       float(scale), int(num_splits), _ptr(seqlens_k), _ptr(workspace),
                                       int(workspace_bytes), _stream(stream), int(in_dtype))


def fa_decode_merge(parts, R, B, H, D, o, lse, stream=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_decode_merge``; returns its status."""
    lib = load()
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    return lib.fa_decode_merge(_ptr(parts), int(R), int(B), int(H), int(D), _ptr(o), _ptr(lse), _stream(stream),
                               int(o_dtype))


def fa_decode_splitkv(q, k_cache, v_cache, o, lse, B, H, Nk, D, scale, num_splits, workspace,
                      workspace_bytes=None, stream=None, in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_decode_splitkv``; returns its status."""
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return lib.fa_decode_splitkv(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), int(B),
                                 int(H), int(Nk), int(D), float(scale), int(num_splits),
                                 _ptr(workspace), int(workspace_bytes), _stream(stream),
                                 int(in_dtype), int(o_dtype))


# Size of the library's fixed decode scratch array (FA_NOALLOC_SCRATCH_BYTES in include/fa.h).
FA_NOALLOC_SCRATCH_BYTES = 32 << 20


def fa_decode_splitkv_noalloc(q, k_cache, v_cache, o, lse, B, H, Nk, D, scale, num_splits,
                              stream=None, in_dtype=None, o_dtype=None) -> int:
    """Marshal to the C ``fa_decode_splitkv_noalloc``: decode for callers that cannot allocate.

    Same results as ``fa_decode_splitkv``; the split partials live in the library's fixed
    per-GPU scratch array instead of a caller workspace, so nothing is allocated per call.
    Calls on one device share that array: do not let two of them overlap on the GPU.
    """
    lib = load()
    if in_dtype is None:
        in_dtype = _dtype_code(q)
    if o_dtype is None:
        o_dtype = _dtype_code(o)
    return lib.fa_decode_splitkv_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                         int(B), int(H), int(Nk), int(D), float(scale),
                                         int(num_splits), _stream(stream), int(in_dtype),
                                         int(o_dtype))


def fa_status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def fa_device_status(clear: bool = True) -> int:
    """Device status word of the current device (synchronises); resets it when ``clear``."""
    out = ctypes.c_int(-1)
    st = load().fa_device_status(ctypes.byref(out), int(bool(clear)))
    if st != FA_OK:
        raise FAError(st, "fa_device_status")
    return out.value


def fa_selftest_wait_timeout(stream=None):
    """Run the bounded-wait self-test; returns (status, waited_ms)."""
    w = ctypes.c_int(0)
    st = load().fa_selftest_wait_timeout(ctypes.byref(w), _stream(stream))
    return int(st), int(w.value)


def fa_abi_version() -> int:
    return int(load().fa_abi_version())


def fa_build_flags() -> int:
    return int(load().fa_build_flags())


# ------------------------------------------------------------------------------------------------
# allocating helpers (torch allocates; the library computes)


def attention(q, k, v, causal=False, scale=None, cu_seqlens=None, out_dtype=None, stream=None,
              prefix_len=None):
    """O, LSE for q [B,Nq,H,D], k/v [B,Nk,H,D] (dense) or packed [total,H,D] with cu_seqlens.

    ``prefix_len`` (not None) selects the prefix mask (causal, with the first prefix_len keys visible
    to every query); ``causal`` is then ignored.
    """
    import torch
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if cu_seqlens is None:
        B, Nq, H, _ = q.shape
        Nk = k.shape[1]
        lse = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32)
    else:
        Nq, H, _ = q.shape
        Nk = k.shape[0]
        B = cu_seqlens.numel() - 1
        lse = torch.empty((H, Nq), device=q.device, dtype=torch.float32)
    o = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    if prefix_len is None:
        st = fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, D, scale, causal, cu_seqlens, stream)
    else:
        st = fa_fwd_prefix(q, k, v, o, lse, B, H, Nq, Nk, D, scale, prefix_len, cu_seqlens, stream)
    if st != FA_OK:
        raise FAError(st, "fa_fwd_prefix" if prefix_len is not None else "fa_fwd")
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal=False, scale=None, grad_dtype=None, stream=None,
                       prefix_len=None, cu_seqlens=None):
    """dQ, dK, dV for the forward o / lse and the upstream dout.

    Dense q [B,Nq,H,D], k/v [B,Nk,H,D], or packed [total,H,D] with ``cu_seqlens``; ``prefix_len``
    (not None) selects the prefix mask of ``attention(..., prefix_len=...)``.
    """
    import torch
    D = q.shape[-1]
    if cu_seqlens is None:
        B, Nq, H, _ = q.shape
        Nk = k.shape[1]
        nb = fa_bwd_workspace_bytes(B, H, Nq)
    else:
        Nq, H, _ = q.shape
        Nk = k.shape[0]
        B = cu_seqlens.numel() - 1
        nb = fa_bwd_workspace_bytes(1, H, Nq)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    grad_dtype = q.dtype if grad_dtype is None else grad_dtype
    dq = torch.empty(q.shape, device=q.device, dtype=grad_dtype)
    dk = torch.empty(k.shape, device=q.device, dtype=grad_dtype)
    dv = torch.empty(v.shape, device=q.device, dtype=grad_dtype)
    ws = torch.empty(nb, device=q.device, dtype=torch.uint8)
    if prefix_len is None and cu_seqlens is None:
        st = fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, D, scale, causal, ws, stream=stream)
    else:
        st = fa_bwd_masked(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, D, scale, causal,
                           0 if prefix_len is None else prefix_len, cu_seqlens, ws, stream=stream)
    if st != FA_OK:
        raise FAError(st, "fa_bwd" if prefix_len is None and cu_seqlens is None else "fa_bwd_masked")
    return dq, dk, dv


def decode(q, k_cache, v_cache, scale=None, num_splits=16, out_dtype=None, workspace=None,
           stream=None, seqlens_k=None):
    """O [B,1,Hq,D], LSE [B,Hq] for one query per (batch, head) over the cache [B,Nk,Hkv,D].

    Hkv < Hq (a divisor of it) or ``seqlens_k`` (int32 [B] on the device) select the grouped /
    ragged entry point ``fa_decode_splitkv_gqa``.
    """
    import torch
    B, _, H, D = q.shape
    Nk, Hkv = k_cache.shape[1], k_cache.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out_dtype = q.dtype if out_dtype is None else out_dtype
    nbytes = fa_decode_workspace_bytes(B, H, D, num_splits)
    if workspace is None:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    o = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    nb = workspace.numel() * workspace.element_size()
    if Hkv == H and seqlens_k is None:
        st = fa_decode_splitkv(q, k_cache, v_cache, o, lse, B, H, Nk, D, scale, num_splits, workspace, nb, stream)
    else:
        st = fa_decode_splitkv_gqa(q, k_cache, v_cache, o, lse, B, H, Hkv, Nk, D, scale, num_splits, seqlens_k,
                                   workspace, nb, stream)
    if st != FA_OK:
        raise FAError(st, "fa_decode_splitkv" if Hkv == H and seqlens_k is None else "fa_decode_splitkv_gqa")
    return o, lse


def decode_paged(q, k_pages, v_pages, block_table, seqlens_k=None, scale=None, num_splits=16, out_dtype=None,
                 workspace=None, stream=None):
    """O [B,1,Hq,D], LSE [B,Hq] for one query per (batch, head) over a paged cache.

    k_pages/v_pages [num_pages, page_size, Hkv, D]; block_table int32 [B, pages_per_seq] on the device
    (entry (b, i): the page holding keys [i*page_size, (i+1)*page_size) of batch item b); seqlens_k
    int32 [B] on the device or None (every table entry in use).
    """
    import torch
    B, _, H, D = q.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    pages_per_seq = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out_dtype = q.dtype if out_dtype is None else out_dtype
    if workspace is None:
        workspace = torch.empty(fa_decode_workspace_bytes(B, H, D, num_splits), device=q.device, dtype=torch.uint8)
    o = torch.empty(q.shape, device=q.device, dtype=out_dtype)
    lse = torch.empty((B, H), device=q.device, dtype=torch.float32)
    st = fa_decode_splitkv_paged(q, k_pages, v_pages, block_table, o, lse, B, H, Hkv, num_pages, page_size,
                                 pages_per_seq, D, scale, num_splits, seqlens_k, workspace, stream=stream)
    if st != FA_OK:
        raise FAError(st, "fa_decode_splitkv_paged")
    return o, lse


from .sharded import decode_sharded, shard_range  # noqa: E402  (key-sharded decode over ranks)
