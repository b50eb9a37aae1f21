"""Score regimes the online softmax must survive: rising row maxima and scores whose exp overflows.

The tiled method keeps a running row max m and, when a later key block raises it, multiplies the
output accumulator and the row sum by exp(m_old - m_new) (Ascend CANN ops-transformer FlashAttention
article, section "代码讲解": the ``m_new`` update and the rescaled ``O_block``).  The max has to be
subtracted at all because the exponential of a raw score overflows: fp16 already for scores of about
11 ("轻松读懂FlashAttention 上", section "内存卡点", the "小知识" note on safe softmax).

With N(0,1) inputs the first key block almost always holds the row max, so ordinary parity cases
never make the kernels rescale.  Here the inputs are built so that they must:
  * rising scores: channel 0 of every query is a constant and channel 0 of the keys a ramp along the
    key axis (seeded_inputs.key_ramp), so each row's max climbs block after block -- by more than
    the kernels' deferred-rescale threshold (2^8) many times per row, or, with a gentle ramp, in
    steps below it so the stale max is carried across several blocks;
  * large scores: fp16 Q and K with standard deviation 3 and scale 0.5, so the largest score of a
    row is far above 88.7, where exp overflows even in fp32.
Every case is compared with the fp64 oracle element by element (|dO| <= 1e-2, |dLSE| <= 1e-3), and
each rising-score case first checks on the CPU that its inputs really raise the max as intended.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import check, to_device, to_f64, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

LOG2E = 1.0 / math.log(2.0)
THRESHOLD_LOG2 = 8.0  # the kernels' deferred-rescale threshold


@pytest.fixture(scope="module", autouse=True)
def built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_tiled_attention_47_b200 import build
    build.build()
    import exact_tiled_attention_47_b200 as fa
    fa.fa_device_status(clear=True)
    yield
    assert fa.fa_device_status(clear=True) == 0


def fa_mod():
    import exact_tiled_attention_47_b200 as fa
    return fa


def rescale_events(qh, kh, scale, causal, block=128):
    """Per query row, how often a key block raises the running max by more than the threshold
    (log2 units), and how often it raises it at all; fp64 scores of one head."""
    nq, nk = qh.shape[0], kh.shape[0]
    s = scale * (qh @ kh.T) * LOG2E
    if causal:
        s = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq), s, -np.inf)
    big = np.zeros(nq, dtype=np.int64)
    any_ = np.zeros(nq, dtype=np.int64)
    m = s[:, :block].max(axis=1)
    stale = m.copy()
    for j in range(block, nk, block):
        bm = s[:, j:j + block].max(axis=1)
        grew = bm > m
        any_ += grew
        jump = bm > stale + THRESHOLD_LOG2
        big += jump
        stale = np.where(jump, bm, stale)
        m = np.maximum(m, bm)
    return big, any_


# ------------------------------------------------------------------------------------------------
# prefill


RISING = [
    # B, N, H, D, dtype, causal, top (natural-log units of the ramp's total rise)
    (1, 1024, 2, 64, "bf16", True, 48.0),
    (1, 1024, 2, 64, "fp16", False, 48.0),
    (1, 777, 2, 128, "bf16", False, 48.0),
    (1, 1024, 2, 128, "fp16", True, 48.0),
    (2, 640, 2, 64, "bf16", True, 12.0),     # gentle: the max grows in steps below the threshold
    (1, 1024, 2, 128, "bf16", True, 12.0),
    (1, 1300, 1, 64, "bf16", False, 300.0),  # steep: every block jumps far past the threshold
]


@pytest.mark.parametrize("case", RISING, ids=[f"n{c[1]}d{c[3]}{c[4]}{'c' if c[5] else 'n'}r{int(c[6])}" for c in RISING])
def test_rising_scores_prefill(case):
    B, N, H, D, dtype, causal, top = case
    fa = fa_mod()
    scale = 0.125
    q, k, v = si.dense_qkv(6100 + N + D, B, N, N, H, D, dtype)
    q, k = si.key_ramp(q, k, dtype, 8.0, top, key_axis=1)
    qf, kf, vf = to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)
    big, any_ = rescale_events(qf[0, :, 0], kf[0, :, 0], scale, causal)
    if top >= 48.0:
        assert np.median(big[N // 2:]) >= 2, "inputs must raise the max past the threshold repeatedly"
    else:
        assert np.median(any_[N // 2:]) >= 2, "inputs must raise the max below the threshold"
    o, lse = fa.attention(*(to_device(t, dtype) for t in (q, k, v)), causal=causal, scale=scale,
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(qf, kf, vf, scale, causal)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", f"rising {case}")


@pytest.mark.parametrize("D,dtype", [(64, "fp16"), (128, "bf16")])
def test_rising_scores_varlen(D, dtype):
    fa = fa_mod()
    lengths = [900, 129, 1, 640, 300]
    H, scale = 2, 0.1
    q, k, v, cu = si.varlen_qkv(6200 + D, lengths, H, D, dtype)
    q, k = si.key_ramp(q, k, dtype, 8.0, 60.0, key_axis=0, cu_seqlens=cu)
    qf, kf, vf = to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)
    big, _ = rescale_events(qf[0:900, 0], kf[0:900, 0], scale, False)
    assert big.min() >= 2
    o, lse = fa.attention(*(to_device(t, dtype) for t in (q, k, v)), scale=scale,
                          cu_seqlens=torch.from_numpy(cu).cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_varlen(qf, kf, vf, cu, scale, False)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "rising varlen")


def test_rising_scores_prefix_mask():
    fa = fa_mod()
    N, H, D, dtype, prefix, scale = 1024, 2, 64, "bf16", 300, 0.125
    q, k, v = si.dense_qkv(6300, 1, N, N, H, D, dtype)
    q, k = si.key_ramp(q, k, dtype, 8.0, 48.0, key_axis=1)
    o, lse = fa.attention(*(to_device(t, dtype) for t in (q, k, v)), scale=scale, prefix_len=prefix,
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale,
                                            True, prefix)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "rising prefix")


LARGE = [
    # B, N, H, D, dtype, causal, out
    (1, 512, 2, 64, "fp16", False, "fp32"),
    (1, 512, 2, 64, "fp16", True, "fp16"),
    (1, 384, 2, 128, "fp16", True, "fp32"),
    (1, 384, 2, 128, "fp16", False, "fp32"),
]
# bf16 is left out on purpose: with nearly one-hot rows the rounding of P to bf16 before the P*V
# product (relative 2^-9) alone moves O by up to 2^-9 * max|V| ~ 1e-2 for N(0,1) values, the size of
# the tolerance; fp16 P (relative 2^-12) keeps that error at ~1e-3, and fp16 is the pages' case.


@pytest.mark.parametrize("case", LARGE, ids=[f"n{c[1]}d{c[3]}{c[4]}{'c' if c[5] else 'n'}{c[6]}" for c in LARGE])
def test_scores_beyond_exp_overflow(case):
    B, N, H, D, dtype, causal, out = case
    fa = fa_mod()
    scale = 0.5
    q, k, v = si.dense_qkv(6400 + N + D, B, N, N, H, D, dtype)
    q = si.batched(6400 + N + D, si.Q_ID, B, (N, H, D), dtype, std=3.0)
    k = si.batched(6400 + N + D, si.K_ID, B, (N, H, D), dtype, std=3.0)
    qf, kf, vf = to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)
    smax = scale * np.einsum("nd,md->nm", qf[0, :, 0], kf[0, :, 0]).max()
    assert smax > 88.8, "some exp(score) must overflow float32 without the max subtraction"
    o, lse = fa.attention(*(to_device(t, dtype) for t in (q, k, v)), causal=causal, scale=scale,
                          out_dtype=torch_dtype(out))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(qf, kf, vf, scale, causal)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, out, f"large {case}")


# ------------------------------------------------------------------------------------------------
# decode (one query per sequence): the split kernel (one query head per KV head) and the grouped
# tensor-core kernel (several query heads per KV head, deferred rescale)


@pytest.mark.parametrize("Hq,Hkv,D,dtype", [(8, 8, 128, "bf16"), (8, 2, 128, "bf16"), (16, 2, 64, "fp16"),
                                            (32, 4, 128, "fp16")])
@pytest.mark.parametrize("top", [48.0, 12.0])
def test_rising_scores_decode(Hq, Hkv, D, dtype, top):
    fa = fa_mod()
    B, Nk, S = 3, 3000, 4
    scale = 1 / math.sqrt(D)
    q, k, v = si.decode_gqa_inputs(6500 + Hq + D, B, Nk, Hq, Hkv, D, dtype)
    q, k = si.key_ramp(q, k, dtype, 8.0 / (scale * 8.0), top, key_axis=1)  # score rise = top
    lens = [Nk, 2049, 700]
    qf, kf, vf = to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)
    big, any_ = rescale_events(qf[0, :, 0], kf[0, :, 0], scale, False, block=64)
    assert (big if top >= 48.0 else any_)[0] >= 4
    o, lse = fa.decode(*(to_device(t, dtype) for t in (q, k, v)), scale=scale, num_splits=S,
                       out_dtype=torch.float32, seqlens_k=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_gqa(qf, kf, vf, scale, lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", f"rising decode Hq{Hq} Hkv{Hkv}")


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4)])
def test_decode_scores_beyond_exp_overflow(Hq, Hkv):
    fa = fa_mod()
    B, Nk, D, dtype, scale, S = 2, 2000, 64, "fp16", 0.5, 8
    q = si.batched(6600 + Hq, si.Q_ID, B, (1, Hq, D), dtype, std=3.0)
    k = si.batched(6600 + Hq, si.K_ID, B, (Nk, Hkv, D), dtype, std=3.0)
    v = si.batched(6600 + Hq, si.V_ID, B, (Nk, Hkv, D), dtype)
    qf, kf, vf = to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)
    assert scale * (kf[0, :, 0] @ qf[0, 0, 0]).max() > 88.8
    o, lse = fa.decode(*(to_device(t, dtype) for t in (q, k, v)), scale=scale, num_splits=S,
                       out_dtype=torch.float32,
                       seqlens_k=None if Hq == Hkv else torch.tensor([Nk, 999], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_gqa(qf, kf, vf, scale, None if Hq == Hkv else [Nk, 999])
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", f"large decode Hq{Hq}")
