"""Key-sharded decode (fa_decode_splitkv_shard + fa_decode_merge) against the fp64 oracle (GPU only).

One GPU stands in for R ranks without any rank waiting on another: the cache is cut into R
contiguous key shards, the shard kernels run one after another into R packed result blocks laid
out exactly as the all-gather of R ranks leaves them, and the merge kernel combines the blocks.
Each shard's own result is checked against the oracle's decode over that shard, and the merged
output against the oracle's decode over the whole cache.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import check, to_device, to_f64, torch_dtype

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


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


def run_shards(q, k, v, dtype, R, S, lens, scale, out="fp32", check_parts=True, block_order=None):
    """Shard results of R key shards into one packed buffer, then the merge; returns (o, lse, parts)."""
    import exact_tiled_attention_47_b200 as fa
    from exact_tiled_attention_47_b200.sharded import part_floats, shard_range
    B, _, Hq, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    nf = part_floats(B, Hq, D)
    assert fa.fa_decode_part_bytes(B, Hq, D) == 4 * nf
    parts = torch.full((R * nf,), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, Hq, D, S), dtype=torch.uint8, device="cuda")
    qd = to_device(q, dtype)
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    order = list(range(R)) if block_order is None else block_order
    for slot, r in enumerate(order):
        off, n = shard_range(Nk, R, r)
        ks = to_device(np.ascontiguousarray(k[:, off:off + n]), dtype)
        vs = to_device(np.ascontiguousarray(v[:, off:off + n]), dtype)
        blk = parts[slot * nf:(slot + 1) * nf]
        st = fa.fa_decode_splitkv_shard(qd, ks, vs, blk, B, Hq, Hkv, n, off, Nk, D, scale, S, sl, ws)
        assert st == 0, fa.fa_status_string(st)
        if check_parts:
            torch.cuda.synchronize()
            o_r, l_r = oracle.attention_decode_shard(to_f64(q, dtype), to_f64(k[:, off:off + n], dtype),
                                                     to_f64(v[:, off:off + n], dtype), scale, off, lens)
            got = blk.cpu().numpy()
            check(got[:B * Hq * D].reshape(B, 1, Hq, D), got[B * Hq * D:B * Hq * (D + 1)].reshape(B, Hq), o_r, l_r,
                  "fp32", f"shard {r} of {R} (keys {off}..{off + n})")
    o = torch.empty((B, 1, Hq, D), dtype=torch_dtype(out), device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    st = fa.fa_decode_merge(parts, R, B, Hq, D, o, lse)
    assert st == 0, fa.fa_status_string(st)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    return o, lse, parts


CASES = [
    # B, Hq, Hkv, Nk_total, D, dtype, shards, splits, out, lengths
    (4, 8, 2, 3000, 128, "bf16", 3, 16, "fp32", [3000, 1000, 1001, 0]),   # lengths on a shard boundary
    (3, 12, 4, 777, 64, "fp16", 2, 8, "fp16", None),                       # full cache, odd shard sizes
    (2, 16, 16, 4096, 128, "bf16", 8, 4, "bf16", [4096, 5]),               # no grouping; 7 empty shards
    (5, 8, 8, 2051, 64, "bf16", 4, 16, "fp32", [1, 513, 514, 2050, 2051]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}hq{c[1]}hkv{c[2]}n{c[3]}d{c[4]}r{c[6]}" for c in CASES])
def test_shard_cases(case):
    B, Hq, Hkv, Nk, D, dtype, R, S, out, lens = case
    scale = 1 / math.sqrt(D)
    q, k, v = si.decode_gqa_inputs(900 + Nk + R, B, Nk, Hq, Hkv, D, dtype)
    o, lse, _ = run_shards(q, k, v, dtype, R, S, lens, scale, out)
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale, lens)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, out,
          f"sharded decode B{B} Hq{Hq} Hkv{Hkv} Nk{Nk} D{D} R{R}")


def test_merge_ignores_block_order():
    # the gathered blocks may arrive in any rank order: the merge is a symmetric function of them
    B, Hq, Hkv, Nk, D, R, S = 2, 8, 2, 1200, 128, 4, 8
    q, k, v = si.decode_gqa_inputs(931, B, Nk, Hq, Hkv, D, "bf16")
    o1, l1, _ = run_shards(q, k, v, "bf16", R, S, [1200, 700], 0.09, check_parts=False)
    o2, l2, _ = run_shards(q, k, v, "bf16", R, S, [1200, 700], 0.09, check_parts=False, block_order=[2, 0, 3, 1])
    np.testing.assert_allclose(o1.cpu().numpy(), o2.cpu().numpy(), rtol=0, atol=1e-6)
    np.testing.assert_allclose(l1.cpu().numpy(), l2.cpu().numpy(), rtol=0, atol=1e-6)


def test_one_shard_equals_plain_decode():
    # R = 1: the shard result holds the whole-cache output; the merge of one block returns it
    import exact_tiled_attention_47_b200 as fa
    B, Hq, Hkv, Nk, D, S = 3, 8, 2, 1500, 128, 16
    q, k, v = si.decode_gqa_inputs(932, B, Nk, Hq, Hkv, D, "bf16")
    lens = [1500, 3, 0]
    o_s, l_s, _ = run_shards(q, k, v, "bf16", 1, S, lens, 0.1, check_parts=False)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o_p, l_p = fa.decode(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), scale=0.1, num_splits=S,
                         out_dtype=torch.float32, seqlens_k=sl)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_p)
    np.testing.assert_allclose(l_s.cpu().numpy(), l_p.cpu().numpy(), rtol=0, atol=1e-5)


def test_decode_sharded_single_process():
    # the public helper with one process: shard = whole cache, no exchange
    import exact_tiled_attention_47_b200 as fa
    from exact_tiled_attention_47_b200.sharded import decode_sharded
    B, Hq, Hkv, Nk, D = 2, 8, 4, 900, 64
    q, k, v = si.decode_gqa_inputs(933, B, Nk, Hq, Hkv, D, "fp16")
    sl = torch.tensor([900, 450], dtype=torch.int32, device="cuda")
    o, lse = decode_sharded(to_device(q, "fp16"), to_device(k, "fp16"), to_device(v, "fp16"), 0, Nk,
                            seqlens_k=sl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, "fp16"), to_f64(k, "fp16"), to_f64(v, "fp16"),
                                                 1 / math.sqrt(D), [900, 450])
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "decode_sharded, one process")


def test_bad_total_length_is_reported():
    # a length beyond the whole cache is caught by every shard and treated as 0
    import exact_tiled_attention_47_b200 as fa
    B, Hq, Hkv, Nk, D, S = 2, 4, 4, 600, 128, 4
    q, k, v = si.decode_gqa_inputs(934, B, Nk, Hq, Hkv, D, "bf16")
    nf = fa.fa_decode_part_bytes(B, Hq, D) // 4
    part = torch.empty(nf, dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, Hq, D, S), dtype=torch.uint8, device="cuda")
    sl = torch.tensor([600, 601], dtype=torch.int32, device="cuda")
    ks = to_device(np.ascontiguousarray(k[:, 300:]), "bf16")
    vs = to_device(np.ascontiguousarray(v[:, 300:]), "bf16")
    st = fa.fa_decode_splitkv_shard(to_device(q, "bf16"), ks, vs, part, B, Hq, Hkv, 300, 300, Nk, D, 0.1, S, sl, ws)
    assert st == 0
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_CU_SEQLENS
    got = part.cpu().numpy()
    lse = got[B * Hq * D:B * Hq * (D + 1)].reshape(B, Hq)
    assert np.all(np.isfinite(lse[0])) and np.all(lse[1] == -np.inf)
    assert np.all(got[Hq * D:2 * Hq * D] == 0)


def test_long_context_sampled():
    # 64k-key cache (the long contexts of "轻松读懂FlashAttention 上", "内存卡点") over 4 shards;
    # the oracle evaluates every (b, h) of the whole cache
    B, Hq, Hkv, Nk, D, R, S = 2, 8, 8, 65536, 128, 4, 16
    q, k, v = si.decode_gqa_inputs(935, B, Nk, Hq, Hkv, D, "bf16")
    lens = [65536, 40000]
    o, lse, _ = run_shards(q, k, v, "bf16", R, S, lens, 1 / math.sqrt(D), check_parts=False)
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"),
                                                 1 / math.sqrt(D), lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "sharded decode, 64k keys over 4 shards")
