"""Decode over a paged cache (fa_decode_splitkv_paged) against the fp64 oracle (GPU only).

The pool is built from the seeded contiguous cache: each batch item's pages sit at shuffled pool
positions, every row past the item's valid length and every spare page holds NaN, and the table
entries past the pages an item needs are -1; none of that may reach the result.
"""
import math

import pytest

import oracle
import seeded_inputs as si
from parity import check, paginate, to_device, to_f64, torch_dtype

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


def run_paged(B, Hq, Hkv, D, dtype, ps, S, out, lens, seed, cap=None):
    import exact_tiled_attention_47_b200 as fa
    scale = 1 / math.sqrt(D)
    Nk = cap or -(-max(lens + [1]) // ps) * ps
    q, k, v = si.decode_gqa_inputs(seed, B, Nk, Hq, Hkv, D, dtype)
    kp, vp, table = paginate(k, v, lens, ps, dtype, seed)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = fa.decode_paged(to_device(q, dtype), to_device(kp, dtype), to_device(vp, dtype),
                             torch.from_numpy(table).cuda(), sl, scale=scale, num_splits=S, out_dtype=torch_dtype(out))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_paged(to_f64(q, dtype), to_f64(kp, dtype), to_f64(vp, dtype), table,
                                                   scale, lens)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, out,
          f"paged decode B{B} Hq{Hq} Hkv{Hkv} D{D} page {ps} S{S}")
    return o, lse


CASES = [
    # B, Hq, Hkv, D, dtype, page size, splits, out, lengths
    (4, 32, 8, 128, "bf16", 16, 8, "fp32", [1000, 1, 0, 777]),     # 4 heads per CTA, four pages per tile
    (3, 8, 8, 64, "fp16", 64, 4, "fp16", [513, 64, 2000]),         # no grouping: CUDA-core kernel
    (2, 16, 1, 64, "bf16", 256, 16, "fp32", [5000, 300]),           # group 16, pages longer than a tile
    (2, 4, 2, 128, "fp16", 32, 8, "fp32", [100, 4097]),             # group 2, two pages per tile
    (2, 12, 4, 128, "bf16", 16, 16, "bf16", [17, 2049]),            # group 3: CUDA-core kernel, 16-row pages
    (3, 16, 2, 64, "bf16", 128, 128, "fp32", [8192, 129, 4000]),    # 128 splits (ranges of 64-key tiles)
]


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}hq{c[1]}hkv{c[2]}d{c[3]}p{c[5]}s{c[6]}" for c in CASES])
def test_paged_cases(case):
    B, Hq, Hkv, D, dtype, ps, S, out, lens = case
    run_paged(B, Hq, Hkv, D, dtype, ps, S, out, lens, seed=900 + ps + S + Hkv)


@pytest.mark.parametrize("Hq,Hkv", [(16, 4), (4, 4)])
def test_paged_equals_contiguous_bitwise(Hq, Hkv):
    # split ranges of whole 64-key tiles on both layouts (here 512 keys each): the same arithmetic in
    # the same order, so the paged result is the contiguous one bit for bit
    import exact_tiled_attention_47_b200 as fa
    B, D, Nk, S, ps, dtype = 3, 128, 2048, 8, 64, "bf16"
    lens = [2048, 1500, 64]
    q, k, v = si.decode_gqa_inputs(950 + Hkv, B, Nk, Hq, Hkv, D, dtype)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    qd = to_device(q, dtype)
    o1, l1 = fa.decode(qd, to_device(k, dtype), to_device(v, dtype), num_splits=S, seqlens_k=sl)
    kp, vp, table = paginate(k, v, lens, ps, dtype, 951)
    o2, l2 = fa.decode_paged(qd, to_device(kp, dtype), to_device(vp, dtype), torch.from_numpy(table).cuda(), sl,
                             num_splits=S)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_full_table_without_lengths():
    # seqlens_k = NULL: every table entry is in use (capacity = pages_per_seq * page_size)
    import exact_tiled_attention_47_b200 as fa
    B, Hq, Hkv, D, ps, dtype = 2, 8, 2, 64, 32, "fp16"
    Nk = 10 * ps
    q, k, v = si.decode_gqa_inputs(960, B, Nk, Hq, Hkv, D, dtype)
    kp, vp, table = paginate(k, v, [Nk] * B, ps, dtype, 961)
    o, lse = fa.decode_paged(to_device(q, dtype), to_device(kp, dtype), to_device(vp, dtype),
                             torch.from_numpy(table).cuda(), None, num_splits=4, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_paged(to_f64(q, dtype), to_f64(kp, dtype), to_f64(vp, dtype), table,
                                                   1 / math.sqrt(D), [Nk] * B)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "paged decode, full tables")


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4)])
def test_bad_table_entry_is_reported(Hq, Hkv):
    # an entry outside the pool that an item needs is caught before anything is read through it:
    # the status becomes FA_ERR_PAGE_TABLE and the items with good tables are still right
    import exact_tiled_attention_47_b200 as fa
    B, D, ps, dtype, S = 3, 64, 64, "bf16", 4
    lens = [600, 600, 600]
    Nk = 640
    q, k, v = si.decode_gqa_inputs(970 + Hkv, B, Nk, Hq, Hkv, D, dtype)
    kp, vp, table = paginate(k, v, lens, ps, dtype, 971)
    bad = table.copy()
    bad[1, 3] = kp.shape[0]  # one past the last page
    bad[2, 0] = -7
    o, lse = fa.decode_paged(to_device(q, dtype), to_device(kp, dtype), to_device(vp, dtype),
                             torch.from_numpy(bad).cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"),
                             num_splits=S, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_PAGE_TABLE
    o_ref, lse_ref = oracle.attention_decode_paged(to_f64(q, dtype), to_f64(kp, dtype), to_f64(vp, dtype), table,
                                                   1 / math.sqrt(D), lens)
    check(o[:1].cpu().numpy(), lse[:1].cpu().numpy(), o_ref[:1], lse_ref[:1], "fp32", "item with a good table")


def test_lengths_past_the_capacity_are_reported():
    import exact_tiled_attention_47_b200 as fa
    B, Hq, Hkv, D, ps, dtype = 2, 8, 2, 128, 16, "bf16"
    Nk = 4 * ps
    q, k, v = si.decode_gqa_inputs(980, B, Nk, Hq, Hkv, D, dtype)
    kp, vp, table = paginate(k, v, [Nk, Nk], ps, dtype, 981)
    sl = torch.tensor([Nk + 1, 10], dtype=torch.int32, device="cuda")
    fa.decode_paged(to_device(q, dtype), to_device(kp, dtype), to_device(vp, dtype), torch.from_numpy(table).cuda(),
                    sl, num_splits=2)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_CU_SEQLENS
