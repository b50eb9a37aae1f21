"""Decode with grouped KV heads and per-sequence cache lengths (fa_decode_splitkv_gqa) against the
fp64 oracle (GPU only)."""
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


def run(B, Hq, Hkv, Nk, D, dtype, S, out, lens, seed, scale=None):
    import exact_tiled_attention_47_b200 as fa
    scale = 1 / math.sqrt(D) if scale is None else scale
    q, k, v = si.decode_gqa_inputs(seed, B, Nk, Hq, Hkv, D, dtype)
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = fa.decode(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype), scale=scale,
                       num_splits=S, out_dtype=torch_dtype(out), seqlens_k=sl)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale, lens)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, out,
          f"decode gqa B{B} Hq{Hq} Hkv{Hkv} Nk{Nk} D{D} S{S}")
    return o, lse


CASES = [
    # B, Hq, Hkv, Nk, D, dtype, splits, out, lengths
    (4, 32, 8, 1000, 128, "bf16", 16, "fp32", [1000, 1, 517, 0]),      # 4 heads per CTA
    (3, 12, 4, 777, 64, "fp16", 8, "fp32", None),                       # group 3: one head per CTA
    (2, 16, 1, 513, 128, "bf16", 4, "bf16", [513, 300]),               # group 16: two CTAs of 8
    (2, 12, 2, 300, 64, "bf16", 16, "fp32", [5, 299]),                 # group 6: CTAs of 2, empty splits
    (2, 8, 8, 300, 128, "bf16", 8, "fp32", [123, 0]),                  # no grouping, ragged only
    (5, 8, 2, 4099, 128, "fp16", 128, "fp16", [4099, 4098, 2048, 129, 128]),
    (2, 16, 2, 1500, 64, "bf16", 16, "fp32", [1500, 700]),            # group 8, D = 64
    (3, 32, 4, 2000, 128, "fp16", 8, "fp32", [2000, 63, 64]),          # group 8; one partial tile
    (4, 4, 1, 700, 64, "fp16", 2, "fp16", [65, 128, 129, 700]),       # group 4 at tile edges
    (2, 32, 2, 1000, 64, "bf16", 4, "fp32", [1000, 511]),             # group 16, D = 64
]


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}hq{c[1]}hkv{c[2]}n{c[3]}d{c[4]}s{c[6]}" for c in CASES])
def test_gqa_cases(case):
    B, Hq, Hkv, Nk, D, dtype, S, out, lens = case
    run(B, Hq, Hkv, Nk, D, dtype, S, out, lens, seed=700 + Nk + S + Hkv)


def test_ungrouped_full_length_equals_plain_decode():
    import exact_tiled_attention_47_b200 as fa
    B, H, Nk, D, S = 3, 4, 1000, 128, 16
    q, k, v = si.decode_inputs(777, B, Nk, H, D, "bf16")
    qd, kd, vd = (to_device(t, "bf16") for t in (q, k, v))
    o1, l1 = fa.decode(qd, kd, vd, num_splits=S)
    nb = fa.fa_decode_workspace_bytes(B, H, D, S)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    full = torch.full((B,), Nk, dtype=torch.int32, device="cuda")
    assert fa.fa_decode_splitkv_gqa(qd, kd, vd, o2, l2, B, H, H, Nk, D, 1 / math.sqrt(D), S, full, ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_lengths_are_reported_and_skipped():
    import exact_tiled_attention_47_b200 as fa
    B, Hq, Hkv, Nk, D, S = 3, 8, 2, 200, 64, 4
    q, k, v = si.decode_gqa_inputs(778, B, Nk, Hq, Hkv, D, "bf16")
    qd, kd, vd = (to_device(t, "bf16") for t in (q, k, v))
    lens = [100, -3, Nk + 1]
    o, lse = fa.decode(qd, kd, vd, num_splits=S, out_dtype=torch.float32,
                       seqlens_k=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_CU_SEQLENS
    on, ln = o.cpu().numpy(), lse.cpu().numpy()
    assert np.all(on[1:] == 0) and np.all(ln[1:] == -np.inf)  # out-of-range lengths count as 0
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q[:1], "bf16"), to_f64(k[:1], "bf16"), to_f64(v[:1], "bf16"),
                                                 1 / math.sqrt(D), [100])
    check(on[:1], ln[:1], o_ref, lse_ref, "fp32", "valid item next to bad lengths")


def test_gqa_full_config_sampled():
    import exact_tiled_attention_47_b200 as fa
    c = si.CONFIGS["decode_gqa"]
    B, Nk, Hq, Hkv, D = c["B"], c["Nk"], c["H"], c["Hkv"], c["D"]
    lens = si.varlen_lengths(c["seed"], B, c["len_lo"], c["len_hi"])
    q, k, v = si.decode_gqa_inputs(c["seed"], B, Nk, Hq, Hkv, D, c["dtype"])
    o, lse = fa.decode(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), scale=c["scale"],
                       num_splits=c["num_splits"], out_dtype=torch.float32,
                       seqlens_k=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    on, ln = o.cpu().numpy(), lse.cpu().numpy()
    for b in (0, 1, 17, 40, B - 1):
        o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q[b:b + 1], "bf16"), to_f64(k[b:b + 1], "bf16"),
                                                     to_f64(v[b:b + 1], "bf16"), c["scale"], [int(lens[b])])
        check(on[b:b + 1], ln[b:b + 1], o_ref, lse_ref, "fp32", f"decode_gqa item {b} len {lens[b]}")


@pytest.mark.parametrize("Hq,Hkv,D,dtype", [(16, 4, 64, "bf16"), (8, 1, 128, "fp16"), (6, 6, 64, "bf16")])
def test_nan_past_the_valid_length_does_not_reach_o(Hq, Hkv, D, dtype):
    # cache rows past an item's valid length may hold anything, NaN included (capacity never
    # written); the last 64-key tile of the tensor-core kernel loads some of them, so their value
    # rows must not enter P V even with P = 0
    import exact_tiled_attention_47_b200 as fa
    B, Nk, S = 3, 1000, 4
    lens = [999, 500, 77]
    q, k, v = si.decode_gqa_inputs(990 + Hq, B, Nk, Hq, Hkv, D, dtype)
    nan = {"bf16": 0x7FC0, "fp16": 0x7E00}[dtype]
    k2, v2 = k.copy(), v.copy()
    for b, L in enumerate(lens):
        k2[b, L:] = nan
        v2[b, L:] = nan
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = fa.decode(to_device(q, dtype), to_device(k2, dtype), to_device(v2, dtype), num_splits=S,
                       out_dtype=torch.float32, seqlens_k=sl)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype),
                                                 1 / math.sqrt(D), lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", f"NaN past the lengths, Hq{Hq} Hkv{Hkv}")
