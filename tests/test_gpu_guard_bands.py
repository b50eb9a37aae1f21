"""Canary guard bands around every buffer the library writes (GPU only).

Out-of-bounds writes are invisible to a parity check that only reads the output's own elements.
Here each output, workspace and result block handed to the C ABI sits between two 4 KiB bands of a
sentinel byte (tests/parity.py, ``Guarded``); after the call the bands must be untouched and the
output must still match the fp64 oracle.  The outputs start out filled with the sentinel as well,
so an element the kernels never write shows up as a parity failure.  The cases are the ragged and
edge shapes of each entry point: tails of partial tiles, rows without keys, empty splits and
shards, a 1-token sequence, more splits than keys.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import Guarded, check, paginate, to_device, to_f64, torch_dtype

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


def fa_mod():
    import exact_tiled_attention_47_b200 as fa
    return fa


def finish(fa, *guards):
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    for g in guards:
        assert g.intact(), "a kernel wrote outside its buffer"


PREFILL = [
    # B, Nq, Nk, H, D, dtype, causal, prefix, out
    (2, 333, 200, 3, 128, "bf16", True, 0, "fp32"),   # leading rows see no key
    (2, 200, 333, 2, 64, "fp16", True, 0, "fp16"),
    (1, 129, 129, 2, 64, "bf16", False, 0, "bf16"),
    (1, 17, 17, 1, 128, "bf16", True, 0, "fp32"),
    (2, 300, 300, 2, 64, "bf16", True, 77, "fp32"),   # prefix mask
    (1, 513, 513, 2, 128, "fp16", True, 600, "fp16"),  # prefix past the end: no mask
]


@pytest.mark.parametrize("case", PREFILL, ids=[f"{c[1]}x{c[2]}d{c[4]}{c[5]}c{int(c[6])}p{c[7]}{c[8]}" for c in PREFILL])
def test_prefill_writes_stay_inside(case):
    B, Nq, Nk, H, D, dtype, causal, prefix, out = case
    fa = fa_mod()
    scale = 1 / math.sqrt(D)
    q, k, v = si.dense_qkv(7100 + Nq + Nk + D, B, Nq, Nk, H, D, dtype)
    qd, kd, vd = (to_device(t, dtype) for t in (q, k, v))
    og = Guarded((B, Nq, H, D), torch_dtype(out))
    lg = Guarded((B, H, Nq), torch.float32)
    if prefix:
        st = fa.fa_fwd_prefix(qd, kd, vd, og.t, lg.t, B, H, Nq, Nk, D, scale, prefix)
    else:
        st = fa.fa_fwd(qd, kd, vd, og.t, lg.t, B, H, Nq, Nk, D, scale, causal)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    finish(fa, og, lg)
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale,
                                            causal or prefix > 0, prefix)
    check(og.t.float().cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref, out, f"guarded {case}")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_writes_stay_inside(causal):
    fa = fa_mod()
    lengths = [1, 300, 0, 129, 511, 2]
    H, D, dtype, scale = 2, 64, "fp16", 0.1
    q, k, v, cu = si.varlen_qkv(7200, lengths, H, D, dtype)
    total = int(cu[-1])
    qd, kd, vd = (to_device(t, dtype) for t in (q, k, v))
    og = Guarded((total, H, D), torch.float32)
    lg = Guarded((H, total), torch.float32)
    st = fa.fa_fwd(qd, kd, vd, og.t, lg.t, len(lengths), H, total, total, D, scale, causal,
                   torch.from_numpy(cu).cuda())
    assert st == fa.FA_OK
    finish(fa, og, lg)
    o_ref, lse_ref = oracle.attention_varlen(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), cu, scale, causal)
    check(og.t.cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref, "fp32", "guarded varlen")


DECODE = [
    # B, Hq, Hkv, Nk, D, dtype, splits, out, lengths (None = full cache, plain entry point)
    (3, 4, 4, 77, 64, "fp16", 16, "fp32", None),          # more splits than keys would need
    (2, 3, 3, 5, 128, "bf16", 16, "bf16", None),          # more splits than keys
    (4, 16, 4, 1000, 128, "bf16", 8, "fp32", [1000, 0, 63, 64]),   # tensor-core grouped kernel
    (3, 12, 4, 700, 64, "fp16", 4, "fp16", [1, 700, 129]),         # group 3: split kernel
]


@pytest.mark.parametrize("case", DECODE, ids=[f"b{c[0]}hq{c[1]}hkv{c[2]}n{c[3]}d{c[4]}s{c[6]}" for c in DECODE])
def test_decode_writes_stay_inside(case):
    B, Hq, Hkv, Nk, D, dtype, S, out, lens = case
    fa = fa_mod()
    scale = 1 / math.sqrt(D)
    q, k, v = si.decode_gqa_inputs(7300 + Nk + S, B, Nk, Hq, Hkv, D, dtype)
    qd, kd, vd = (to_device(t, dtype) for t in (q, k, v))
    og = Guarded((B, 1, Hq, D), torch_dtype(out))
    lg = Guarded((B, Hq), torch.float32)
    nb = fa.fa_decode_workspace_bytes(B, Hq, D, S)
    wg = Guarded((nb,), torch.uint8)
    if lens is None:
        st = fa.fa_decode_splitkv(qd, kd, vd, og.t, lg.t, B, Hq, Nk, D, scale, S, wg.t, nb)
    else:
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        st = fa.fa_decode_splitkv_gqa(qd, kd, vd, og.t, lg.t, B, Hq, Hkv, Nk, D, scale, S, sl, wg.t, nb)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    finish(fa, og, lg, wg)
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale, lens)
    check(og.t.float().cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref, out, f"guarded decode {case}")


@pytest.mark.parametrize("Hq,Hkv,ps", [(16, 4, 16), (6, 6, 64)])
def test_paged_decode_writes_stay_inside(Hq, Hkv, ps):
    fa = fa_mod()
    B, D, S, dtype = 3, 128, 8, "bf16"
    lens = [700, 1, 129]
    Nk = -(-max(lens) // ps) * ps
    scale = 1 / math.sqrt(D)
    q, k, v = si.decode_gqa_inputs(7700 + ps, B, Nk, Hq, Hkv, D, dtype)
    kp, vp, table = paginate(k, v, lens, ps, dtype, 7701)
    og = Guarded((B, 1, Hq, D), torch.float32)
    lg = Guarded((B, Hq), torch.float32)
    nb = fa.fa_decode_workspace_bytes(B, Hq, D, S)
    wg = Guarded((nb,), torch.uint8)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st = fa.fa_decode_splitkv_paged(to_device(q, dtype), to_device(kp, dtype), to_device(vp, dtype),
                                    torch.from_numpy(table).cuda(), og.t, lg.t, B, Hq, Hkv, kp.shape[0], ps,
                                    table.shape[1], D, scale, S, sl, wg.t, nb)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    finish(fa, og, lg, wg)
    o_ref, lse_ref = oracle.attention_decode_paged(to_f64(q, dtype), to_f64(kp, dtype), to_f64(vp, dtype), table,
                                                   scale, lens)
    check(og.t.cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref, "fp32", f"guarded paged decode page {ps}")


def test_shard_blocks_and_merge_stay_inside():
    fa = fa_mod()
    from exact_tiled_attention_47_b200.sharded import shard_range
    B, Hq, Hkv, Nk, D, dtype, R, S = 3, 8, 2, 1500, 128, "bf16", 4, 8
    scale = 1 / math.sqrt(D)
    lens = [1500, 374, 0]
    q, k, v = si.decode_gqa_inputs(7400, B, Nk, Hq, Hkv, D, dtype)
    qd = to_device(q, dtype)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    pb = fa.fa_decode_part_bytes(B, Hq, D)
    parts = Guarded((R * pb // 4,), torch.float32)
    nb = fa.fa_decode_workspace_bytes(B, Hq, D, S)
    wg = Guarded((nb,), torch.uint8)
    for r in range(R):
        off, n = shard_range(Nk, R, r)
        ks = to_device(np.ascontiguousarray(k[:, off:off + n]), dtype)
        vs = to_device(np.ascontiguousarray(v[:, off:off + n]), dtype)
        blk = parts.t[r * pb // 4:(r + 1) * pb // 4]
        assert fa.fa_decode_splitkv_shard(qd, ks, vs, blk, B, Hq, Hkv, n, off, Nk, D, scale, S, sl, wg.t, nb) == 0
    og = Guarded((B, 1, Hq, D), torch.float32)
    lg = Guarded((B, Hq), torch.float32)
    assert fa.fa_decode_merge(parts.t, R, B, Hq, D, og.t, lg.t) == 0
    finish(fa, parts, wg, og, lg)
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale, lens)
    check(og.t.cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref, "fp32", "guarded shard merge")


@pytest.mark.parametrize("Nq,Nk,D,causal,gdt", [(333, 200, 128, True, "fp32"), (200, 333, 64, True, "bf16"),
                                                (130, 130, 64, False, "fp32")])
def test_backward_writes_stay_inside(Nq, Nk, D, causal, gdt):
    fa = fa_mod()
    B, H, dtype, scale = 2, 2, "bf16", 0.125
    q, k, v = si.dense_qkv(7500 + Nq + D, B, Nq, Nk, H, D, dtype)
    do = si.batched(7500 + Nq + D, 3, B, (Nq, H, D), dtype)
    qd, kd, vd, dod = (to_device(t, dtype) for t in (q, k, v, do))
    o, lse = fa.attention(qd, kd, vd, causal=causal, scale=scale)
    gt = torch_dtype(gdt)
    dq, dk, dv = Guarded((B, Nq, H, D), gt), Guarded((B, Nk, H, D), gt), Guarded((B, Nk, H, D), gt)
    nb = fa.fa_bwd_workspace_bytes(B, H, Nq)
    wg = Guarded((nb,), torch.uint8)
    st = fa.fa_bwd(qd, kd, vd, o, dod, lse, dq.t, dk.t, dv.t, B, H, Nq, Nk, D, scale, causal, wg.t, nb)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    finish(fa, dq, dk, dv, wg)
    refs = oracle.attention_dense_backward(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype),
                                           to_f64(do, dtype), scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        gn = g.t.float().cpu().numpy()
        m = max(np.abs(r).max(), 1e-6)
        assert np.abs(gn - r).max() / m <= 2e-2, name


def test_noalloc_decode_writes_stay_inside():
    fa = fa_mod()
    B, H, Nk, D, dtype, S = 2, 4, 900, 128, "bf16", 16
    scale = 1 / math.sqrt(D)
    q, k, v = si.decode_inputs(7600, B, Nk, H, D, dtype)
    qd, kd, vd = (to_device(t, dtype) for t in (q, k, v))
    og = Guarded((B, 1, H, D), torch.float32)
    lg = Guarded((B, H), torch.float32)
    assert fa.fa_decode_splitkv_noalloc(qd, kd, vd, og.t, lg.t, B, H, Nk, D, scale, S) == fa.FA_OK
    finish(fa, og, lg)
    o_ref, lse_ref = oracle.attention_decode(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale)
    check(og.t.cpu().numpy(), lg.t.cpu().numpy(), o_ref, lse_ref[:, :, 0], "fp32", "guarded noalloc")


def test_masked_backward_writes_stay_inside():
    fa = fa_mod()
    lengths, H, D, dtype, prefix = [300, 1, 0, 129], 2, 128, "bf16", 50
    q, k, v, cu = si.varlen_qkv(7700, lengths, H, D, dtype)
    total = int(cu[-1])
    do = si.batch_item(7700, 3, 0, (total, H, D), dtype)
    qd, kd, vd, dod = (to_device(t, dtype) for t in (q, k, v, do))
    cut = torch.from_numpy(cu).cuda()
    o, lse = fa.attention(qd, kd, vd, scale=0.1, cu_seqlens=cut, prefix_len=prefix)
    gs = [Guarded((total, H, D), torch.float32) for _ in range(3)]
    nb = fa.fa_bwd_workspace_bytes(1, H, total)
    wg = Guarded((nb,), torch.uint8)
    st = fa.fa_bwd_masked(qd, kd, vd, o, dod, lse, gs[0].t, gs[1].t, gs[2].t, len(lengths), H, total, total, D, 0.1,
                          1, prefix, cut, wg.t, nb)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    finish(fa, *gs, wg)
    refs = oracle.attention_varlen_backward(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), to_f64(do, dtype),
                                            cu, 0.1, True, prefix)
    for name, g, r in zip(("dq", "dk", "dv"), gs, refs):
        m = max(np.abs(r).max(), 1e-6)
        assert np.abs(g.t.cpu().numpy() - r).max() / m <= 2e-2, name
