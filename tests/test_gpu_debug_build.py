"""The index-checking debug build (libfa_sm100_debug.so, FA_DEBUG) on the GPU.

With no memory checker available, the debug build is the out-of-bounds evidence: every plain global
load and store of the kernels (those no TMA descriptor bounds) checks its index against its buffer
and, instead of touching memory outside it, records FA_ERR_BOUNDS in the device status word.  These
tests run every entry point of the debug library on ragged and edge shapes and require the status
word to stay clear and the results to match the fp64 oracle.

The same build also turns off the causal block skip of the prefill and backward kernels: they walk
every key (query) block and let the mask zero the invisible ones.  Skipping a fully masked block must
change nothing -- its P is exactly zero -- so the release library's outputs and gradients must equal
the debug library's bit for bit (causal, with Nq < Nk and Nq > Nk, the prefix mask, packed varlen).
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import check, paginate, to_device, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_tiled_attention_47_b200 import build
    import exact_tiled_attention_47_b200 as fa
    build.build()
    build.build(debug=True)
    rel = fa._lib.load()
    dbg = fa._lib.load(fa.DEBUG_LIB_PATH)
    assert rel.fa_build_flags() == 0 and dbg.fa_build_flags() == fa.FA_BUILD_DEBUG
    return fa, rel, dbg


@pytest.fixture
def use_debug(libs, monkeypatch):
    """Route the package's calls to the debug library for one test (its own status word too)."""
    fa, _, dbg = libs
    monkeypatch.setattr(fa._lib, "_lib", dbg)
    fa.fa_device_status(clear=True)
    yield fa
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0, "an index check of the debug build fired"


SKIP_CASES = [
    # B, Nq, Nk, H, D, dtype, prefix (None = causal)
    (2, 700, 700, 2, 64, "bf16", None),
    (1, 513, 513, 2, 128, "fp16", None),
    (2, 200, 333, 2, 64, "bf16", None),    # Nq < Nk
    (2, 333, 200, 2, 128, "bf16", None),   # Nq > Nk: rows without keys
    (1, 640, 640, 2, 64, "bf16", 130),     # prefix mask
]


@pytest.mark.parametrize("case", SKIP_CASES, ids=[f"{c[1]}x{c[2]}d{c[4]}p{c[6]}" for c in SKIP_CASES])
def test_causal_skip_equals_mask_everything(libs, monkeypatch, case):
    fa, rel, dbg = libs
    B, Nq, Nk, H, D, dtype, prefix = case
    q, k, v = si.dense_qkv(8100 + Nq + Nk + D, B, Nq, Nk, H, D, dtype)
    args = [to_device(t, dtype) for t in (q, k, v)]
    kw = dict(causal=True, scale=1 / math.sqrt(D), out_dtype=torch.float32, prefix_len=prefix)
    o1, l1 = fa.attention(*args, **kw)  # release: fully masked blocks skipped
    torch.cuda.synchronize()
    monkeypatch.setattr(fa._lib, "_lib", dbg)
    fa.fa_device_status(clear=True)
    o2, l2 = fa.attention(*args, **kw)  # debug: every block walked and masked
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_varlen_causal_skip_equals_mask_everything(libs, monkeypatch):
    fa, rel, dbg = libs
    lengths = [300, 1, 129, 0, 700]
    q, k, v, cu = si.varlen_qkv(8200, lengths, 2, 64, "fp16")
    args = [to_device(t, "fp16") for t in (q, k, v)]
    cut = torch.from_numpy(cu).cuda()
    o1, l1 = fa.attention(*args, causal=True, scale=0.1, cu_seqlens=cut, out_dtype=torch.float32)
    torch.cuda.synchronize()
    monkeypatch.setattr(fa._lib, "_lib", dbg)
    fa.fa_device_status(clear=True)
    o2, l2 = fa.attention(*args, causal=True, scale=0.1, cu_seqlens=cut, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal,out", [(False, torch.bfloat16), (True, torch.float32)])
def test_debug_prefill_ragged(use_debug, causal, out):
    fa = use_debug
    B, Nq, Nk, H, D = 2, 333, 257, 3, 128
    q, k, v = si.dense_qkv(8300, B, Nq, Nk, H, D, "bf16")
    o, lse = fa.attention(*(to_device(t, "bf16") for t in (q, k, v)), causal=causal, scale=0.09, out_dtype=out)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"), 0.09, causal)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "bf16" if out == torch.bfloat16 else "fp32",
          "debug prefill")


def test_debug_varlen(use_debug):
    fa = use_debug
    lengths = [1, 511, 0, 260, 2]
    q, k, v, cu = si.varlen_qkv(8400, lengths, 2, 64, "fp16")
    o, lse = fa.attention(*(to_device(t, "fp16") for t in (q, k, v)), scale=0.1,
                          cu_seqlens=torch.from_numpy(cu).cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_varlen(to_f64(q, "fp16"), to_f64(k, "fp16"), to_f64(v, "fp16"), cu, 0.1)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "debug varlen")


@pytest.mark.parametrize("Hq,Hkv,D,S,lens", [(4, 4, 128, 16, None), (16, 4, 128, 8, [1000, 0, 65]),
                                             (12, 4, 64, 4, [1, 700, 129]), (3, 3, 64, 128, [5, 600, 1000])])
def test_debug_decode(use_debug, Hq, Hkv, D, S, lens):
    fa = use_debug
    B, Nk = 3, 1000
    q, k, v = si.decode_gqa_inputs(8500 + Hq + S, B, Nk, Hq, Hkv, D, "bf16")
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = fa.decode(*(to_device(t, "bf16") for t in (q, k, v)), num_splits=S, out_dtype=torch.float32,
                       seqlens_k=sl)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"),
                                                 1 / math.sqrt(D), lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "debug decode")


@pytest.mark.parametrize("Hq,Hkv,ps", [(16, 4, 16), (4, 4, 128)])
def test_debug_paged_decode(use_debug, Hq, Hkv, ps):
    fa = use_debug
    B, D, S = 3, 64, 4
    lens = [1000, 0, 65]
    Nk = -(-max(lens) // ps) * ps
    q, k, v = si.decode_gqa_inputs(8700 + ps, B, Nk, Hq, Hkv, D, "bf16")
    kp, vp, table = paginate(k, v, lens, ps, "bf16", 8701)
    o, lse = fa.decode_paged(*(to_device(t, "bf16") for t in (q, kp, vp)), torch.from_numpy(table).cuda(),
                             torch.tensor(lens, dtype=torch.int32, device="cuda"), num_splits=S,
                             out_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode_paged(to_f64(q, "bf16"), to_f64(kp, "bf16"), to_f64(vp, "bf16"), table,
                                                   1 / math.sqrt(D), lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "debug paged decode")


def test_debug_shard_and_merge(use_debug):
    fa = use_debug
    from exact_tiled_attention_47_b200.sharded import shard_range
    B, Hq, Hkv, Nk, D, R, S = 2, 8, 2, 1500, 128, 3, 8
    scale = 1 / math.sqrt(D)
    lens = [1500, 499]
    q, k, v = si.decode_gqa_inputs(8600, B, Nk, Hq, Hkv, D, "bf16")
    qd = to_device(q, "bf16")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    pf = fa.fa_decode_part_bytes(B, Hq, D) // 4
    parts = torch.empty(R * pf, dtype=torch.float32, device="cuda")
    nb = fa.fa_decode_workspace_bytes(B, Hq, D, S)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    for r in range(R):
        off, n = shard_range(Nk, R, r)
        ks = to_device(np.ascontiguousarray(k[:, off:off + n]), "bf16")
        vs = to_device(np.ascontiguousarray(v[:, off:off + n]), "bf16")
        assert fa.fa_decode_splitkv_shard(qd, ks, vs, parts[r * pf:(r + 1) * pf], B, Hq, Hkv, n, off, Nk, D, scale,
                                          S, sl, ws) == 0
    o = torch.empty((B, 1, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    assert fa.fa_decode_merge(parts, R, B, Hq, D, o, lse) == 0
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode_gqa(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"), scale, lens)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "debug shard merge")


@pytest.mark.parametrize("Nq,Nk,D,causal", [(333, 200, 128, True), (200, 333, 64, True), (130, 130, 64, False)])
def test_debug_backward(use_debug, Nq, Nk, D, causal):
    fa = use_debug
    B, H, scale = 2, 2, 0.125
    q, k, v = si.dense_qkv(8700 + Nq + D, B, Nq, Nk, H, D, "bf16")
    do = si.batched(8700 + Nq + D, 3, B, (Nq, H, D), "bf16")
    qd, kd, vd, dod = (to_device(t, "bf16") for t in (q, k, v, do))
    o, lse = fa.attention(qd, kd, vd, causal=causal, scale=scale)
    grads = fa.attention_backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    refs = oracle.attention_dense_backward(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"),
                                           to_f64(do, "bf16"), scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        m = max(np.abs(r).max(), 1e-6)
        assert np.abs(g.cpu().numpy() - r).max() / m <= 2e-2, name


def test_debug_noalloc_decode(use_debug):
    fa = use_debug
    B, H, Nk, D, S = 2, 4, 900, 128, 16
    q, k, v = si.decode_inputs(8800, B, Nk, H, D, "bf16")
    qd, kd, vd = (to_device(t, "bf16") for t in (q, k, v))
    o = torch.empty((B, 1, H, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    assert fa.fa_decode_splitkv_noalloc(qd, kd, vd, o, lse, B, H, Nk, D, 1 / math.sqrt(D), S) == 0
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_decode(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"), 1 / math.sqrt(D))
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref[:, :, 0], "fp32", "debug noalloc")


@pytest.mark.parametrize("prefix,cu", [(0, False), (90, False), (0, True)])
def test_backward_skip_equals_mask_everything(libs, monkeypatch, prefix, cu):
    """The backward's causal block skip (dQ: key blocks past the diagonal; dK/dV: query blocks before
    it) changes nothing: the release library's gradients equal the debug library's bit for bit."""
    fa, rel, dbg = libs
    scale = 0.125
    if cu:
        q, k, v, cus = si.varlen_qkv(8900, [300, 1, 129, 0, 260], 2, 64, "bf16")
        total = int(cus[-1])
        do = si.batch_item(8900, 3, 0, (total, 2, 64), "bf16")
        kw = dict(cu_seqlens=torch.from_numpy(cus).cuda())
    else:
        q, k, v = si.dense_qkv(8900 + prefix, 2, 333, 333, 2, 64, "bf16")
        do = si.batched(8900 + prefix, 3, 2, (333, 2, 64), "bf16")
        kw = {}
    if prefix:
        kw["prefix_len"] = prefix
    args = [to_device(t, "bf16") for t in (q, k, v)]
    dod = to_device(do, "bf16")

    def run():
        o, lse = fa.attention(*args, causal=True, scale=scale, **kw)
        return fa.attention_backward(*args, o, lse, dod, causal=True, scale=scale, grad_dtype=torch.float32, **kw)

    g1 = run()
    torch.cuda.synchronize()
    monkeypatch.setattr(fa._lib, "_lib", dbg)
    fa.fa_device_status(clear=True)
    g2 = run()
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
