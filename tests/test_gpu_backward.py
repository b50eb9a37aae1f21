"""GPU gradients (fa_bwd: dQ, dK, dV) against the fp64 backward oracle.

Tolerance: P and dS are rounded to the 16-bit input type before their tensor-core products (relative
2^-9 for bf16) and the row term rowsum(dO * O) uses the 16-bit forward output, so each gradient
carries a relative error of order 1e-3 of its largest magnitude; the bound below is 2e-2 of that
magnitude, which a wrong mask, index or transposed operand exceeds by far.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import to_device, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
REL_TOL = 2e-2


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


def run_bwd(B, Nq, Nk, H, D, dtype, scale, causal, seed, grad_dtype=torch.float32):
    import exact_tiled_attention_47_b200 as fa
    q, k, v = si.dense_qkv(seed, B, Nq, Nk, H, D, dtype)
    do = si.batched(seed, 3, B, (Nq, H, D), dtype)  # tensor id 3: the upstream gradient
    qt, kt, vt, dot = (to_device(t, dtype) for t in (q, k, v, do))
    o, lse = fa.attention(qt, kt, vt, causal=causal, scale=scale)  # O in the input type, as training uses
    dq, dk, dv = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=causal, scale=scale, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    rq, rk, rv = oracle.attention_dense_backward(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype),
                                                 to_f64(do, dtype), scale, causal)
    errs = []
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        gn = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(gn).all(), name
        m = max(np.abs(r).max(), 1e-6)
        e = np.abs(gn - r).max() / m
        errs.append(e)
        print(f"{name}: max|ref| {m:.3e}  max|err|/max|ref| {e:.2e}")
        assert e <= REL_TOL, (name, e)
    return errs


CASES = [
    # B, Nq, Nk, H, D, dtype, scale, causal
    (1, 128, 128, 1, 64, "bf16", 0.125, False),
    (2, 300, 300, 2, 64, "fp16", 0.1, True),
    (1, 256, 256, 2, 128, "bf16", 1 / math.sqrt(128), True),
    (2, 200, 333, 2, 64, "bf16", 0.125, True),     # Nq < Nk
    (2, 333, 200, 2, 128, "bf16", 0.125, True),    # Nq > Nk: leading rows see no key
    (1, 384, 384, 2, 128, "bf16", 0.09, False),
    (1, 1024, 1024, 1, 64, "bf16", 0.125, True),
    (1, 17, 17, 1, 128, "fp16", 0.125, False),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[1]}x{c[2]}h{c[3]}d{c[4]}{c[5]}{'c' if c[7] else 'n'}" for c in CASES])
def test_backward_cases(case):
    B, Nq, Nk, H, D, dtype, scale, causal = case
    run_bwd(B, Nq, Nk, H, D, dtype, scale, causal, seed=4000 + Nq + 7 * Nk + D)


def test_backward_bf16_gradients():
    run_bwd(1, 256, 256, 2, 64, "bf16", 0.125, True, seed=4100, grad_dtype=torch.bfloat16)


def test_backward_deterministic():
    import exact_tiled_attention_47_b200 as fa
    q, k, v = si.dense_qkv(4200, 1, 300, 300, 2, 64, "bf16")
    do = si.batched(4200, 3, 1, (300, 2, 64), "bf16")
    qt, kt, vt, dot = (to_device(t, "bf16") for t in (q, k, v, do))
    o, lse = fa.attention(qt, kt, vt, causal=True)
    g1 = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=True, grad_dtype=torch.float32)
    g2 = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=True, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_backward_full_size_sampled():
    import exact_tiled_attention_47_b200 as fa
    c = si.CONFIGS["prefill_d64"]
    B, N, H, D, dt, scale = c["B"], c["Nq"], c["H"], c["D"], c["dtype"], c["scale"]
    q, k, v = si.dense_qkv(c["seed"], B, N, N, H, D, dt)
    do = si.batched(c["seed"], 3, B, (N, H, D), dt)
    qt, kt, vt, dot = (to_device(t, dt) for t in (q, k, v, do))
    o, lse = fa.attention(qt, kt, vt, causal=True, scale=scale)
    dq, dk, dv = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=True, scale=scale, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    # identities that hold at any size: dS rows sum to zero, P rows sum to one
    dof = dot.float()
    assert (dk.sum(dim=1).abs().max() / dk.abs().max()).item() < 2e-2
    assert ((dv.sum(dim=1) - dof.sum(dim=1)).abs().max() / dof.sum(dim=1).abs().max()).item() < 2e-2
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095, N - 1], rng.integers(0, N, 10)]))
    for b, h in [(0, 0), (B - 1, H - 1)]:
        f = lambda x: to_f64(x[b, :, h], dt)
        rq, rk, rv = oracle.attention_rows_backward(f(q), f(k), f(v), f(do), scale, rows, rows, causal=True)
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            gn = g[b, :, h].cpu().numpy().astype(np.float64)[rows]
            m = max(np.abs(r).max(), 1e-6)
            e = np.abs(gn - r).max() / m
            print(f"full b{b} h{h} {name}: max|ref| {m:.3e} rel err {e:.2e}")
            assert e <= REL_TOL, (name, e)


# ------------------------------------------------------------------------------------------------
# the prefix-LM mask and packed varlen sequences (fa_bwd_masked)


def _grad_errors(got, refs):
    errs = []
    for name, g, r in zip(("dq", "dk", "dv"), got, refs):
        gn = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(gn).all(), name
        m = max(np.abs(r).max(), 1e-6)
        e = np.abs(gn - r).max() / m
        print(f"{name}: max|ref| {m:.3e} rel err {e:.2e}")
        errs.append(e)
        assert e <= REL_TOL, (name, e)
    return errs


PREFIX_CASES = [
    # B, Nq, Nk, H, D, dtype, prefix
    (2, 300, 300, 2, 64, "bf16", 77),
    (1, 513, 513, 2, 128, "fp16", 200),
    (2, 200, 333, 2, 64, "bf16", 150),   # Nq < Nk, prefix inside the first key tile
    (1, 256, 256, 1, 128, "bf16", 300),  # prefix past the end: no mask at all
    (1, 384, 384, 2, 64, "bf16", 130),   # prefix ending inside the second key tile
]


@pytest.mark.parametrize("case", PREFIX_CASES, ids=[f"{c[1]}x{c[2]}d{c[4]}p{c[6]}" for c in PREFIX_CASES])
def test_backward_prefix_mask(case):
    import exact_tiled_attention_47_b200 as fa
    B, Nq, Nk, H, D, dtype, prefix = case
    scale = 1 / math.sqrt(D)
    seed = 4300 + Nq + Nk + prefix
    q, k, v = si.dense_qkv(seed, B, Nq, Nk, H, D, dtype)
    do = si.batched(seed, 3, B, (Nq, H, D), dtype)
    qt, kt, vt, dot = (to_device(t, dtype) for t in (q, k, v, do))
    o, lse = fa.attention(qt, kt, vt, scale=scale, prefix_len=prefix)
    grads = fa.attention_backward(qt, kt, vt, o, lse, dot, scale=scale, prefix_len=prefix, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    refs = oracle.attention_dense_backward(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), to_f64(do, dtype),
                                           scale, True, prefix)
    _grad_errors(grads, refs)


VARLEN_CASES = [
    # lengths, H, D, dtype, causal, prefix
    ([1, 300, 0, 129, 511], 2, 64, "fp16", False, 0),
    ([1, 300, 0, 129, 511], 2, 64, "fp16", True, 0),
    ([700, 17, 256], 2, 128, "bf16", True, 0),
    ([700, 17, 256], 2, 128, "bf16", False, 0),
    ([260, 5, 400], 2, 64, "bf16", True, 100),  # prefix per sequence
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=[f"v{len(c[0])}d{c[2]}c{int(c[4])}p{c[5]}" for c in VARLEN_CASES])
def test_backward_varlen(case):
    import exact_tiled_attention_47_b200 as fa
    lengths, H, D, dtype, causal, prefix = case
    scale = 0.1
    seed = 4400 + D + 3 * prefix + int(causal)
    q, k, v, cu = si.varlen_qkv(seed, lengths, H, D, dtype)
    total = int(cu[-1])
    do = si.batch_item(seed, 3, 0, (total, H, D), dtype)
    qt, kt, vt, dot = (to_device(t, dtype) for t in (q, k, v, do))
    cut = torch.from_numpy(cu).cuda()
    pl = prefix if prefix else None
    o, lse = fa.attention(qt, kt, vt, causal=causal, scale=scale, cu_seqlens=cut, prefix_len=pl)
    grads = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=causal, scale=scale, cu_seqlens=cut, prefix_len=pl,
                                  grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    refs = oracle.attention_varlen_backward(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), to_f64(do, dtype),
                                            cu, scale, causal or prefix > 0, prefix)
    _grad_errors(grads, refs)


def test_backward_varlen_equals_dense_per_sequence():
    """Packed varlen gradients equal each sequence's dense gradients computed alone (bit for bit)."""
    import exact_tiled_attention_47_b200 as fa
    lengths, H, D = [130, 7, 260], 2, 64
    q, k, v, cu = si.varlen_qkv(4500, lengths, H, D, "bf16")
    total = int(cu[-1])
    do = si.batch_item(4500, 3, 0, (total, H, D), "bf16")
    qt, kt, vt, dot = (to_device(t, "bf16") for t in (q, k, v, do))
    cut = torch.from_numpy(cu).cuda()
    o, lse = fa.attention(qt, kt, vt, causal=True, scale=0.1, cu_seqlens=cut)
    g = fa.attention_backward(qt, kt, vt, o, lse, dot, causal=True, scale=0.1, cu_seqlens=cut, grad_dtype=torch.float32)
    for b in range(len(lengths)):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        sl = lambda x: x[s0:s1][None]
        od, ld = fa.attention(sl(qt), sl(kt), sl(vt), causal=True, scale=0.1)
        gd = fa.attention_backward(sl(qt), sl(kt), sl(vt), od, ld, sl(dot), causal=True, scale=0.1,
                                   grad_dtype=torch.float32)
        torch.cuda.synchronize()
        for a, bb in zip(g, gd):
            assert torch.equal(a[s0:s1], bb[0])
