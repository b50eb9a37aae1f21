"""Prefill parity: the sm_100a kernels through the C ABI against the fp64 oracle (GPU only).

Small cases compare every output element; the full-size workloads compare sampled rows that the
oracle evaluates one by one.  Inputs come from the seeded generator, bit-identical on both sides.
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


def fa_mod():
    import exact_tiled_attention_47_b200 as fa
    return fa


def run_dense(B, Nq, Nk, H, D, dtype, scale, causal, out_dtype, seed):
    fa = fa_mod()
    q, k, v = si.dense_qkv(seed, B, Nq, Nk, H, D, dtype)
    qt, kt, vt = (to_device(t, dtype) for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, causal=causal, scale=scale, out_dtype=torch_dtype(out_dtype))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype),
                                            scale, causal)
    return check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, out_dtype,
                 f"B{B} Nq{Nq} Nk{Nk} H{H} D{D} {dtype} causal={causal} out={out_dtype}")


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_config(causal):
    c = si.CONFIGS["tiny"]
    run_dense(c["B"], c["Nq"], c["Nk"], c["H"], c["D"], c["dtype"], c["scale"], causal, "fp32", c["seed"])


CASES = [
    # B, Nq, Nk, H, D, dtype, scale, causal, out
    (1, 256, 256, 2, 128, "bf16", 1 / math.sqrt(128), False, "fp32"),
    (1, 256, 256, 2, 128, "bf16", 1 / math.sqrt(128), True, "fp32"),
    (2, 300, 300, 3, 64, "fp16", 0.1, True, "fp32"),
    (2, 300, 300, 3, 64, "fp16", 0.1, False, "fp32"),
    (1, 1, 1, 1, 64, "bf16", 0.125, False, "fp32"),
    (1, 1, 1, 1, 128, "bf16", 0.125, True, "fp32"),
    (1, 17, 17, 2, 64, "bf16", 0.125, True, "fp32"),
    (1, 127, 127, 2, 128, "fp16", 0.09, True, "fp32"),
    (1, 129, 129, 2, 128, "bf16", 0.09, True, "fp32"),
    (2, 200, 333, 2, 64, "bf16", 0.125, True, "fp32"),    # Nq < Nk, bottom-right causal
    (2, 333, 200, 2, 128, "bf16", 0.125, True, "fp32"),   # Nq > Nk: leading rows see no key
    (1, 100, 700, 2, 128, "bf16", 0.125, False, "fp32"),
    (2, 384, 384, 4, 128, "bf16", 1 / math.sqrt(128), True, "bf16"),
    (2, 256, 256, 4, 64, "fp16", 0.125, False, "fp16"),
    (1, 1024, 1024, 2, 128, "bf16", 1 / math.sqrt(128), True, "fp32"),
    (1, 1024, 1024, 2, 64, "bf16", 0.125, False, "fp32"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}h{c[3]}d{c[4]}{c[5]}{'c' if c[7] else 'n'}{c[8]}" for c in CASES])
def test_dense_cases(case):
    B, Nq, Nk, H, D, dtype, scale, causal, out = case
    run_dense(B, Nq, Nk, H, D, dtype, scale, causal, out, seed=1000 + Nq + 7 * Nk + D)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,dtype", [(64, "fp16"), (128, "bf16")])
def test_varlen_small(causal, D, dtype):
    fa = fa_mod()
    lengths = [1, 17, 128, 129, 300, 513, 64, 255]
    H, scale = 3, 0.1
    q, k, v, cu = si.varlen_qkv(77, lengths, H, D, dtype)
    qt, kt, vt = (to_device(t, dtype) for t in (q, k, v))
    cut = torch.from_numpy(cu).cuda()
    o, lse = fa.attention(qt, kt, vt, causal=causal, scale=scale, cu_seqlens=cut, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_varlen(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), cu,
                                             scale, causal)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "varlen small")


def test_varlen_matches_dense_per_sequence():
    """Packed varlen equals running each sequence on its own in dense mode (key padding semantics)."""
    fa = fa_mod()
    lengths = [130, 7, 260]
    H, D = 2, 64
    q, k, v, cu = si.varlen_qkv(5, lengths, H, D, "fp16")
    qt, kt, vt = (to_device(t, "fp16") for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, scale=0.1, cu_seqlens=torch.from_numpy(cu).cuda(),
                          out_dtype=torch.float32)
    for b, L in enumerate(lengths):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        od, ld = fa.attention(qt[s0:s1][None], kt[s0:s1][None], vt[s0:s1][None], scale=0.1,
                              out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(od[0], o[s0:s1])
        assert torch.equal(ld[0], lse[:, s0:s1])


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_closed_form(causal):
    """Q = 0: every visible key has score 0, so O is the mean of the visible V rows, LSE = ln(count)."""
    fa = fa_mod()
    B, N, H, D = 1, 300, 2, 128
    _, k, v = si.dense_qkv(9, B, N, N, H, D, "bf16")
    qt = torch.zeros((B, N, H, D), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.attention(qt, to_device(k, "bf16"), to_device(v, "bf16"), causal=causal, scale=0.125,
                          out_dtype=torch.float32)
    vf = to_f64(v, "bf16")
    cnt = np.arange(1, N + 1) if causal else np.full(N, N)
    csum = np.cumsum(vf, axis=1)
    mean = csum / cnt[None, :, None, None] if causal else np.broadcast_to(vf.mean(axis=1, keepdims=True), vf.shape)
    lse_ref = np.broadcast_to(np.log(cnt)[None, None, :], (B, H, N))
    check(o.cpu().numpy(), lse.cpu().numpy(), mean, lse_ref, "fp32", "Q=0")


def test_causal_row_zero_is_first_value_row():
    fa = fa_mod()
    B, N, H, D = 2, 256, 4, 64
    q, k, v = si.dense_qkv(11, B, N, N, H, D, "bf16")
    o, lse = fa.attention(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), causal=True,
                          scale=0.125, out_dtype=torch.float32)
    vf, qf, kf = to_f64(v, "bf16"), to_f64(q, "bf16"), to_f64(k, "bf16")
    on = o.cpu().numpy()
    # a single visible key: O_0 = V_0 up to fp32 rounding of the one weight (exact in the oracle)
    np.testing.assert_allclose(on[:, 0], vf[:, 0], rtol=1e-6, atol=1e-7)
    exp = 0.125 * np.einsum("bhd,bhd->bh", qf[:, 0], kf[:, 0])
    assert np.max(np.abs(lse.cpu().numpy()[:, :, 0] - exp)) <= 1e-3


def test_deterministic_bitwise():
    fa = fa_mod()
    q, k, v = si.dense_qkv(12, 2, 640, 640, 4, 128, "bf16")
    args = [to_device(t, "bf16") for t in (q, k, v)]
    o1, l1 = fa.attention(*args, causal=True)
    o2, l2 = fa.attention(*args, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_cu_seqlens_is_reported_not_run():
    """A decreasing cu_seqlens is detected on the device: its tiles are skipped, status is set."""
    fa = fa_mod()
    H, D, total = 2, 64, 300
    qt = torch.zeros((total, H, D), dtype=torch.float16, device="cuda")
    cu = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device="cuda")
    fa.fa_device_status(clear=True)
    o, lse = fa.attention(qt, qt, qt, scale=0.1, cu_seqlens=cu, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_CU_SEQLENS


# ------------------------------------------------------------------------------------------------
# full-size workloads, sampled rows


def _sample_rows(N, rng, n=48):
    fixed = [0, 1, 63, 64, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1]
    rnd = rng.integers(0, N, size=n - len(fixed))
    return np.unique(np.clip(np.concatenate([fixed, rnd]), 0, N - 1))


@pytest.mark.parametrize("name", ["prefill_d64", "prefill_d128"])
@pytest.mark.parametrize("out", ["fp32", "bf16"])
def test_full_size_sampled(name, out):
    fa = fa_mod()
    c = si.CONFIGS[name]
    B, N, H, D = c["B"], c["Nq"], c["H"], c["D"]
    q, k, v = si.dense_qkv(c["seed"], B, N, N, H, D, c["dtype"])
    qt, kt, vt = (to_device(t, c["dtype"]) for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, causal=c["causal"], scale=c["scale"], out_dtype=torch_dtype(out))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    rng = np.random.default_rng(123)
    pairs = {(0, 0), (B - 1, H - 1)} | {(int(rng.integers(B)), int(rng.integers(H))) for _ in range(4)}
    for b, h in sorted(pairs):
        rows = _sample_rows(N, rng)
        ob = o[b, :, h].float().cpu().numpy()[rows]
        lb = lse[b, h].cpu().numpy()[rows]
        ro, rl = oracle.attention_rows(to_f64(q[b, :, h], c["dtype"]), to_f64(k[b, :, h], c["dtype"]),
                                       to_f64(v[b, :, h], c["dtype"]), rows, c["scale"], c["causal"])
        check(ob, lb, ro, rl, out, f"{name} b{b} h{h}")
    # every output finite, every LSE finite (no row is fully masked in these workloads)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_varlen_full_config():
    fa = fa_mod()
    inp = si.config_inputs("varlen")
    c = inp["cfg"]
    dt = c["dtype"]
    qt, kt, vt = (to_device(inp[x], dt) for x in ("q", "k", "v"))
    cu = inp["cu_seqlens"]
    o, lse = fa.attention(qt, kt, vt, causal=False, scale=c["scale"], cu_seqlens=torch.from_numpy(cu).cuda(),
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    on, ln = o.cpu().numpy(), lse.cpu().numpy()
    qf, kf, vf = (to_f64(inp[x], dt) for x in ("q", "k", "v"))
    rng = np.random.default_rng(7)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        h = int(rng.integers(c["H"]))
        ro, rl = oracle.attention_head(qf[s0:s1, h], kf[s0:s1, h], vf[s0:s1, h], c["scale"])
        check(on[s0:s1, h], ln[h, s0:s1], ro, rl, "fp32", f"varlen seq {b} head {h}")


def test_partial_last_head_group():
    """Work units run longest-first inside groups of heads whose K/V take about 64 MB.  With 65536 keys
    of D = 128 a head's K/V is 32 MB, so two heads form a group and the third head is a group of its
    own: the last, partial group's units must still all be computed (sampled rows of every head)."""
    fa = fa_mod()
    B, N, H, D, dt, scale = 1, 65536, 3, 128, "bf16", 1 / math.sqrt(128)
    q, k, v = si.dense_qkv(2200, B, N, N, H, D, dt)
    o, lse = fa.attention(*(to_device(t, dt) for t in (q, k, v)), causal=True, scale=scale, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    rows = np.array([0, 1, 255, 256, 30000, N - 257, N - 256, N - 1])
    for h in range(H):
        ro, rl = oracle.attention_rows(to_f64(q[0, :, h], dt), to_f64(k[0, :, h], dt), to_f64(v[0, :, h], dt), rows,
                                       scale, True)
        check(o[0, :, h].float().cpu().numpy()[rows], lse[0, h].cpu().numpy()[rows], ro, rl, "bf16",
              f"head {h} of a partial group")


@pytest.mark.parametrize("D,dtype", [(64, "bf16"), (128, "fp16")])
def test_16bit_output_is_fp32_output_rounded(D, dtype):
    """Full tiles of a 16-bit O are written through shared memory by TMA stores, partial tiles by
    per-thread stores; both must equal the fp32 output rounded to the 16-bit type, bit for bit."""
    fa = fa_mod()
    B, N, H = 2, 700, 3  # tiles 0-4 full, tile 5 partial, per batch item
    q, k, v = si.dense_qkv(2300 + D, B, N, N, H, D, dtype)
    args = [to_device(t, dtype) for t in (q, k, v)]
    for causal in (False, True):
        o16, l16 = fa.attention(*args, causal=causal, scale=0.1)
        o32, l32 = fa.attention(*args, causal=causal, scale=0.1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(o16, o32.to(o16.dtype)), causal
        assert torch.equal(l16, l32)
