"""GPU parity of the prefix mask (fa_fwd_prefix) against the fp64 oracle.

The prefix-LM reading of the prefix mask named on the Hugging Face page ("原因分析", item 1): causal,
except that the first prefix_len keys of a sequence are visible to all its queries.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
from parity import check, to_device, to_f64, torch_dtype

pytestmark = pytest.mark.gpu


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


CASES = [
    # B, Nq, Nk, H, D, dtype, scale, prefix
    (2, 300, 300, 3, 64, "fp16", 0.1, 100),
    (1, 384, 384, 2, 128, "bf16", 1 / math.sqrt(128), 200),
    (2, 200, 333, 2, 64, "bf16", 0.125, 150),    # Nq < Nk
    (2, 333, 200, 2, 128, "bf16", 0.125, 50),    # Nq > Nk: rows before the diagonal see the prefix
    (1, 1024, 1024, 2, 64, "bf16", 0.125, 700),  # prefix ends inside a key block
    (1, 1024, 1024, 2, 128, "bf16", 0.09, 512),  # prefix ends on a block boundary
    (1, 257, 257, 2, 128, "fp16", 0.09, 1),
    (1, 17, 17, 1, 64, "bf16", 0.125, 16),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[1]}x{c[2]}d{c[4]}{c[5]}p{c[7]}" for c in CASES])
def test_prefix_dense(case):
    B, Nq, Nk, H, D, dtype, scale, prefix = case
    fa = fa_mod()
    q, k, v = si.dense_qkv(3000 + Nq + 7 * Nk + prefix, B, Nq, Nk, H, D, dtype)
    qt, kt, vt = (to_device(t, dtype) for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, scale=scale, prefix_len=prefix, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale,
                                            causal=True, prefix=prefix)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", f"prefix {case}")


@pytest.mark.parametrize("D", [64, 128])
def test_prefix_limits_match_causal_and_full(D):
    fa = fa_mod()
    B, N, H = 1, 600, 2
    q, k, v = si.dense_qkv(3100 + D, B, N, N, H, D, "bf16")
    qt, kt, vt = (to_device(t, "bf16") for t in (q, k, v))
    o0, l0 = fa.attention(qt, kt, vt, scale=0.1, prefix_len=0, out_dtype=torch.float32)
    oc, lc = fa.attention(qt, kt, vt, scale=0.1, causal=True, out_dtype=torch.float32)
    of_, lf = fa.attention(qt, kt, vt, scale=0.1, prefix_len=N + 5, out_dtype=torch.float32)
    on, ln = fa.attention(qt, kt, vt, scale=0.1, causal=False, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o0, oc) and torch.equal(l0, lc)
    assert torch.equal(of_, on) and torch.equal(lf, ln)


@pytest.mark.parametrize("D,dtype", [(64, "fp16"), (128, "bf16")])
def test_prefix_varlen(D, dtype):
    fa = fa_mod()
    lengths = [1, 17, 128, 129, 300, 513, 64, 255]
    H, scale, prefix = 3, 0.1, 100
    q, k, v, cu = si.varlen_qkv(3200 + D, lengths, H, D, dtype)
    qt, kt, vt = (to_device(t, dtype) for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, scale=scale, cu_seqlens=torch.from_numpy(cu).cuda(), prefix_len=prefix,
                          out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_varlen(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), cu, scale,
                                             causal=True, prefix=prefix)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "prefix varlen")


def test_prefix_zero_query_closed_form():
    # Q = 0: O_i is the mean of the visible V rows, LSE_i = ln(min(Nk, max(prefix, i + 1)))
    fa = fa_mod()
    N, H, D, prefix = 400, 1, 64, 150
    _, k, v = si.dense_qkv(3300, 1, N, N, H, D, "bf16")
    qt = torch.zeros((1, N, H, D), device="cuda", dtype=torch.bfloat16)
    kt, vt = to_device(k, "bf16"), to_device(v, "bf16")
    o, lse = fa.attention(qt, kt, vt, scale=0.125, prefix_len=prefix, out_dtype=torch.float32)
    torch.cuda.synchronize()
    vf = to_f64(v, "bf16")[0, :, 0]
    vis = np.minimum(N, np.maximum(prefix, np.arange(N) + 1))
    o_ref = np.stack([vf[:c].mean(axis=0) for c in vis])
    check(o[0, :, 0].cpu().numpy(), lse[0, 0].cpu().numpy(), o_ref, np.log(vis.astype(np.float64)), "fp32",
          "prefix Q=0")


def test_prefix_full_size_sampled():
    fa = fa_mod()
    c = si.CONFIGS["prefill_d64"]
    B, N, H, D, prefix = c["B"], c["Nq"], c["H"], c["D"], 3000
    q, k, v = si.dense_qkv(c["seed"], B, N, N, H, D, c["dtype"])
    qt, kt, vt = (to_device(t, c["dtype"]) for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, scale=c["scale"], prefix_len=prefix, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    rng = np.random.default_rng(321)
    fixed = [0, 1, 127, 128, prefix - 1, prefix, prefix + 1, N // 2, N - 1]
    rows = np.unique(np.concatenate([fixed, rng.integers(0, N, size=30)]))
    for b, h in [(0, 0), (B - 1, H - 1), (1, 7)]:
        ro, rl = oracle.attention_rows(to_f64(q[b, :, h], c["dtype"]), to_f64(k[b, :, h], c["dtype"]),
                                       to_f64(v[b, :, h], c["dtype"]), rows, c["scale"], True, prefix=prefix)
        check(o[b, :, h].cpu().numpy()[rows], lse[b, h].cpu().numpy()[rows], ro, rl, "fp32",
              f"prefix full b{b} h{h}")
