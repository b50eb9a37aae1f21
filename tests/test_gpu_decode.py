"""Decode (Nq = 1, split-KV + LSE combine) parity against the fp64 oracle (GPU only)."""
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


def run(B, H, Nk, D, dtype, S, out, seed, scale=None):
    import exact_tiled_attention_47_b200 as fa
    scale = 1 / math.sqrt(D) if scale is None else scale
    q, k, v = si.decode_inputs(seed, B, Nk, H, D, dtype)
    o, lse = fa.decode(to_device(q, dtype), to_device(k, dtype), to_device(v, dtype), scale=scale,
                       num_splits=S, out_dtype=torch_dtype(out))
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_decode(to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype), scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref[:, :, 0], out,
          f"decode B{B} H{H} Nk{Nk} D{D} S{S}")
    return o, lse


CASES = [
    # B, H, Nk, D, dtype, splits, out
    (3, 4, 1000, 128, "bf16", 16, "fp32"),
    (3, 4, 1000, 128, "bf16", 1, "fp32"),
    (3, 4, 1000, 128, "bf16", 7, "bf16"),
    (2, 3, 77, 64, "fp16", 16, "fp32"),
    (2, 3, 5, 64, "fp16", 16, "fp16"),     # more splits than keys: empty splits
    (1, 1, 1, 128, "bf16", 16, "fp32"),
    (2, 2, 4099, 64, "bf16", 128, "fp32"),
    (4, 8, 2048, 128, "fp16", 3, "fp32"),
]


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}h{c[1]}n{c[2]}d{c[3]}{c[4]}s{c[5]}{c[6]}" for c in CASES])
def test_decode_cases(case):
    B, H, Nk, D, dtype, S, out = case
    run(B, H, Nk, D, dtype, S, out, seed=500 + Nk + S)


def test_split_count_invariance():
    import exact_tiled_attention_47_b200 as fa
    q, k, v = si.decode_inputs(21, 4, 3000, 8, 128, "bf16")
    args = [to_device(t, "bf16") for t in (q, k, v)]
    o1, l1 = fa.decode(*args, num_splits=1, out_dtype=torch.float32)
    o16, l16 = fa.decode(*args, num_splits=16, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(o1 - o16)).item() <= 1e-5
    assert torch.max(torch.abs(l1 - l16)).item() <= 1e-5


def test_decode_full_config():
    c = si.CONFIGS["decode"]
    import exact_tiled_attention_47_b200 as fa
    q, k, v = si.decode_inputs(c["seed"], c["B"], c["Nk"], c["H"], c["D"], c["dtype"])
    o, lse = fa.decode(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), scale=c["scale"],
                       num_splits=c["num_splits"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    on, ln = o.cpu().numpy(), lse.cpu().numpy()
    rng = np.random.default_rng(3)
    for b in sorted(set([0, c["B"] - 1] + list(rng.integers(0, c["B"], 6)))):
        for h in range(c["H"]):
            ro, rl = oracle.attention_head(to_f64(q[b, :, h], "bf16"), to_f64(k[b, :, h], "bf16"),
                                           to_f64(v[b, :, h], "bf16"), c["scale"])
            check(on[b, 0, h][None], ln[b, h][None], ro, rl, "fp32", f"decode full b{b} h{h}")
