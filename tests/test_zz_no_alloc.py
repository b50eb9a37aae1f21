"""The decode entry point for callers that cannot allocate device memory.

fa_decode_splitkv_noalloc serves callers that cannot obtain a workspace at call time (for example
an engine that reserves all device memory at start-up and forbids later allocation): it keeps the
split partials in the library's fixed per-GPU scratch array.  These tests check, through the C ABI,
that it returns exactly what fa_decode_splitkv (caller workspace) returns and what the fp64 oracle
gives -- on two calls in a row with different shapes, the second smaller and with empty splits, so
leftovers in the shared array from the first call would show -- and that problems too large for the
fixed array are refused before any launch.
This file is named so that pytest collects it last.
"""
import math

import pytest

import seeded_inputs as si
from parity import to_device

torch = pytest.importorskip("torch")

A = 0x100000  # 16-byte aligned fake address; only used where validation fails before any launch


@pytest.fixture(scope="module")
def fa():
    from exact_tiled_attention_47_b200 import build
    build.build()
    import exact_tiled_attention_47_b200 as fa_mod
    fa_mod._lib.load()
    return fa_mod


def test_too_large_for_the_fixed_scratch_is_refused(fa):
    B, H, D, S = 256, 64, 128, 16  # needs ~135 MB of partials, above the 32 MiB array
    assert fa.fa_decode_workspace_bytes(B, H, D, S) > fa.FA_NOALLOC_SCRATCH_BYTES
    st = fa._lib.load().fa_decode_splitkv_noalloc(A, A, A, A, A, B, H, 100, D, 0.1, S, None, 0, 0)
    assert st == fa.FA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls(fa):
    """Two calls in a row with different layouts in the shared array: the first larger (more heads,
    more splits, D = 128), the second smaller (D = 64, a cache shorter than its splits need, so most
    splits are empty).  Each must equal fa_decode_splitkv bit for bit -- the same kernels on the same
    partition -- and match the fp64 oracle within the parity tolerances."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from parity import check, to_f64
    calls = [
        # seed, B, H, Nk, D, splits, dtype
        (41, 8, 32, 4100, 128, 64, "bf16"),
        (42, 3, 5, 700, 64, 16, "fp16"),   # 700 keys, splits of at least 512: 14 empty splits
    ]
    fa.fa_device_status(clear=True)
    for seed, B, H, Nk, D, S, dt in calls:
        scale = 1.0 / math.sqrt(D)
        qb, kb, vb = si.decode_inputs(seed, B, Nk, H, D, dt)
        q, k, v = (to_device(t, dt) for t in (qb, kb, vb))
        o_ref, lse_ref = fa.decode(q, k, v, scale=scale, num_splits=S, out_dtype=torch.float32)
        o = torch.full((B, 1, H, D), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        st = fa.fa_decode_splitkv_noalloc(q, k, v, o, lse, B, H, Nk, D, scale, S)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        torch.cuda.synchronize()
        assert fa.fa_device_status(clear=True) == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), (seed, "differs from the workspace entry point")
        om, lm = oracle.attention_decode(to_f64(qb, dt), to_f64(kb, dt), to_f64(vb, dt), scale)
        check(o.cpu().numpy(), lse.cpu().numpy(), om, lm[:, :, 0], "fp32", f"noalloc call seed {seed}")
