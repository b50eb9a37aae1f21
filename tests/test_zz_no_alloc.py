"""The decode entry point for callers that cannot allocate device memory.

fa_decode_splitkv_noalloc serves callers that cannot obtain a workspace at call time (for example
an engine that reserves all device memory at start-up and forbids later allocation): it keeps the
split partials in the library's fixed per-GPU scratch array.  These tests check, through the C ABI,
that it returns what fa_decode_splitkv (caller workspace) returns -- on two calls in a row, the
second on different inputs, so leftovers in the shared array from the first call cannot leak into
the second -- and that problems too large for the fixed array are refused before any launch.
This file is named so that pytest collects it last.
"""
import math

import numpy as np
import pytest

import seeded_inputs as si
from parity import LSE_TOL, O_TOL, to_device

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
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, H, Nk, D, S = 8, 16, 3000, 128, 16
    scale = 1.0 / math.sqrt(D)
    fa.fa_device_status(clear=True)
    for call, seed in enumerate((41, 42)):
        q, k, v = (to_device(t, "bf16") for t in si.decode_inputs(seed, B, Nk, H, D, "bf16"))
        o_ref, lse_ref = fa.decode(q, k, v, scale=scale, num_splits=S, out_dtype=torch.float32)
        o = torch.empty((B, 1, H, D), dtype=torch.float32, device="cuda")
        lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        st = fa.fa_decode_splitkv_noalloc(q, k, v, o, lse, B, H, Nk, D, scale, S)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        torch.cuda.synchronize()
        assert fa.fa_device_status(clear=True) == 0
        do = torch.max(torch.abs(o - o_ref)).item()
        dl = torch.max(torch.abs(lse - lse_ref)).item()
        assert do <= O_TOL and dl <= LSE_TOL, (call, do, dl)
        assert np.isfinite(o.cpu().numpy()).all()
