"""Failure detection on the GPU without a fault: a kernel's bounded wait on a barrier that nothing
arrives on ends with FA_ERR_TIMEOUT in the device status word, and the context stays usable."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from parity import check, to_device, to_f64

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


def test_bounded_wait_times_out_and_context_survives():
    import exact_tiled_attention_47_b200 as fa
    st, waited_ms = fa.fa_selftest_wait_timeout()
    assert st == fa.FA_OK
    assert 900 <= waited_ms <= 10000, waited_ms          # the wait limit is one second
    assert fa.fa_device_status(clear=True) == fa.FA_ERR_TIMEOUT
    assert fa.fa_device_status(clear=True) == fa.FA_OK   # cleared
    # the same context still computes correctly
    q, k, v = si.dense_qkv(4300, 1, 200, 200, 2, 64, "bf16")
    qt, kt, vt = (to_device(t, "bf16") for t in (q, k, v))
    o, lse = fa.attention(qt, kt, vt, causal=True, scale=0.125, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.fa_device_status(clear=True) == 0
    o_ref, lse_ref = oracle.attention_dense(to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16"), 0.125, True)
    check(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fp32", "after the timeout")
