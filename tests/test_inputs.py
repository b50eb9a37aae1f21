"""Pins of the seeded input generator (CPU only).

Both the oracle and the CUDA path consume these bits, so a mistake here would not show up as a
parity failure: the rounding to bf16/fp16 is checked against independent conversions (torch's and
numpy's), and the stream layout (per config seed, tensor id and batch item) against its stated
properties.
"""
import numpy as np
import torch

import seeded_inputs as si


def _bf16_bits_torch(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e30).astype(np.float32),
                        (rng.standard_normal(1000) * 1e-30).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38], dtype=np.float32)])
    np.testing.assert_array_equal(si.round_to_bits(x, "bf16"), _bf16_bits_torch(x))


def test_bf16_ties_round_to_even():
    # float32 values exactly halfway between two bf16 values: the low 16 bits are 0x8000
    hi = np.array([0x3F80, 0x3F81, 0x4049, 0x404A, 0xC0A0, 0xC0A1], dtype=np.uint32)
    x = ((hi << np.uint32(16)) | np.uint32(0x8000)).view(np.float32)
    got = si.round_to_bits(x, "bf16")
    expect = np.where(hi % 2 == 0, hi, hi + 1).astype(np.uint16)  # the even neighbour
    np.testing.assert_array_equal(got, expect)
    np.testing.assert_array_equal(got, _bf16_bits_torch(x))


def test_fp16_rounding_matches_torch():
    x = np.random.default_rng(12).standard_normal(50000).astype(np.float32) * 30
    t = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(si.round_to_bits(x, "fp16"), t)


def test_widening_is_exact_and_within_half_ulp():
    x = np.random.default_rng(13).standard_normal(20000).astype(np.float32)
    for dt, ulp_bits in (("bf16", 8), ("fp16", 11)):
        bits = si.round_to_bits(x, dt)
        w = si.bits_to_float(bits, dt)
        # values already in the 16-bit type widen exactly and round-trip
        np.testing.assert_array_equal(si.round_to_bits(w.astype(np.float32), dt), bits)
        err = np.abs(w - x.astype(np.float64))
        normal = np.abs(x) >= (2.0 ** -14 if dt == "fp16" else 2.0 ** -126)
        assert (err[normal] / np.abs(x[normal])).max() <= 2.0 ** -ulp_bits + 1e-12
        if dt == "fp16":  # below the normal range: half of the subnormal spacing 2^-24
            assert err[~normal].max(initial=0.0) <= 2.0 ** -25


def test_streams_per_tensor_and_batch_item():
    a = si.batch_item(5, si.K_ID, 3, (7, 2, 8), "bf16")
    np.testing.assert_array_equal(a, si.batch_item(5, si.K_ID, 3, (7, 2, 8), "bf16"))  # regenerates alone
    assert not np.array_equal(a, si.batch_item(5, si.V_ID, 3, (7, 2, 8), "bf16"))       # tensor id matters
    assert not np.array_equal(a, si.batch_item(5, si.K_ID, 4, (7, 2, 8), "bf16"))       # batch item matters
    assert not np.array_equal(a, si.batch_item(6, si.K_ID, 3, (7, 2, 8), "bf16"))       # config seed matters
    big = si.batched(5, si.K_ID, 6, (300, 4, 64), "bf16")  # large enough for the threaded path
    for b in range(6):
        np.testing.assert_array_equal(big[b], si.batch_item(5, si.K_ID, b, (300, 4, 64), "bf16"))
    vals = si.bits_to_float(big, "bf16")
    assert abs(vals.mean()) < 0.01 and abs(vals.std() - 1.0) < 0.01  # standard normal draws


def test_varlen_lengths_and_packing():
    lens = si.varlen_lengths(4, 64, 128, 2048)
    np.testing.assert_array_equal(lens, si.varlen_lengths(4, 64, 128, 2048))
    assert lens.min() >= 128 and lens.max() <= 2048
    assert set(si.varlen_lengths(1, 4000, 3, 5).tolist()) == {3, 4, 5}  # both ends inclusive
    q, k, v, cu = si.varlen_qkv(9, [3, 1, 4], 2, 8, "fp16")
    assert cu.tolist() == [0, 3, 4, 8] and cu.dtype == np.int32
    np.testing.assert_array_equal(k[3:4], si.batch_item(9, si.K_ID, 1, (1, 2, 8), "fp16"))
