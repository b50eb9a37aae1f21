"""Helpers for GPU-versus-oracle parity tests.

Tolerances (fixed by the target): max |O_gpu - O_ref| <= 1e-2 and max |LSE_gpu - LSE_ref| <= 1e-3
for bf16/fp16 inputs with fp32 accumulation, checked element by element.  When O is written in a
16-bit type the stored value also carries that type's rounding, so the O bound becomes
1e-2 + |O_ref| * 2^-8 (bf16, half an ulp at 8 significand bits) or 1e-2 + |O_ref| * 2^-11 (fp16).
"""
from __future__ import annotations

import numpy as np

import seeded_inputs as si

O_TOL = 1e-2
LSE_TOL = 1e-3


def torch_dtype(name):
    import torch
    return {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[name]


def to_device(bits: np.ndarray, dtype: str, device="cuda"):
    """uint16 bit patterns -> torch tensor of the 16-bit type on the device (identical bits)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch_dtype(dtype))


def to_f64(bits, dtype):
    return si.bits_to_float(bits, dtype)


def o_tolerance(o_ref: np.ndarray, out_dtype: str) -> np.ndarray:
    rel = {"fp32": 0.0, "bf16": 2.0 ** -8, "fp16": 2.0 ** -11}[out_dtype]
    return O_TOL + np.abs(o_ref) * rel


def check(o_gpu, lse_gpu, o_ref, lse_ref, out_dtype="fp32", what=""):
    """Element-wise parity; returns a small report dict and asserts the bounds."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert lse_gpu.shape == lse_ref.shape, (lse_gpu.shape, lse_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    do = np.abs(o_gpu - o_ref)
    tol = o_tolerance(o_ref, out_dtype)
    bad_o = int(np.count_nonzero(do > tol))
    inf_ref = np.isinf(lse_ref)
    assert np.array_equal(np.isinf(lse_gpu), inf_ref), f"{what}: -inf LSE pattern differs"
    assert np.all(lse_gpu[inf_ref] == lse_ref[inf_ref])
    dl = np.abs(lse_gpu[~inf_ref] - lse_ref[~inf_ref]) if np.any(~inf_ref) else np.zeros(1)
    bad_l = int(np.count_nonzero(dl > LSE_TOL))
    rep = dict(max_do=float(do.max(initial=0.0)), mean_do=float(do.mean()) if do.size else 0.0,
               max_dlse=float(dl.max(initial=0.0)), bad_o=bad_o, bad_lse=bad_l)
    assert bad_o == 0 and bad_l == 0, f"{what}: {rep}"
    return rep


GUARD_BYTES = 4096  # sentinel bytes before and after a guarded buffer (keeps 16-byte alignment)
GUARD_FILL = 0xA5


class Guarded:
    """A device tensor with sentinel-filled guard bands on both sides (canaries for stray writes).

    ``t`` is the tensor the kernel gets; ``intact()`` checks that not one byte of either band (nor
    of the padding up to the next 256 bytes) changed.  The tensor itself starts filled with the
    sentinel too, so any element a kernel forgets to write is visible as well.
    """

    def __init__(self, shape, dtype, device="cuda"):
        import torch
        shape = tuple(int(x) for x in shape)
        elem = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(np.prod(shape, dtype=np.int64)) * elem
        padded = (self.nbytes + 255) // 256 * 256
        self.raw = torch.full((2 * GUARD_BYTES + padded,), GUARD_FILL, dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        import torch
        lo = self.raw[:GUARD_BYTES]
        hi = self.raw[GUARD_BYTES + self.nbytes:]
        return bool(torch.all(lo == GUARD_FILL).item() and torch.all(hi == GUARD_FILL).item())


NAN_BITS = {"bf16": 0x7FC0, "fp16": 0x7E00}  # a quiet NaN of each 16-bit type


def paginate(k_bits, v_bits, lens, ps, dtype, seed, spare=3, shuffle=True):
    """Pool [P, ps, Hkv, D] (16-bit patterns) and block table [B, pages_per_seq] (int32) holding the
    contiguous cache's valid rows; NaN everywhere else, -1 in the table entries no item needs."""
    B, Nk, Hkv, D = k_bits.shape
    pps = -(-Nk // ps)
    need = [-(-int(L) // ps) for L in lens]
    P = sum(need) + spare
    perm = np.random.default_rng(seed).permutation(P) if shuffle else np.arange(P)
    kp = np.full((P, ps, Hkv, D), NAN_BITS[dtype], dtype=np.uint16)
    vp = np.full((P, ps, Hkv, D), NAN_BITS[dtype], dtype=np.uint16)
    table = np.full((B, pps), -1, dtype=np.int32)
    t = 0
    for b, L in enumerate(lens):
        for i in range(need[b]):
            page = int(perm[t])
            t += 1
            table[b, i] = page
            n = min(ps, int(L) - i * ps)
            kp[page, :n] = k_bits[b, i * ps:i * ps + n]
            vp[page, :n] = v_bits[b, i * ps:i * ps + n]
    return kp, vp, table
