"""Pins of the oracle's own binary16 converters against numpy's (a library
routine, IEEE 754 round-to-nearest-even with subnormals)."""
import numpy as np

import oracle


def _is_nan16(h):
    return ((h & 0x7C00) == 0x7C00) & ((h & 0x3FF) != 0)


def test_half_to_float_all_65536_patterns():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_float(h)
    want = h.view(np.float16).astype(np.float32)
    nan = _is_nan16(h)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    assert np.isnan(got[nan]).all()
    # payload is widened, not canonicalised
    assert np.array_equal(got[nan].view(np.uint32) & 0x7FFFFF,
                          (h[nan].astype(np.uint32) & 0x3FF) << 13)


def _check_f32_to_f16(bits):
    x = bits.astype(np.uint32).view(np.float32)
    got = oracle.float_to_half(x)
    want = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan]), bits[~nan][got[~nan] != want[~nan]][:8]
    assert _is_nan16(got[nan]).all()


def test_float_to_half_rounding_boundaries_every_exponent():
    # every sign/exponent/top-10-mantissa prefix, with the 13 dropped bits at
    # zero, just below, at and just above the halfway point, and all ones
    hi = np.arange(1 << 19, dtype=np.uint64) << 13
    for lo in (0x0000, 0x0001, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x0800, 0x1800):
        _check_f32_to_f16(hi | lo)


def test_float_to_half_subnormal_and_overflow_range_dense():
    rs = np.random.default_rng(1234)
    # results in the binary16 subnormal range: fp32 exponents 101..113
    exp = rs.integers(100, 114, size=1 << 21).astype(np.uint64)
    man = rs.integers(0, 1 << 23, size=1 << 21).astype(np.uint64)
    sign = rs.integers(0, 2, size=1 << 21).astype(np.uint64)
    _check_f32_to_f16((sign << 31) | (exp << 23) | man)
    # exact ties at every drop width of the subnormal path
    ties = []
    for e in range(101, 114):
        drop = 14 - (e - 127 + 15)
        if 1 <= drop <= 24:
            for q in (0, 1, 2, 3, 0x1FF, 0x200, 0x3FF):
                full = (q << drop) | (1 << (drop - 1))
                if full >> 23 == 1:
                    ties.append((e << 23) | (full & 0x7FFFFF))
    _check_f32_to_f16(np.array(ties, dtype=np.uint64))
    # around the largest finite binary16 (65504) and the rounding to infinity
    top = np.arange(0x477F0000, 0x47801000, dtype=np.uint64)
    _check_f32_to_f16(top)
    _check_f32_to_f16(top | (1 << 31))


def test_float_to_half_random_patterns():
    rs = np.random.default_rng(99)
    _check_f32_to_f16(rs.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64))


def test_specials():
    vals = np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65520.0, 65519.996, 2.0 ** -24,
                     2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -14, 1.0, -1.0],
                    dtype=np.float32)
    got = oracle.float_to_half(vals)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)
    assert got[1] == 0x8000 and got[4] == 0x7BFF and got[5] == 0x7C00 and got[8] == 0


# --- bfloat16: pinned against torch's bfloat16 casts (a library routine) ---

def _torch_bf16_bits(x32):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_to_float_all_65536_patterns():
    import torch
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_float(h)
    want = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(want)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    assert np.isnan(got[nan]).all()


def _check_f32_to_bf16(bits):
    x = bits.astype(np.uint32).view(np.float32)
    got = oracle.float_to_bf16(x)
    want = _torch_bf16_bits(x)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan])
    assert (((got[nan] & 0x7F80) == 0x7F80) & ((got[nan] & 0x7F) != 0)).all()


def test_float_to_bf16_rounding_boundaries_every_prefix():
    hi = np.arange(1 << 16, dtype=np.uint64) << 16
    for lo in (0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000):
        _check_f32_to_bf16(hi | lo)


def test_float_to_bf16_random_patterns():
    rs = np.random.default_rng(17)
    _check_f32_to_bf16(rs.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64))
