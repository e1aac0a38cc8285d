"""Comparison helpers shared by the tests (ulp distances, NaN-aware equality)."""
import numpy as np


def _ordered32(x):
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.where(b < 0, -(b & 0x7FFFFFFF), b)


def _ordered16(h):
    b = np.ascontiguousarray(h, dtype=np.uint16).astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def ulp32(a, b):
    """Elementwise distance in fp32 units in the last place (+0 == -0)."""
    return np.abs(_ordered32(a) - _ordered32(b))


def ulp16(a_bits, b_bits):
    """Elementwise distance in fp16 ulps between uint16 bit patterns."""
    return np.abs(_ordered16(a_bits) - _ordered16(b_bits))


def assert_f32_close(got, want, max_ulp, what=""):
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    nan_g, nan_w = np.isnan(got), np.isnan(want)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    d = ulp32(got[~nan_g], want[~nan_w])
    worst = int(d.max()) if d.size else 0
    assert worst <= max_ulp, f"{what}: {worst} ulp > {max_ulp} (at {int(np.argmax(d))})"


def assert_f16_close(got_bits, want_bits, max_ulp, what=""):
    got = np.asarray(got_bits, np.uint16)
    want = np.asarray(want_bits, np.uint16)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    nan_g = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
    nan_w = ((want & 0x7C00) == 0x7C00) & ((want & 0x3FF) != 0)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    d = ulp16(got[~nan_g], want[~nan_w])
    worst = int(d.max()) if d.size else 0
    assert worst <= max_ulp, f"{what}: {worst} fp16 ulp > {max_ulp} (at {int(np.argmax(d))})"


def assert_bf16_close(got_bits, want_bits, max_ulp, what=""):
    got = np.asarray(got_bits, np.uint16)
    want = np.asarray(want_bits, np.uint16)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
    nan_w = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    d = ulp16(got[~nan_g], want[~nan_w])   # sign-magnitude order holds for both formats
    worst = int(d.max()) if d.size else 0
    assert worst <= max_ulp, f"{what}: {worst} bf16 ulp > {max_ulp} (at {int(np.argmax(d))})"


def read_golden(path):
    """Parse a golden fixture: '#' comments, then whitespace-separated rows."""
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows
