"""Pins of the oracle's E4M3 codec against things other than itself.

* closed forms worked by hand from the format's field formula (golden fixture);
* PyTorch's own float8_e4m3fn conversion (a library routine) for decode and encode;
* a brute-force arg-min encoder over all 127 magnitudes, on a structured sweep of
  every FP32 exponent and top mantissa bits with the rounding-critical low bits;
* hand-constructed ties, saturation and signed zeros.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import e4m3
from tests.conftest import GOLDEN


def _closed_forms():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_closed_forms.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, value = line.split()[:2]
            rows.append((int(code, 16), float(value)))
    return rows


def test_decode_closed_forms():
    rows = _closed_forms()
    assert len(rows) >= 20
    for code, value in rows:
        got = e4m3.DECODE_F64[code]
        if math.isnan(value):
            assert math.isnan(got), hex(code)
        else:
            assert got == value, hex(code)
            assert math.copysign(1.0, got) == math.copysign(1.0, value), hex(code)


def test_decode_matches_torch_float8_e4m3fn():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(e4m3.DECODE_F64))
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan], e4m3.DECODE_F64[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(e4m3.DECODE_F64[~nan]))


def _torch_encode(x):
    """Library routine: clamp to +-448 (the saturating step), then PyTorch's RNE cast."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _structured_sweep():
    """Every sign, every FP32 exponent field up to 2^9, every value of the top ten
    mantissa bits, and low 13 bits drawn from patterns that decide rounding."""
    sign = np.array([0, 1], dtype=np.uint32)
    exp = np.arange(0, 137, dtype=np.uint32)  # 2^(136-127) = 512 > 448
    top = np.arange(1024, dtype=np.uint32)
    low = np.array([0, 1, 0x0FFF, 0x1000, 0x1001, 0x1FFF], dtype=np.uint32)
    bits = (sign[:, None, None, None] << 31) | (exp[None, :, None, None] << 23) \
        | (top[None, None, :, None] << 13) | low[None, None, None, :]
    return bits.reshape(-1).view(np.float32)


def test_encode_matches_bruteforce_structured():
    x = _structured_sweep()
    fast = e4m3.encode(x)
    for i in range(0, x.size, 1 << 16):
        sl = slice(i, i + (1 << 16))
        assert np.array_equal(fast[sl], e4m3.encode_bruteforce(x[sl])), i


def test_encode_matches_torch_structured_and_random():
    x = _structured_sweep()
    assert np.array_equal(e4m3.encode(x), _torch_encode(x))
    rng = np.random.default_rng(1234)
    bits = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    y = bits.view(np.float32)
    y = y[np.isfinite(y) & (np.abs(y) <= 500.0)]
    assert y.size > 1 << 20
    assert np.array_equal(e4m3.encode(y), _torch_encode(y))


def test_encode_exact_ties_go_to_even():
    pos = e4m3.DECODE_F64[:0x7F]
    for c in range(0x7E):
        mid = np.float32((pos[c] + pos[c + 1]) / 2)  # exact in FP32
        assert float(mid) == (pos[c] + pos[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert e4m3.encode(mid) == want, hex(c)
        assert e4m3.encode(-mid) == (want | 0x80), hex(c)
        above = np.nextafter(mid, np.float32(np.inf))
        below = np.nextafter(mid, np.float32(-np.inf))
        assert e4m3.encode(above) == c + 1
        assert e4m3.encode(below) == c


def test_encode_saturates_and_keeps_sign_of_zero():
    cases = [
        (448.0, 0x7E), (463.99, 0x7E), (464.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE), (-449.0, 0xFE),
        (0.0, 0x00), (-0.0, 0x80), (1e-30, 0x00), (-1e-30, 0x80),
        (2.0 ** -10, 0x00), (-(2.0 ** -10), 0x80), (2.0 ** -9, 0x01),
    ]
    for x, want in cases:
        assert e4m3.encode(np.float32(x)) == want, x
    just_above_tie = np.nextafter(np.float32(2.0 ** -10), np.float32(1))
    assert e4m3.encode(just_above_tie) == 0x01


def test_encode_roundtrips_every_finite_code():
    finite = [c for c in range(256) if c not in e4m3.NAN_CODES]
    vals = e4m3.DECODE_F64[finite].astype(np.float32)
    assert np.array_equal(e4m3.encode(vals), np.array(finite, dtype=np.uint8))


@pytest.mark.slow
def test_encode_exhaustive_all_fp32_in_range():
    """Every FP32 bit pattern with |x| <= 464 against PyTorch's cast (opt-in, minutes)."""
    chunk = 1 << 24
    for start in range(0, 1 << 32, chunk):
        bits = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        x = x[np.isfinite(x) & (np.abs(x) <= 464.0)]
        if x.size:
            assert np.array_equal(e4m3.encode(x), _torch_encode(x)), start
