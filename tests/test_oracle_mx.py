"""Pins of the oracle's power-of-two (UE8M0) scale mode.

* The exponent rule against its definition in exact rationals: 448 * 2**e >= amax and
  448 * 2**(e-1) < amax for every non-clamped group, on BF16 magnitudes over the whole
  exponent range (subnormals included), plus the clamp and the all-zero group.
* A 1x128 group worked by hand (tests/golden/quant_1x128_pow2_worked.json): scale byte
  and codes, including a tie, the smallest subnormal and a signed zero.
* Every code is the nearest E4M3 value to x * 2**-e (brute force over the decode table,
  ties to even), nothing saturates, and the largest decoded magnitude of a non-clamped
  group lies in (224, 448].
* The three geometries agree with the 1x128 group routine on explicit regroupings, and
  scales_from_ue8m0 inverts the byte encoding exactly.
"""

import json
import os
from fractions import Fraction

import numpy as np

from oracle import e4m3, mx
from oracle.quant import bf16_bits_to_f32
from tests.conftest import GOLDEN


def _bf16_magnitudes(rng, n):
    bits = rng.integers(0, 0x7F80, size=n).astype(np.uint16)  # every finite positive BF16 pattern
    return bf16_bits_to_f32(bits)


def test_exponent_rule_exact():
    rng = np.random.default_rng(0)
    amax = np.concatenate([_bf16_magnitudes(rng, 20000),
                           np.array([448.0, 449.0, 224.0, 224.5, 1.0, 1.75, 3.5, 2.0 ** -133, 0.0],
                                    dtype=np.float32)])
    e = mx.pow2_exponent(amax)
    for a, k in zip(amax, e):
        a = Fraction(float(a))
        if a == 0:
            assert k == -127
            continue
        hi = Fraction(448) * Fraction(2) ** int(k)
        if k > -127:
            assert hi >= a and hi / 2 < a, (a, k)
        else:
            assert hi >= a  # clamped: the smallest exponent the byte can hold
    hand = dict(zip([448.0, 449.0, 224.0, 224.5, 1.0, 1.75, 3.5], [0, 1, -1, 0, -8, -8, -7]))
    for a, k in hand.items():
        assert mx.pow2_exponent(np.float32(a)) == k, a


def test_worked_group():
    with open(os.path.join(GOLDEN, "quant_1x128_pow2_worked.json")) as f:
        doc = json.load(f)
    x = np.zeros(128, dtype=np.float32)
    for el in doc["elements"]:
        x[el["index"]] = el["x"]
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)  # every value above is exact in BF16
    assert np.array_equal(bf16_bits_to_f32(bits), x)
    q, b = mx.quant_1x128_pow2(bits.reshape(1, 128))
    assert int(b[0, 0]) == doc["scale_byte"] == doc["e"] + 127
    want = np.zeros(128, dtype=np.uint8)
    for el in doc["elements"]:
        want[el["index"]] = int(el["code"], 16)
    assert np.array_equal(q[0], want)


def test_codes_are_nearest_and_unsaturated():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128)).astype(np.float32) * (2.0 ** rng.integers(-30, 30, size=(64, 1)))
    x[3] = 0.0
    x[4, ::2] = -0.0
    x[5] *= np.float32(2.0 ** -120)  # a group near the bottom of the range
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xf = bf16_bits_to_f32(bits).astype(np.float64)
    q, b = mx.quant_1x128_pow2(bits)
    s = mx.scales_from_ue8m0(b[0]).astype(np.float64)
    finite = e4m3.DECODE_F64[:127]
    for r in range(64):
        y = xf[r] / s[r]
        assert np.all(np.abs(y) <= 448.0)
        dec = e4m3.decode(q[r])
        err = np.abs(np.abs(y)[:, None] - finite[None, :])
        best = finite[np.argmin(err, axis=1)]
        tie = np.sum(np.isclose(err, err.min(axis=1, keepdims=True), rtol=0, atol=0), axis=1) > 1
        ok = (np.abs(dec) == best) | tie
        assert np.all(ok), r
        assert np.all(np.signbit(dec) == np.signbit(xf[r]))  # signs kept, zeros included
        amax = np.abs(xf[r]).max()
        if amax > 0 and b[0, r] > 0:
            assert 224.0 < np.abs(dec).max() <= 448.0


def test_geometries_and_byte_inverse():
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((300, 256)) * 0.02).astype(np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    q, qt, b = mx.quant_128x128_pow2(bits)
    assert np.array_equal(qt, q.T)
    for i in range(3):
        for j in range(2):
            blk = bf16_bits_to_f32(bits[128 * i:128 * i + 128, 128 * j:128 * j + 128])
            qb, bb = mx.quantize_groups_pow2(blk.reshape(1, -1))
            assert bb[0] == b[i, j]
            assert np.array_equal(qb.reshape(blk.shape), q[128 * i:128 * i + 128, 128 * j:128 * j + 128])
    x = (rng.standard_normal((256, 384))).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    qt2, bt2 = mx.quant_1x128_transposed_pow2(xb)
    q3, b3 = mx.quant_1x128_pow2(np.ascontiguousarray(xb.T))
    assert np.array_equal(qt2, q3) and np.array_equal(bt2, b3)
    all_bytes = np.arange(255, dtype=np.uint8)
    s = mx.scales_from_ue8m0(all_bytes).astype(np.float64)
    assert np.array_equal(s, np.exp2(all_bytes.astype(np.float64) - 127))
    assert np.array_equal(mx.pow2_exponent(s * 448.0) + 127, all_bytes.astype(np.int64))
