"""Pins of the NVFP4 oracle (oracle/nvfp4.py) against things other than itself.

- the E2M1 value table, from the field formula and written out by hand;
- the encoder against a brute-force arg-min, with every tie and its neighbours;
- a hand-worked row of four groups (tests/golden/nvfp4_blocks_worked.json);
- invariants that a dropped divisor, a wrong tensor scale or a wrong tie rule would break:
  the group holding the tensor's amax gets the factor 448, every group's largest element
  encodes to +-6, and every code is within half a step of x / S;
- nibble order and the transposed layout;
- the contraction against an exact rational triple loop.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import e4m3, nvfp4
from oracle.quant import bf16_bits_to_f32

HERE = os.path.dirname(os.path.abspath(__file__))


def f32_to_bf16_bits(x):
    """Round-to-nearest-even float32 -> BF16 bit patterns (test input helper)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def test_e2m1_table():
    assert nvfp4.E2M1_DECODE[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert nvfp4.E2M1_DECODE[8:].tolist() == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert np.signbit(nvfp4.E2M1_DECODE[8])


def test_e2m1_encode_matches_bruteforce():
    mags = nvfp4.E2M1_POS
    mids = (mags[1:] + mags[:-1]) / 2
    pts = np.concatenate([mags, mids, [6.5, 7.0, 12.0, 1e30, 1e-30, 0.0]]).astype(np.float32)
    near = np.concatenate([np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rng = np.random.default_rng(0)
    rnd = rng.uniform(-8, 8, size=4000).astype(np.float32)
    v = np.concatenate([pts, -pts, near, -near, rnd, np.array([-0.0], dtype=np.float32)]).astype(np.float32)
    assert np.array_equal(nvfp4.e2m1_encode(v), nvfp4.e2m1_encode_bruteforce(v))


@pytest.mark.parametrize("v,code", [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
                                    (5.0001, 7), (4.9999, 6), (7.0, 7), (100.0, 7), (-0.25, 8), (-0.0, 8),
                                    (-1.75, 12), (0.2500001, 1)])
def test_e2m1_ties_and_saturation(v, code):
    assert int(nvfp4.e2m1_encode(np.float32(v))) == code


def test_worked_groups():
    g = json.load(open(os.path.join(HERE, "golden", "nvfp4_blocks_worked.json")))
    x = np.array(g["x"], dtype=np.float32).reshape(1, 64)
    bits = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(bits), x), "the fixture's values are BF16 numbers"
    packed, f, amax = nvfp4.quant_1x16(bits)
    assert float(amax) == g["tensor_amax"]
    assert f.reshape(-1).tolist() == g["factors"]
    assert nvfp4.unpack(packed).reshape(4, 16).tolist() == g["codes"]


def _rand_bits(rng, r, c, scale=1.0):
    x = rng.standard_normal((r, c)).astype(np.float32) * scale
    x[rng.random((r, c)) < 0.01] *= 40.0  # a few large values
    return f32_to_bf16_bits(x)


def test_tensor_max_group_factor_is_448_and_group_maxima_encode_to_6():
    rng = np.random.default_rng(1)
    bits = _rand_bits(rng, 24, 256)
    packed, f, amax = nvfp4.quant_1x16(bits)
    x = bf16_bits_to_f32(bits)
    r, j = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert f[r, j // 16] == 0x7E  # 448: the tensor scale was amax / (6 * 448)
    codes = nvfp4.unpack(packed).reshape(24, 16, 16)
    groups = np.abs(x).reshape(24, 16, 16)
    s_t = float(nvfp4.tensor_scale(amax))
    for a in range(24):
        for b in range(16):
            d_over_s = float(groups[a, b].max()) / 6.0 / s_t
            if d_over_s < 2.0 ** -6:  # a subnormal factor is coarser than the argument below
                continue
            k = int(np.argmax(groups[a, b]))
            # dec(e) is within 2**-4 of d / s_t, so |x_max| / S lies in [5.65, 6.4]: code 6
            assert codes[a, b, k] & 0x7 == 7


def test_codes_within_half_a_step():
    rng = np.random.default_rng(2)
    bits = _rand_bits(rng, 16, 512, scale=3.0)
    packed, f, amax = nvfp4.quant_1x16(bits)
    x = bf16_bits_to_f32(bits).astype(np.float64)
    S = e4m3.decode(f).astype(np.float32) * nvfp4.tensor_scale(amax)
    v = x / np.repeat(S.astype(np.float64), 16, axis=1)
    q = nvfp4.e2m1_decode(nvfp4.unpack(packed))
    half_step = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    assert np.all(np.abs(v - q) <= half_step + 1e-12)
    assert np.all(np.abs(q) <= 6.0)


def test_pack_nibble_order_and_roundtrip():
    assert nvfp4.pack(np.array([1, 2], dtype=np.uint8)).tolist() == [0x21]
    rng = np.random.default_rng(3)
    c = rng.integers(0, 16, size=(5, 32), dtype=np.uint8)
    assert np.array_equal(nvfp4.unpack(nvfp4.pack(c)), c)


def test_transposed_is_rows_of_transpose():
    rng = np.random.default_rng(4)
    bits = _rand_bits(rng, 64, 48)
    pt, ft, at = nvfp4.quant_1x16_transposed(bits)
    assert pt.shape == (48, 32) and ft.shape == (48, 4)
    x = bf16_bits_to_f32(bits)
    # group (c, j) covers rows 16 j .. 16 j + 15 of column c
    x_t = x.T.reshape(48, 4, 16)
    codes, f = nvfp4.quantize_groups(x_t, at)
    assert np.array_equal(f, ft)
    assert np.array_equal(nvfp4.pack(codes.reshape(48, 64)), pt)


def test_all_zero_tensor():
    bits = np.zeros((2, 32), dtype=np.uint16)
    bits[1, 3] = 0x8000  # -0
    p, f, a = nvfp4.quant_1x16(bits)
    assert float(a) == 0.0 and not f.any()
    assert nvfp4.unpack(p)[1, 3] == 8 and nvfp4.unpack(p).sum() == 8


def test_gemm_ref_exact_rational():
    rng = np.random.default_rng(5)
    m, n, k = 3, 2, 48
    a_bits = _rand_bits(rng, m, k)
    b_bits = _rand_bits(rng, n, k, scale=0.01)
    aq, af, aa = nvfp4.quant_1x16(a_bits)
    bq, bf, ba = nvfp4.quant_1x16(b_bits)
    got = nvfp4.gemm_ref(aq, af, aa, bq, bf, ba)
    sa, sb = Fraction(float(nvfp4.tensor_scale(aa))), Fraction(float(nvfp4.tensor_scale(ba)))
    ca, cb = nvfp4.unpack(aq), nvfp4.unpack(bq)
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for t in range(k):
                va = Fraction(nvfp4.e2m1_decode_code(int(ca[i, t]))) * Fraction(e4m3.decode_code(int(af[i, t // 16]))) * sa
                vb = Fraction(nvfp4.e2m1_decode_code(int(cb[j, t]))) * Fraction(e4m3.decode_code(int(bf[j, t // 16]))) * sb
                acc += va * vb
            assert abs(Fraction(got[i, j]) - acc) <= abs(acc) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)
    na, nb = nvfp4.row_col_norms(aq, af, aa, bq, bf, ba)
    da = nvfp4.dequant(aq, af, aa)
    assert np.allclose(na, [np.sqrt(sum(float(v) ** 2 for v in row)) for row in da], rtol=1e-14)
    assert nb.shape == (n,)
