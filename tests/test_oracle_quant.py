"""Pins of the oracle's blockwise quantisers.

* a 1x128 block worked by hand (golden fixture) with a power-of-two scale, covering
  exact codes, E4M3 ties, subnormal codes, underflow and signed zeros;
* invariants on every block of seeded heavy-tailed and outlier data: a non-zero
  block's amax maps to +-448 exactly, codes are never NaN, each code is the nearest
  E4M3 value to x/s (checked in float64), signs agree, s*448 reproduces amax to FP32
  rounding;
* locality: a planted outlier changes only the scale and codes of its own block, which
  pins the block geometry and the scale index layout of all three quantisers;
* special cases: an all-zero block, a constant block, a partial 128x128 row block.
"""

import json
import os

import numpy as np
import torch

from oracle import e4m3, quant
from tests.conftest import GOLDEN
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl


def _bits(x_f32):
    """float32 values that are exactly BF16 -> their BF16 bit patterns."""
    x = np.asarray(x_f32, dtype=np.float32)
    b = x.view(np.uint32)
    assert np.all(b & 0xFFFF == 0), "value is not exactly representable in BF16"
    return (b >> 16).astype(np.uint16)


def _seeded_bits(shape, seed, std=1.0, outliers=()):
    g = torch.Generator().manual_seed(seed)
    x = wl.heavy_tailed(shape, std, g, "cpu")
    if outliers:
        x[:, list(outliers)] *= 50.0
    return wl.bf16_bits(wl.bf16(x))


def test_worked_1x128_block():
    with open(os.path.join(GOLDEN, "quant_1x128_worked.json")) as f:
        gold = json.load(f)
    x = np.zeros(128, dtype=np.float32)
    for e in gold["elements"]:
        x[e["index"]] = e["x"]
    q, s = quant.quant_1x128(_bits(x)[None, :])
    assert s.shape == (1, 1) and s[0, 0] == np.float32(gold["scale"])
    listed = {e["index"] for e in gold["elements"]}
    for e in gold["elements"]:
        assert q[0, e["index"]] == int(e["code"], 16), e
        assert np.float32(e["x"]) / s[0, 0] == np.float32(e["x_over_s"])
    for i in range(128):
        if i not in listed:
            assert q[0, i] == 0x00


def _check_block_invariants(x_f32, codes, scales):
    """x_f32 [G, g] groups, codes [G, g], scales [G]."""
    amax = np.max(np.abs(x_f32), axis=1)
    dec = e4m3.decode(codes)
    assert not np.any(np.isnan(dec)), "NaN code emitted"
    nz = amax > 0
    assert np.all(np.max(np.abs(dec[nz]), axis=1) == 448.0)
    assert np.all(scales[~nz] == 0) and np.all(codes[~nz] & 0x7F == 0)
    # s * 448 reproduces amax within FP32 rounding of the division: half an ulp of s,
    # relative for a normal s and at most 2^-150 absolute for a subnormal one
    s64 = scales[nz].astype(np.float64)
    bound = 448.0 * np.maximum(s64 * 2.0 ** -24, 2.0 ** -150)
    assert np.all(np.abs(s64 * 448.0 - amax[nz]) <= bound)
    # each code is the nearest E4M3 value to the FP32 quotient (in float64, exactly)
    quot = (x_f32[nz] / scales[nz][:, None]).astype(np.float64)
    pos = e4m3.DECODE_F64[:0x7F]
    a = np.minimum(np.abs(quot), 448.0)
    err = np.abs(np.abs(dec[nz]) - a)
    idx = np.searchsorted(pos, a)
    gap_lo = a - pos[np.maximum(idx - 1, 0)]
    gap_hi = pos[np.minimum(idx, 0x7E)] - a
    assert np.all(err <= np.minimum(np.where(gap_lo >= 0, gap_lo, np.inf), np.abs(gap_hi)) + 0.0)
    assert np.array_equal(np.signbit(dec), np.signbit(x_f32))


def test_1x128_invariants_heavy_tailed_and_outliers():
    bits = _seeded_bits((256, 1024), seed=7, outliers=(17, 130, 131, 400))
    q, s = quant.quant_1x128(bits)
    assert q.shape == (256, 1024) and s.shape == (8, 256)
    x = quant.bf16_bits_to_f32(bits)
    _check_block_invariants(x.reshape(-1, 128), q.reshape(-1, 128), s.T.reshape(-1))


def test_1x128_invariants_tiny_and_subnormal_magnitudes():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    x *= np.float32(2.0) ** rng.integers(-140, -100, size=(64, 1)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)  # truncate to BF16
    q, s = quant.quant_1x128(bits)
    xf = quant.bf16_bits_to_f32(bits)
    _check_block_invariants(xf.reshape(-1, 128), q.reshape(-1, 128), s.T.reshape(-1))
    assert np.any(s < np.finfo(np.float32).tiny), "the sweep should reach subnormal scales"


def test_1x128_locality_pins_scale_layout():
    bits = _seeded_bits((8, 512), seed=11)
    q0, s0 = quant.quant_1x128(bits)
    x = quant.bf16_bits_to_f32(bits).copy()
    r, c = 5, 300  # block (row 5, column block 2)
    x[r, c] = 1000.0
    q1, s1 = quant.quant_1x128(_bits(x))
    ds = np.argwhere(s0 != s1)
    assert ds.tolist() == [[2, 5]]
    dq = np.argwhere(q0 != q1)
    assert np.all(dq[:, 0] == r) and np.all(dq[:, 1] // 128 == 2)


def test_transposed_locality_pins_token_blocks():
    bits = _seeded_bits((384, 16), seed=12)  # T = 384 tokens, C = 16 channels
    qt0, st0 = quant.quant_1x128_transposed(bits)
    assert qt0.shape == (16, 384) and st0.shape == (3, 16)
    x = quant.bf16_bits_to_f32(bits).copy()
    x[200, 9] = -1000.0  # token 200 -> token block 1, channel 9
    qt1, st1 = quant.quant_1x128_transposed(_bits(x))
    assert np.argwhere(st0 != st1).tolist() == [[1, 9]]
    dq = np.argwhere(qt0 != qt1)
    assert np.all(dq[:, 0] == 9) and np.all(dq[:, 1] // 128 == 1)
    assert qt1[9, 200] == 0xFE  # the outlier itself is the block amax -> -448
    # the same codes as the row-wise quantiser applied to the explicit transpose
    q_rt, s_rt = quant.quant_1x128(np.ascontiguousarray(_bits(x).T))
    assert np.array_equal(q_rt, qt1) and np.array_equal(s_rt, st1)


def test_128x128_locality_partial_block_and_transpose():
    bits = _seeded_bits((300, 256), seed=13, std=0.02)  # 3 row blocks, last has 44 rows
    q0, qt0, s0 = quant.quant_128x128(bits)
    assert s0.shape == (3, 2) and qt0.shape == (256, 300)
    assert np.array_equal(qt0, q0.T)
    x = quant.bf16_bits_to_f32(bits).copy()
    x[290, 10] = 5.0  # row block 2 (partial), column block 0
    q1, _, s1 = quant.quant_128x128(_bits(x))
    assert np.argwhere(s0 != s1).tolist() == [[2, 0]]
    assert s1[2, 0] == np.float32(5.0) / np.float32(448.0)
    dq = np.argwhere(q0 != q1)
    assert np.all(dq[:, 0] >= 256) and np.all(dq[:, 1] < 128)
    blk = quant.bf16_bits_to_f32(_bits(x))[256:300, 0:128]
    _check_block_invariants(blk.reshape(1, -1), q1[256:300, 0:128].reshape(1, -1), s1[2:3, 0])


def test_zero_and_constant_blocks():
    x = np.zeros((2, 256), dtype=np.float32)
    x[0, 5] = -0.0
    x[1, 128:] = 0.75  # constant block: every code is 448, s = 0.75/448
    q, s = quant.quant_1x128(_bits(x))
    assert s[0, 0] == 0 and s[1, 0] == 0 and s[0, 1] == 0
    assert q[0, 5] == 0x80 and np.all(np.delete(q[0], 5) == 0)
    assert s[1, 1] == np.float32(0.75) / np.float32(448.0)
    assert np.all(q[1, 128:] == 0x7E)
