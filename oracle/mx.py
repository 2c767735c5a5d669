"""Power-of-two (UE8M0) scale mode of the blockwise quantisers (test infrastructure only).

The method's groups ("Paper walkthrough: Puro-2B ...", section "Lever 2: use blockwise
FP8 from step zero": 1x128 along the reduction dimension for activations and gradients,
128x128 blocks for weights) with each scale restricted to a power of two, stored as an
unsigned exponent byte (UE8M0, the scale-factor format of the tensor cores' block-scaled
FP8 MMAs, which apply such scales inside the MMA). The pages fix only FP8 with local
scales; this mode is a variant of the GEMM path, not the pages' own scale formula, and
takes these readings:

  e    = the smallest integer with 448 * 2**e >= amax   (the method's s = amax / 448,
                                                         rounded up to a power of two)
         clamped to [-127, 127]; an all-zero group takes e = -127
  byte = e + 127                                        (UE8M0; 0xFF, the NaN code, unused)
  q    = E4M3_RNE(x * 2**-e)                            (an exact scaling: |x| * 2**-e <= 448,
                                                         so nothing saturates)

Inputs are BF16 bit patterns; x * 2**-e is formed in float32, where it is exact for
every BF16 x and every e this rule yields (the product lies between 2**-6 and 448 or is
zero). Dequantised values decode(q) * 2**e are exact in float64, so the FP64 GEMM of
oracle.gemm applies unchanged with scales_from_ue8m0.
"""

import numpy as np

from . import e4m3
from .quant import BLOCK, bf16_bits_to_f32

E_MIN, E_MAX = -127, 127


def pow2_exponent(amax) -> np.ndarray:
    """e per group: the smallest integer with 448 * 2**e >= amax, clamped to [-127, 127];
    -127 where amax == 0. Exact: amax and 448 * 2**e are exact in float64."""
    a = np.asarray(amax, dtype=np.float64)
    e = np.full(a.shape, E_MIN, dtype=np.int64)
    pos = a > 0
    # a first estimate from log2, then corrected with exact comparisons
    est = np.zeros(a.shape, dtype=np.int64)
    est[pos] = np.ceil(np.log2(a[pos] / 448.0)).astype(np.int64)
    for _ in range(3):
        too_small = pos & (448.0 * np.exp2(est.astype(np.float64)) < a)
        est = np.where(too_small, est + 1, est)
        too_big = pos & (448.0 * np.exp2((est - 1).astype(np.float64)) >= a)
        est = np.where(too_big, est - 1, est)
    e[pos] = est[pos]
    return np.clip(e, E_MIN, E_MAX)


def scales_from_ue8m0(b) -> np.ndarray:
    """The scales 2**(byte - 127) as float32 (exact, 2**-127 included)."""
    return np.exp2(np.asarray(b, dtype=np.float64) - 127.0).astype(np.float32)


def quantize_groups_pow2(x: np.ndarray):
    """Groups along the last axis of float32 x [..., g] -> (codes uint8 like x, UE8M0 bytes
    uint8 of shape x.shape[:-1])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    e = pow2_exponent(amax)
    inv = np.exp2(-e.astype(np.float64)).astype(np.float32)  # 2**-e, exact in float32
    y = x * inv[..., None]
    assert y.dtype == np.float32
    assert np.all(np.abs(y) <= 448.0), "a power-of-two scale of at least amax / 448 never saturates"
    return e4m3.encode(y), (e + 127).astype(np.uint8)


def quant_1x128_pow2(x_bits: np.ndarray):
    """X [R, C] in 1x128 groups along C -> (Xq uint8 [R, C], scale bytes uint8 [C/128, R])."""
    x = bf16_bits_to_f32(x_bits)
    r, c = x.shape
    assert c % BLOCK == 0
    q, b = quantize_groups_pow2(x.reshape(r, c // BLOCK, BLOCK))
    return q.reshape(r, c), np.ascontiguousarray(b.T)


def quant_1x128_transposed_pow2(x_bits: np.ndarray):
    """X [T, C] in 1x128 groups along T, transposed: (XqT [C, T], bytes [T/128, C])."""
    return quant_1x128_pow2(np.ascontiguousarray(np.asarray(x_bits, dtype=np.uint16).T))


def quant_128x128_pow2(w_bits: np.ndarray):
    """W [R, C] in 128x128 blocks -> (Wq [R, C], WqT [C, R], bytes [ceil(R/128), C/128]).
    A partial last row block takes its amax over the rows that exist."""
    w = bf16_bits_to_f32(w_bits)
    r, c = w.shape
    assert c % BLOCK == 0
    rb, cb = -(-r // BLOCK), c // BLOCK
    q = np.empty((r, c), dtype=np.uint8)
    b = np.empty((rb, cb), dtype=np.uint8)
    for i in range(rb):
        r0, r1 = i * BLOCK, min(r, (i + 1) * BLOCK)
        rows = r1 - r0
        blocks = w[r0:r1].reshape(rows, cb, BLOCK).transpose(1, 0, 2).reshape(cb, rows * BLOCK)
        qb, bb = quantize_groups_pow2(blocks)
        q[r0:r1] = qb.reshape(cb, rows, BLOCK).transpose(1, 0, 2).reshape(rows, c)
        b[i] = bb
    return q, np.ascontiguousarray(q.T), b
