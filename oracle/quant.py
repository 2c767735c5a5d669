"""Blockwise BF16 -> E4M3 quantisers of the oracle (test infrastructure only).

Block geometry follows "Paper walkthrough: Puro-2B ...", section "Lever 2: use
blockwise FP8 from step zero": activations and their gradients get one scale per 128
consecutive elements along the reduction dimension ("1x128"), weights one scale per
128x128 block. For the weight-gradient GEMM the reduction dimension is the token
dimension, so its operands are quantised in 1x128 groups along tokens: here that is
the 1x128 routine applied to the explicit transpose.

Per block (any geometry), in FP32 as the method fixes it:
  amax = max |x|                       (exact: BF16 -> FP32 is exact)
  s    = amax / 448                    (correctly rounded FP32 division)
  q    = E4M3_RNE_sat(x / s)           (correctly rounded FP32 division, then encode)
  amax == 0  ->  s = 0 and q = sign-preserving zero (0x00 / 0x80), no division.

Inputs are BF16 given as their uint16 bit patterns. NumPy float32 division is IEEE
correctly rounded and keeps subnormals, which is the precision the method uses.
"""

import numpy as np

from . import e4m3

BLOCK = 128
FP8_MAX = np.float32(448.0)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact BF16 -> FP32: a BF16 value is the top half of the FP32 bit pattern."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize_groups(x: np.ndarray):
    """Quantise float32 groups laid along the last axis.

    ``x`` has shape [..., g]; every slice ``x[i, ..., :]`` is one scaling group.
    Returns (codes uint8 of x's shape, scales float32 of shape x.shape[:-1]).
    """
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)  # float32, exact
    s = amax / FP8_MAX  # float32 / float32 -> correctly rounded float32
    assert s.dtype == np.float32
    assert np.all((s > 0) | (amax == 0)), "a non-zero amax never gives a zero scale"
    zero = amax == 0
    divisor = np.where(zero, np.float32(1.0), s).astype(np.float32)
    # amax == 0: every x is +-0 and x / 1 keeps it, so the code is the signed zero.
    quotient = x / divisor[..., None]
    assert quotient.dtype == np.float32
    return e4m3.encode(quotient), s.astype(np.float32)


def quant_1x128(x_bits: np.ndarray):
    """1x128 quantisation along the columns (the reduction dim) of X [R, C].

    Returns Xq uint8 [R, C] and S float32 [C/128, R] (block-major: S[j, r] is the
    scale of X[r, 128*j : 128*j + 128]). Requires C % 128 == 0.
    """
    x = bf16_bits_to_f32(x_bits)
    r, c = x.shape
    assert c % BLOCK == 0, "the reduction dimension must be a multiple of 128"
    q, s = quantize_groups(x.reshape(r, c // BLOCK, BLOCK))
    return q.reshape(r, c), np.ascontiguousarray(s.T)


def quant_1x128_transposed(x_bits: np.ndarray):
    """1x128 quantisation along the rows (tokens) of X [T, C], output transposed.

    Equivalent by definition to quant_1x128 of the transpose X^T [C, T]:
    returns XqT uint8 [C, T] and ST float32 [T/128, C]. Requires T % 128 == 0.
    """
    xt = np.ascontiguousarray(np.asarray(x_bits, dtype=np.uint16).T)
    return quant_1x128(xt)


def quant_128x128(w_bits: np.ndarray):
    """128x128 block quantisation of W [R, C] (weights; C is the reduction dim).

    Returns Wq uint8 [R, C], WqT uint8 [C, R] (the same codes transposed) and
    S float32 [ceil(R/128), C/128]. A partial last row-block takes its amax over the
    rows that exist. Requires C % 128 == 0.
    """
    w = bf16_bits_to_f32(w_bits)
    r, c = w.shape
    assert c % BLOCK == 0, "the reduction dimension must be a multiple of 128"
    rb = -(-r // BLOCK)
    cb = c // BLOCK
    q = np.empty((r, c), dtype=np.uint8)
    s = np.empty((rb, cb), dtype=np.float32)
    for i in range(rb):
        r0, r1 = i * BLOCK, min(r, (i + 1) * BLOCK)
        rows = r1 - r0
        # [rows, cb, 128] -> [cb, rows * 128]: one group per 128x128 block
        blocks = w[r0:r1].reshape(rows, cb, BLOCK).transpose(1, 0, 2).reshape(cb, rows * BLOCK)
        qb, sb = quantize_groups(blocks)
        q[r0:r1] = qb.reshape(cb, rows, BLOCK).transpose(1, 0, 2).reshape(rows, c)
        s[i] = sb
    return q, np.ascontiguousarray(q.T), s
