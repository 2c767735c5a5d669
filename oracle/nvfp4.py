"""NVFP4 mode of the blockwise path (test infrastructure only).

The pages mention FP4 only as a capability of the hardware they chose (the jj-blog page,
the paragraph after its Table 2: among the GPUs within reach, the RTX 5090 was the one with
FP4 support). They give no FP4 recipe. This mode takes NVIDIA's published NVFP4 format as
the reading, with the method's own choices (scales from the tensor being quantised, groups
along the reduction dimension, correctly rounded FP32 arithmetic) carried over:

  element   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
            0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities, no NaN
  group     16 consecutive elements along the reduction dimension ("1x16")
  factor    one UE4M3 per group (the E4M3 format without its sign bit)
  tensor    one FP32 scale per tensor
  s_t  = amax_t / 2688                  (2688 = 6 * 448; correctly rounded FP32)
  d    = amax_g / 6                     (correctly rounded FP32)
  e    = E4M3_RNE_sat(d / s_t)          (correctly rounded FP32 quotient, then the E4M3
                                         encoder of the FP8 path; never above 448 because
                                         amax_g <= amax_t, so the saturation only guards
                                         rounding)
  S    = dec(e) * s_t                   (correctly rounded FP32 product)
  q    = E2M1_RNE_sat(x / S)            (correctly rounded FP32 quotient, nearest E2M1
                                         magnitude, ties to the even code, saturating at 6)
  S == 0 (an all-zero tensor or group, or a factor that rounds to zero): q = signed zero.
  value of a code: dec(q) * dec(e) * s_t, exact in float64.

Storage: two codes per byte, element 2i in the low nibble and 2i+1 in the high nibble;
factors row-major, F[r, j] is the factor of X[r, 16j : 16j + 16]. The transposed mode is
the same rule applied to X's transpose (groups of 16 consecutive tokens for the wgrad
operands). Inputs must be finite.
"""

import numpy as np

from . import e4m3
from .quant import bf16_bits_to_f32

GROUP = 16
E2M1_MAX = 6.0
TENSOR_DIV = np.float32(2688.0)  # 6 * 448

# magnitudes of the codes 0..7 (sign in bit 3)
E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode_code(code: int) -> float:
    """Value of one E2M1 code from its fields (exact)."""
    sign = -1.0 if code & 0x8 else 1.0
    exp_field = (code >> 1) & 0x3
    mant = code & 0x1
    if exp_field == 0:
        return sign * 0.5 * mant  # subnormal: mantissa * 2**(1 - bias - 1)
    return sign * (1.0 + 0.5 * mant) * 2.0 ** (exp_field - 1)


E2M1_DECODE = np.array([e2m1_decode_code(c) for c in range(16)], dtype=np.float64)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_DECODE[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code of float32 values (ties to the even code, saturating at 6).

    Distances are formed in float64, where the difference of a float32 and one of the
    eight magnitudes is exact, so ties are detected exactly. The sign is kept, so a
    negative value that rounds to zero gives the code 0x8.
    """
    v = np.asarray(v, dtype=np.float32)
    neg = np.signbit(v)
    a = np.minimum(np.abs(v).astype(np.float64), E2M1_MAX)
    hi = np.minimum(np.searchsorted(E2M1_POS, a, side="left"), 7)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - E2M1_POS[lo]
    d_hi = E2M1_POS[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    return code | (neg.astype(np.uint8) << 3)


def e2m1_encode_bruteforce(v: np.ndarray) -> np.ndarray:
    """Independent slow encoder: arg-min over the eight magnitudes, even code on a tie."""
    v = np.asarray(v, dtype=np.float32).reshape(-1)
    neg = np.signbit(v)
    a = np.minimum(np.abs(v).astype(np.float64), E2M1_MAX)
    dist = np.abs(a[:, None] - E2M1_POS[None, :])
    cand = dist == dist.min(axis=1, keepdims=True)
    even = (np.arange(8) % 2 == 0)[None, :]
    pick = cand & even
    code = np.where(pick.any(axis=1), pick.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)
    return code | (neg.astype(np.uint8) << 3)


def tensor_scale(amax_t) -> np.float32:
    """s_t = amax_t / 2688 in correctly rounded FP32."""
    return np.float32(amax_t) / TENSOR_DIV


def quantize_groups(x: np.ndarray, amax_t):
    """Quantise float32 groups of 16 laid along the last axis, with tensor amax ``amax_t``.

    Returns (codes uint8 [..., 16] one per element, factors uint8 [...] UE4M3).
    """
    x = np.asarray(x, dtype=np.float32)
    assert x.shape[-1] == GROUP
    s_t = tensor_scale(amax_t)
    amax_g = np.max(np.abs(x), axis=-1)
    d = amax_g / np.float32(6.0)
    assert d.dtype == np.float32
    if s_t > 0:
        e = e4m3.encode(d / s_t)  # non-negative: the code has no sign bit set
    else:
        e = np.zeros(d.shape, dtype=np.uint8)
    S = (e4m3.decode(e).astype(np.float32) * s_t).astype(np.float32)
    zero = S == 0
    divisor = np.where(zero, np.float32(1.0), S).astype(np.float32)
    quotient = x / divisor[..., None]
    assert quotient.dtype == np.float32
    # S == 0: every value of the group is stored as a signed zero
    quotient = np.where(zero[..., None], quotient * np.float32(0.0), quotient)
    return e2m1_encode(quotient), e.astype(np.uint8)


def tensor_amax(x_bits: np.ndarray) -> np.float32:
    return np.float32(np.max(np.abs(bf16_bits_to_f32(x_bits)))) if np.size(x_bits) else np.float32(0.0)


def pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte along the last axis: element 2i low nibble, 2i+1 high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def quant_1x16(x_bits: np.ndarray):
    """1x16 NVFP4 quantisation along the columns of X [R, C] (C % 16 == 0).

    Returns (packed codes uint8 [R, C/2], factors uint8 [R, C/16], tensor amax float32).
    """
    x = bf16_bits_to_f32(x_bits)
    r, c = x.shape
    assert c % GROUP == 0
    amax_t = tensor_amax(x_bits)
    codes, f = quantize_groups(x.reshape(r, c // GROUP, GROUP), amax_t)
    return pack(codes.reshape(r, c)), f.reshape(r, c // GROUP), amax_t


def quant_1x16_transposed(x_bits: np.ndarray):
    """The 1x16 rule on X's transpose: groups of 16 consecutive rows of X [R, C].

    Returns (packed codes uint8 [C, R/2], factors uint8 [C, R/16], tensor amax float32).
    """
    return quant_1x16(np.ascontiguousarray(np.asarray(x_bits).T))


def dequant(packed: np.ndarray, factors: np.ndarray, amax_t) -> np.ndarray:
    """Values of a quantised [R, K] operand in float64: dec(q) * dec(e) * s_t (exact)."""
    codes = unpack(packed)
    r, k = codes.shape
    f = e4m3.decode(np.asarray(factors, dtype=np.uint8))  # [R, K/16]
    s_t = float(tensor_scale(amax_t))
    return e2m1_decode(codes) * np.repeat(f, GROUP, axis=1)[:, :k] * s_t


def gemm_ref(aq, a_f, a_amax, bq, b_f, b_amax) -> np.ndarray:
    """C[M, N] = A . B^T of two operands quantised along their K, in float64."""
    return dequant(aq, a_f, a_amax) @ dequant(bq, b_f, b_amax).T


def row_col_norms(aq, a_f, a_amax, bq, b_f, b_amax):
    """Euclidean norms of the dequantised rows of A and of B (the elementwise bound's factors)."""
    a = dequant(aq, a_f, a_amax)
    b = dequant(bq, b_f, b_amax)
    return np.sqrt(np.sum(a * a, axis=1)), np.sqrt(np.sum(b * b, axis=1))
