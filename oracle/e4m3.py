"""E4M3 codec of the oracle (test infrastructure only).

The pages name the format only as "FP8" ("Paper walkthrough: Puro-2B ...", section
"Lever 2: use blockwise FP8 from step zero"). The encoding used here is the E4M3
variant of the OCP 8-bit floating point format: one sign bit, four exponent bits with
bias 7, three mantissa bits; subnormals when the exponent field is 0; the pattern with
exponent 15 and mantissa 7 (0x7F, 0xFF) is NaN; there are no infinities, so the
largest finite magnitude is 1.75 * 2**8 = 448 and the smallest subnormal is 2**-9.

Encoding is "round to nearest, ties to even, saturate to the largest finite value":
the nearest representable value is chosen, an exact tie goes to the code whose
mantissa least significant bit is 0, magnitudes above 448 clamp to 448, and the sign
of the input is kept (a negative value that rounds to zero gives 0x80).
"""

import math

import numpy as np

NAN_CODES = (0x7F, 0xFF)
MAX_FINITE = 448.0


def decode_code(code: int) -> float:
    """Value of one E4M3 code, evaluated from the field formula (float, exact)."""
    sign = -1.0 if code & 0x80 else 1.0
    exp_field = (code >> 3) & 0xF
    mant = code & 0x7
    if exp_field == 0xF and mant == 0x7:
        return math.nan
    if exp_field == 0:
        return sign * (mant / 8.0) * 2.0 ** -6
    return sign * (1.0 + mant / 8.0) * 2.0 ** (exp_field - 7)


# 256-entry decode table in float64 (every finite E4M3 value is exact in float64).
DECODE_F64 = np.array([decode_code(c) for c in range(256)], dtype=np.float64)

# The 127 non-negative finite values, codes 0x00..0x7E. They increase with the code,
# so the index of a value in this array is its code.
_POS_VALUES = DECODE_F64[:0x7F].copy()
assert np.all(np.diff(_POS_VALUES) > 0)


def decode(codes: np.ndarray) -> np.ndarray:
    """Decode an array of uint8 codes to float64 (NaN for 0x7F / 0xFF)."""
    return DECODE_F64[np.asarray(codes, dtype=np.uint8)]


def encode(x: np.ndarray) -> np.ndarray:
    """Encode finite float32 values to E4M3 codes (RNE, ties to even, saturating).

    The magnitude is clamped to 448, then the two neighbouring representable values
    are found by binary search and the nearer one is taken; distances are formed in
    float64, where the difference of two such float32 numbers is exact, so ties are
    detected exactly. NaN inputs are outside the method's domain.
    """
    x = np.asarray(x, dtype=np.float32)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x).astype(np.float64), MAX_FINITE)
    hi = np.searchsorted(_POS_VALUES, a, side="left")  # first value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    return code | (neg.astype(np.uint8) << 7)


def encode_bruteforce(x: np.ndarray) -> np.ndarray:
    """Slow independent encoder: arg-min of the distance to all 127 magnitudes.

    Used only to pin :func:`encode`. Ties are resolved by preferring the even code.
    """
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x).astype(np.float64), MAX_FINITE)
    dist = np.abs(a[:, None] - _POS_VALUES[None, :])  # [n, 127]
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among the (one or two) nearest codes prefer the even one
    even = (np.arange(0x7F) % 2 == 0)[None, :]
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    code = np.where(has_even, pick_even.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)
    return code | (neg.astype(np.uint8) << 7)
