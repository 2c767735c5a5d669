"""Pins of the oracle's FP64 reference contraction.

* exact rational brute force (``fractions.Fraction``, scalar triple loop, codes decoded
  from the field formula one by one) on tiny non-square shapes with M and N tails, for
  all three operand layouts; a transposed operand, a swapped scale index or a dropped
  K block fails it;
* a closed-form exact-integer case: ternary-and-power-of-two codes with power-of-two
  scales, where C is an integer combination computable in int64;
* linearity in the scales (doubling As doubles C exactly);
* the method's own premise, informational: on the outlier-channel GEMM, blockwise
  scales give a smaller error than one scale per tensor.
"""

from fractions import Fraction

import numpy as np
import torch

from oracle import e4m3, gemm, quant
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38  # no NaN codes
    return c


def _rand_scales(rng, shape):
    return (rng.random(shape) * 2.0 ** rng.integers(-12, 4, size=shape)).astype(np.float32)


def _b_scale(layout, b_s, n, k):
    if layout == "fprop":
        return b_s[n // 128][k // 128]
    if layout == "dgrad":
        return b_s[k // 128][n // 128]
    return b_s[k // 128][n]


def _brute(aq, a_s, bq, b_s, layout):
    m_, k_ = aq.shape
    n_ = bq.shape[0]
    out = [[Fraction(0)] * n_ for _ in range(m_)]
    for m in range(m_):
        for n in range(n_):
            acc = Fraction(0)
            for k in range(k_):
                av = Fraction(e4m3.decode_code(int(aq[m, k]))) * Fraction(float(a_s[k // 128][m]))
                bv = Fraction(e4m3.decode_code(int(bq[n, k]))) * Fraction(float(_b_scale(layout, b_s, n, k)))
                acc += av * bv
            out[m][n] = acc
    return out


def _b_scale_shape(layout, n, k):
    nb, kb = -(-n // 128), k // 128
    return {"fprop": (nb, kb), "dgrad": (kb, nb), "wgrad": (kb, n)}[layout]


def test_bruteforce_rational_all_layouts_with_tails():
    rng = np.random.default_rng(5)
    m, n, k = 3, 130, 256
    for layout in gemm.LAYOUTS:
        aq, bq = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
        a_s = _rand_scales(rng, (k // 128, m))
        b_s = _rand_scales(rng, _b_scale_shape(layout, n, k))
        ref = gemm.gemm_ref(aq, a_s, bq, b_s, layout)
        exact = _brute(aq, a_s, bq, b_s, layout)
        mag = np.abs(gemm.dequant_1x128(aq, a_s)) @ np.abs(gemm.dequant_b(bq, b_s, layout)).T
        for i in range(m):
            for j in range(n):
                assert abs(Fraction(float(ref[i, j])) - exact[i][j]) <= Fraction(mag[i, j]) * Fraction(1, 2 ** 45), (layout, i, j)


def test_exact_integer_closed_form():
    """Codes in {0, +-0.5, +-1, +-2}, scales 2^e: C = sum_kb 2^(ea+eb) * integer dot."""
    rng = np.random.default_rng(6)
    m, n, k = 40, 136, 384
    vals = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0])
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    ia = rng.integers(0, 7, size=(m, k))
    ib = rng.integers(0, 7, size=(n, k))
    aq, bq = codes[ia], codes[ib]
    a_int, b_int = (vals[ia] * 2).astype(np.int64), (vals[ib] * 2).astype(np.int64)  # x2 -> integers
    kb = k // 128
    ea = rng.integers(-6, 6, size=(kb, m))
    for layout in gemm.LAYOUTS:
        eb = rng.integers(-6, 6, size=_b_scale_shape(layout, n, k))
        a_s = (2.0 ** ea).astype(np.float32)
        b_s = (2.0 ** eb).astype(np.float32)
        want = np.zeros((m, n))
        for j in range(kb):
            part = a_int[:, j * 128:(j + 1) * 128] @ b_int[:, j * 128:(j + 1) * 128].T  # int64
            if layout == "fprop":
                sb = 2.0 ** eb[np.arange(n) // 128, j]
            elif layout == "dgrad":
                sb = 2.0 ** eb[j, np.arange(n) // 128]
            else:
                sb = 2.0 ** eb[j, :]
            want += part / 4.0 * (2.0 ** ea[j])[:, None] * sb[None, :]
        got = gemm.gemm_ref(aq, a_s, bq, b_s, layout)
        assert np.array_equal(got, want), layout


def test_linearity_in_scales():
    rng = np.random.default_rng(8)
    m, n, k = 16, 64, 256
    aq, bq = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
    a_s, b_s = _rand_scales(rng, (2, m)), _rand_scales(rng, (2, n))
    c1 = gemm.gemm_ref(aq, a_s, bq, b_s, "wgrad")
    c2 = gemm.gemm_ref(aq, a_s * np.float32(2), bq, b_s, "wgrad")
    assert np.array_equal(c2, 2 * c1)


def test_rows_helper_matches_full():
    rng = np.random.default_rng(9)
    aq, bq = _rand_codes(rng, (50, 256)), _rand_codes(rng, (70, 256))
    a_s, b_s = _rand_scales(rng, (2, 50)), _rand_scales(rng, (1, 2))
    full = gemm.gemm_ref(aq, a_s, bq, b_s, "fprop")
    rows = [0, 7, 49]
    part = gemm.gemm_ref_rows(aq, a_s, bq, b_s, "fprop", rows)
    # same sums, BLAS may order them differently for a 3-row product
    assert np.allclose(part, full[rows], rtol=1e-12, atol=1e-12 * np.abs(full).max())


def test_blockwise_beats_per_tensor_on_outlier_channels():
    a, w = wl.small_gemm(seed=0)
    a_bits, w_bits = wl.bf16_bits(a), wl.bf16_bits(w)
    exact = quant.bf16_bits_to_f32(a_bits).astype(np.float64) @ quant.bf16_bits_to_f32(w_bits).astype(np.float64).T
    aq, a_s = quant.quant_1x128(a_bits)
    wq, _, w_s = quant.quant_128x128(w_bits)
    blockwise = gemm.gemm_ref(aq, a_s, wq, w_s, "fprop")
    # one scale for the whole activation tensor
    qa_t, sa_t = quant.quantize_groups(quant.bf16_bits_to_f32(a_bits).reshape(1, -1))
    a_t = e4m3.decode(qa_t.reshape(a.shape)) * np.float64(sa_t[0])
    per_tensor = a_t @ gemm.dequant_weight_blocks(wq, w_s).T
    err_b = np.linalg.norm(blockwise - exact) / np.linalg.norm(exact)
    err_t = np.linalg.norm(per_tensor - exact) / np.linalg.norm(exact)
    assert err_b < err_t
    assert err_b < 0.05


def test_wgrad_accumulate_is_input_plus_contraction():
    """The accumulation reference adds the wgrad contraction to the given buffer: zero
    input gives the contraction itself, and accumulating twice equals adding 2 dW (exact
    here: integer-valued operands)."""
    rng = np.random.default_rng(5)
    codes = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)   # 0, +-1, +-2
    m, n, k = 40, 24, 256
    aq = codes[rng.integers(0, 5, size=(m, k))]
    bq = codes[rng.integers(0, 5, size=(n, k))]
    a_s = np.ones((k // 128, m), np.float32)
    b_s = np.full((k // 128, n), 2.0, np.float32)
    dw = gemm.gemm_ref(aq, a_s, bq, b_s, "wgrad")
    assert np.array_equal(gemm.wgrad_accumulate_ref(np.zeros((m, n), np.float32), aq, a_s, bq, b_s), dw)
    c0 = rng.integers(-1000, 1000, size=(m, n)).astype(np.float32)
    once = gemm.wgrad_accumulate_ref(c0, aq, a_s, bq, b_s)
    twice = gemm.wgrad_accumulate_ref(once, aq, a_s, bq, b_s)
    assert np.array_equal(twice, c0 + 2 * dw)
    # brute force on a tiny case: dW[m, n] = sum_t dY[t, m] X[t, n] with the token scales
    brute = np.zeros((m, n))
    dec = e4m3.decode(aq) * np.repeat(a_s.T, 128, axis=1), e4m3.decode(bq) * np.repeat(b_s.T, 128, axis=1)
    for i in range(m):
        for j in range(n):
            brute[i, j] = float(np.dot(dec[0][i], dec[1][j]))
    assert np.array_equal(once, c0 + brute)


def _brute_norm(values):
    """sqrt of an exactly accumulated sum of squares (Fraction), as a float."""
    ss = sum((v * v for v in values), Fraction(0))
    return float(ss) ** 0.5


def test_row_col_norms_bruteforce_all_layouts_with_tails():
    """row_col_norms gives ||A_deq[m, :]||_2 and ||B_deq[n, :]||_2, the factors of the GEMM
    tolerance's elementwise bound. Brute force: every code decoded from the field formula,
    times its own scale looked up with the layout's index rule, squared and summed exactly.
    Scales are random and far from 1 and the scale grids are not square, so squared norms,
    norms of the raw codes, or the B scales of another layout all fail this."""
    rng = np.random.default_rng(11)
    m, n, k = 5, 259, 384   # an M tail, and an N tail that ends a 128-row weight block early
    for layout in gemm.LAYOUTS:
        aq, bq = _rand_codes(rng, (m, k)), _rand_codes(rng, (n, k))
        a_s = _rand_scales(rng, (k // 128, m))
        b_s = _rand_scales(rng, _b_scale_shape(layout, n, k))
        an, bn = gemm.row_col_norms(aq, a_s, bq, b_s, layout)
        assert an.shape == (m,) and bn.shape == (n,)
        for i in range(m):
            want = _brute_norm([Fraction(e4m3.decode_code(int(aq[i, kk]))) * Fraction(float(a_s[kk // 128][i]))
                                for kk in range(k)])
            assert abs(an[i] - want) <= 1e-12 * want, (layout, "A", i)
        for j in range(n):
            want = _brute_norm([Fraction(e4m3.decode_code(int(bq[j, kk])))
                                * Fraction(float(_b_scale(layout, b_s, j, kk))) for kk in range(k)])
            assert abs(bn[j] - want) <= 1e-12 * want, (layout, "B", j)
        # the rows= form (used on sampled full-size outputs) gives the same A norms
        rows = [4, 0, 2]
        an_rows, bn_rows = gemm.row_col_norms(aq, a_s, bq, b_s, layout, rows=rows)
        assert np.array_equal(an_rows, an[rows]) and np.array_equal(bn_rows, bn)
