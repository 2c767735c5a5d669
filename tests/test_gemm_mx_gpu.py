"""GPU parity of the block-scaled GEMM (power-of-two UE8M0 scales, puro_fp8_mx_gemm) against
the FP64 oracle with the scales 2^(byte - 127).

* exact-integer case: codes in {0, +-0.5, +-1, +-2} and scale bytes 124..129 make every
  partial and sum exact in FP32, so the BF16 output must equal the oracle's result rounded
  to BF16 bit for bit, in all three layouts, with M and N tails;
* random codes and scale bytes over several tiles with ragged M / N tails (tolerance);
* end to end from BF16: the GPU's power-of-two quantisers and the block-scaled GEMM against
  oracle.mx's quantisers and the FP64 GEMM, for the small outlier GEMM and a Qwen3-1.7B
  layer's linears at 8192 tokens (sampled rows and column blocks);
* the same operands through the FP32-scale GEMM (puro_fp8_gemm_blockwise with the bytes
  turned into float scales) give the same result within the tolerance.
Tolerance: relative Frobenius <= 2e-3 and |err| <= 1e-2 ||a_m|| ||b_n|| (tests/parity.py).
"""

import numpy as np
import pytest
import torch

from oracle import gemm as ogemm
from oracle import mx as omx
from tests.parity import bf16_to_f64, check_gemm, host_bits, oracle_gemm_sampled
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"
LAYOUTS = ("fprop", "dgrad", "wgrad")


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _b_scale_shape(layout, n, k):
    nb, kb = -(-n // 128), k // 128
    return {"fprop": (nb, kb), "dgrad": (kb, nb), "wgrad": (kb, n)}[layout]


def _to_dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in arrays]


def _bits(c):
    return c.cpu().view(torch.int16).numpy()


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(128, 256, 128), (200, 264, 384), (1, 8, 128), (300, 520, 1024)])
def test_exact_integer_case_bitexact(pf, layout, m, n, k):
    rng = np.random.default_rng(m + n + k + 11)
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    aq = codes[rng.integers(0, 7, size=(m, k))]
    bq = codes[rng.integers(0, 7, size=(n, k))]
    a_b = rng.integers(124, 130, size=(k // 128, m)).astype(np.uint8)
    b_b = rng.integers(124, 130, size=_b_scale_shape(layout, n, k)).astype(np.uint8)
    ref = ogemm.gemm_ref(aq, omx.scales_from_ue8m0(a_b), bq, omx.scales_from_ue8m0(b_b), layout)
    assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))
    want = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = _bits(pf.mx_gemm(*_to_dev(aq, a_b, bq, b_b), layout))
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} mismatches, first at {mism[:4].tolist()}"


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(130, 136, 640), (512, 768, 2048), (77, 1000, 256), (384, 2056, 384)])
def test_random_codes_tolerance(pf, layout, m, n, k):
    rng = np.random.default_rng(7 * m + n + 1)
    aq = rng.integers(0, 256, size=(m, k)).astype(np.uint8)
    bq = rng.integers(0, 256, size=(n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x38
    bq[(bq & 0x7F) == 0x7F] = 0xB8
    a_b = rng.integers(112, 124, size=(k // 128, m)).astype(np.uint8)
    b_b = rng.integers(112, 124, size=_b_scale_shape(layout, n, k)).astype(np.uint8)
    a_s, b_s = omx.scales_from_ue8m0(a_b), omx.scales_from_ue8m0(b_b)
    c = pf.mx_gemm(*_to_dev(aq, a_b, bq, b_b), layout)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)
    an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, layout)
    check_gemm(bf16_to_f64(c), ref, an, bn, f"mx {layout} {m}x{n}x{k}")
    # the FP32-scale GEMM on the same operands, with the bytes as float scales
    c32 = pf.gemm(*_to_dev(aq, a_s, bq, b_s), layout)
    check_gemm(bf16_to_f64(c32), ref, an, bn, f"fp32-scale {layout} {m}x{n}x{k}")


def test_extreme_scale_bytes(pf):
    """Bytes at the ends of the range the quantisers produce (0 = 2^-127, 254 = 2^127) in
    pairs whose products stay representable: 2^-127 * 2^127 and the like."""
    m, n, k = 128, 256, 512
    rng = np.random.default_rng(5)
    codes = np.array([0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    aq = codes[rng.integers(0, 6, size=(m, k))]
    bq = codes[rng.integers(0, 6, size=(n, k))]
    lo = rng.integers(0, 4, size=(k // 128, m))
    a_b = np.where(rng.random((k // 128, 1)) < 0.5, lo, 254 - lo).astype(np.uint8)   # per K block
    b_b = (254 - a_b[:, :1].astype(np.int64) + rng.integers(-2, 3, size=(k // 128, n))).clip(0, 254)
    b_b = b_b.astype(np.uint8)
    a_s, b_s = omx.scales_from_ue8m0(a_b), omx.scales_from_ue8m0(b_b)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, "wgrad")
    c = pf.mx_gemm(*_to_dev(aq, a_b, bq, b_b), "wgrad")
    an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, "wgrad")
    check_gemm(bf16_to_f64(c), ref, an, bn, "extreme scale bytes")


def test_small_outlier_gemm_end_to_end(pf):
    a, w = wl.small_gemm(seed=0)
    aq, a_b = pf.quantize_1x128_pow2(a.to(DEV))
    wq, wqt, w_b = pf.quantize_128x128_pow2(w.to(DEV))
    c = pf.mx_gemm(aq, a_b, wq, w_b, "fprop")
    aq_r, ab_r = omx.quant_1x128_pow2(host_bits(a))
    wq_r, _, wb_r = omx.quant_128x128_pow2(host_bits(w))
    a_s, w_s = omx.scales_from_ue8m0(ab_r), omx.scales_from_ue8m0(wb_r)
    ref = ogemm.gemm_ref(aq_r, a_s, wq_r, w_s, "fprop")
    an, bn = ogemm.row_col_norms(aq_r, a_s, wq_r, w_s, "fprop")
    check_gemm(bf16_to_f64(c), ref, an, bn, "small outlier GEMM, power-of-two scales")


def _sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(n, k), replace=False))


def _check_sampled(c_gpu, layout, a, b, rows, nblocks, what):
    c_ref, cols, an, bn = oracle_gemm_sampled(layout, a, b, rows, nblocks, scales="pow2")
    got = bf16_to_f64(c_gpu[torch.as_tensor(rows, device=DEV)][:, torch.as_tensor(cols, device=DEV)])
    check_gemm(got, c_ref, an, bn, what)


def test_layer_full_size_sampled(pf):
    T = 8192
    fwd = wl.layer_forward(1, T, DEV, layer=0)
    grads = wl.layer_grads(2, T, DEV, layer=0)
    for (name, x, w), (_, dy) in zip(fwd, grads):
        xq, xb = pf.quantize_1x128_pow2(x)
        wq, wqt, wb = pf.quantize_128x128_pow2(w)
        dyt, dybt, dyq, dyb = pf.quantize_1x128_transposed_pow2(dy, dual=True)
        xt, xbt = pf.quantize_1x128_transposed_pow2(x)
        y = pf.mx_gemm(xq, xb, wq, wb, "fprop")
        dx = pf.mx_gemm(dyq, dyb, wqt, wb, "dgrad")
        dw = pf.mx_gemm(dyt, dybt, xt, xbt, "wgrad")
        n_out, k_in = w.shape
        rows_t = _sample(T, 40, seed=1)
        _check_sampled(y, "fprop", x, w, rows_t, _sample(n_out // 128, 2, 2), f"{name} fprop")
        _check_sampled(dx, "dgrad", dy, w, rows_t, _sample(k_in // 128, 2, 3), f"{name} dgrad")
        _check_sampled(dw, "wgrad", dy, x, _sample(n_out, 40, 4), _sample(k_in // 128, 2, 5),
                       f"{name} wgrad")
    pf.puro_fp8_sync_status()
