"""GPU parity of the blockwise GEMM against the FP64 oracle.

* exact-integer case: codes in {0, +-0.5, +-1, +-2} and power-of-two scales make every
  FP32 partial and sum exact, so the BF16 output must equal the oracle's result rounded
  to BF16 bit for bit, in all three layouts, with M and N tails;
* hand-built random codes and scales over several tiles with ragged M / N tails;
* the small outlier GEMM (256 x 384 x 512) end to end: GPU quantisers + GPU GEMM
  against oracle quantisers + FP64 GEMM from the same BF16 inputs;
* full-size Qwen3-1.7B-shaped layer (4096 tokens, all four linears, fprop, dgrad and
  wgrad) and the LM head, on sampled output rows and column blocks.
Tolerance: relative Frobenius <= 2e-3 and |err| <= 1e-2 ||a_m|| ||b_n|| (tests/parity.py).
"""

import numpy as np
import pytest
import torch

from oracle import gemm as ogemm
from oracle import quant as oquant
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


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(128, 256, 128), (200, 264, 384), (1, 8, 128), (300, 520, 1024)])
def test_exact_integer_case_bitexact(pf, layout, m, n, k):
    rng = np.random.default_rng(m + n + k)
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    aq = codes[rng.integers(0, 7, size=(m, k))]
    bq = codes[rng.integers(0, 7, size=(n, k))]
    # partials are multiples of 1/4 below 2^9; scale products 2^-6 .. 2^4 keep every
    # partial, product and running FP32 sum within 24 significant bits: exact
    a_s = (2.0 ** rng.integers(-3, 3, size=(k // 128, m))).astype(np.float32)
    b_s = (2.0 ** rng.integers(-3, 3, size=_b_scale_shape(layout, n, k))).astype(np.float32)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)  # exact in float64 and in FP32
    assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))
    want = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    c = pf.gemm(*_to_dev(aq, a_s, bq, b_s), layout)
    got = c.cpu().view(torch.int16).numpy()
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} mismatches, first at {mism[:4].tolist()}"


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(130, 136, 640), (512, 768, 2048), (77, 1000, 256)])
def test_random_codes_tolerance(pf, layout, m, n, k):
    rng = np.random.default_rng(7 * m + n)
    aq = rng.integers(0, 256, size=(m, k)).astype(np.uint8)
    bq = rng.integers(0, 256, size=(n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x38
    bq[(bq & 0x7F) == 0x7F] = 0xB8
    a_s = (rng.random((k // 128, m)) * 2.0 ** -6).astype(np.float32)
    b_s = (rng.random(_b_scale_shape(layout, n, k)) * 2.0 ** -6).astype(np.float32)
    c = pf.gemm(*_to_dev(aq, a_s, bq, b_s), layout)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)
    an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, layout)
    check_gemm(bf16_to_f64(c), ref, an, bn, f"{layout} {m}x{n}x{k}")


def test_small_outlier_gemm_end_to_end(pf):
    a, w = wl.small_gemm(seed=0)
    a_d, w_d = a.to(DEV), w.to(DEV)
    aq, a_s = pf.quantize_1x128(a_d)
    wq, wqt, w_s = pf.quantize_128x128(w_d)
    c = pf.gemm(aq, a_s, wq, w_s, "fprop")
    aq_r, as_r = oquant.quant_1x128(host_bits(a))
    wq_r, _, ws_r = oquant.quant_128x128(host_bits(w))
    ref = ogemm.gemm_ref(aq_r, as_r, wq_r, ws_r, "fprop")
    an, bn = ogemm.row_col_norms(aq_r, as_r, wq_r, ws_r, "fprop")
    check_gemm(bf16_to_f64(c), ref, an, bn, "small outlier GEMM")


def _layer_step(pf, x, w, dy):
    """All three GEMMs of one linear layer through the library."""
    xq, xs = pf.quantize_1x128(x)
    wq, wqt, ws = pf.quantize_128x128(w)
    dyt, dyst, dyq, dys = pf.quantize_1x128_transposed(dy, dual=True)
    xt, xst = pf.quantize_1x128_transposed(x)
    y = pf.gemm(xq, xs, wq, ws, "fprop")
    dx = pf.gemm(dyq, dys, wqt, ws, "dgrad")
    dw = pf.gemm(dyt, dyst, xt, xst, "wgrad")
    return y, dx, dw


def _check_sampled(c_gpu, layout, a, b, rows, nblocks, what):
    c_ref, cols, an, bn = oracle_gemm_sampled(layout, a, b, rows, nblocks)
    got = bf16_to_f64(c_gpu[torch.as_tensor(rows, device=DEV)][:, torch.as_tensor(cols, device=DEV)])
    check_gemm(got, c_ref, an, bn, what)


def _sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(n, k), replace=False))


def test_layer_full_size_sampled(pf):
    T = 4096
    fwd = wl.layer_forward(1, T, DEV)
    grads = wl.layer_grads(2, T, DEV)
    for (name, x, w), (_, dy) in zip(fwd, grads):
        y, dx, dw = _layer_step(pf, x, w, dy)
        n_out, k_in = w.shape
        rows_t = _sample(T, 48, seed=1)
        _check_sampled(y, "fprop", x, w, rows_t, _sample(n_out // 128, 3, 2), f"{name} fprop")
        _check_sampled(dx, "dgrad", dy, w, rows_t, _sample(k_in // 128, 3, 3), f"{name} dgrad")
        _check_sampled(dw, "wgrad", dy, x, _sample(n_out, 48, 4), _sample(k_in // 128, 2, 5),
                       f"{name} wgrad")


@pytest.mark.parametrize("tokens", [4096, 8192])
def test_lm_head_full_size_sampled(pf, tokens):
    h, w, dl = wl.lm_head(3, tokens, DEV)
    logits, dh, dw = _layer_step(pf, h, w, dl)
    nb_vocab = w.shape[0] // 128
    rows_t = _sample(tokens, 32, seed=1)
    _check_sampled(logits, "fprop", h, w, rows_t, list(_sample(nb_vocab - 1, 2, 2)) + [nb_vocab - 1],
                   "lm_head fprop")
    _check_sampled(dh, "dgrad", dl, w, rows_t, _sample(16, 2, 3), "lm_head dgrad")
    _check_sampled(dw, "wgrad", dl, h, _sample(w.shape[0], 32, 4), _sample(16, 2, 5), "lm_head wgrad")


def test_status_clean_after_parity_runs(pf):
    pf.puro_fp8_sync_status()


# ------------------------------------------------------------------ FP32 wgrad accumulation

def _exact_integer_operands(layout, m, n, k, seed):
    """Codes in {0, +-0.5, +-1, +-2} and power-of-two scales (as in the exact-integer case
    above): with K <= 1024 every FP32 partial, product and sum is exact."""
    rng = np.random.default_rng(seed)
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    aq = codes[rng.integers(0, 7, size=(m, k))]
    bq = codes[rng.integers(0, 7, size=(n, k))]
    a_s = (2.0 ** rng.integers(-3, 3, size=(k // 128, m))).astype(np.float32)
    b_s = (2.0 ** rng.integers(-3, 3, size=_b_scale_shape(layout, n, k))).astype(np.float32)
    return aq, a_s, bq, b_s


# puro_fp8_gemm_wgrad_acc_f32: C (FP32) += the wgrad product, one FP32 add per element.

@pytest.mark.parametrize("m,n,k", [(128, 256, 128), (200, 264, 384), (1, 8, 128), (300, 520, 1024)])
def test_wgrad_acc_f32_exact_integer_bitexact(pf, m, n, k):
    aq, a_s, bq, b_s = _exact_integer_operands("wgrad", m, n, k, 5 * m + n + k)
    rng = np.random.default_rng(m * n)
    c_in = rng.integers(-4096, 4096, size=(m, n)).astype(np.float32) / 4   # exact with the sums
    dw = ogemm.gemm_ref(aq, a_s, bq, b_s, "wgrad")
    c = torch.from_numpy(c_in).to(DEV)
    ops = _to_dev(aq, a_s, bq, b_s)
    pf.puro_fp8_gemm_wgrad_acc_f32(*ops, c)
    once = c.cpu().numpy().astype(np.float64)
    want = ogemm.wgrad_accumulate_ref(c_in, aq, a_s, bq, b_s)
    assert np.array_equal(want, want.astype(np.float32).astype(np.float64))
    mism = np.argwhere(once != want)
    assert mism.size == 0, f"{len(mism)} mismatches, first at {mism[:4].tolist()}"
    pf.puro_fp8_gemm_wgrad_acc_f32(*ops, c)      # accumulating again adds dW once more
    assert np.array_equal(c.cpu().numpy().astype(np.float64), c_in + 2 * dw)


def test_wgrad_acc_f32_random_codes_tolerance(pf):
    m, n, k = 520, 776, 1280
    rng = np.random.default_rng(17)
    aq = rng.integers(0, 256, size=(m, k)).astype(np.uint8)
    bq = rng.integers(0, 256, size=(n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x38
    bq[(bq & 0x7F) == 0x7F] = 0xB8
    a_s = (rng.random((k // 128, m)) * 2.0 ** -6).astype(np.float32)
    b_s = (rng.random((k // 128, n)) * 2.0 ** -6).astype(np.float32)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, "wgrad")
    c_in = (rng.standard_normal((m, n)) * np.abs(ref).mean()).astype(np.float32)
    c = torch.from_numpy(c_in).to(DEV)
    pf.puro_fp8_gemm_wgrad_acc_f32(*_to_dev(aq, a_s, bq, b_s), c)
    got = c.cpu().numpy().astype(np.float64)
    an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, "wgrad")
    # the added product meets the GEMM tolerance; the final FP32 add rounds once more
    check_gemm(got - c_in.astype(np.float64), ref, an, bn, "wgrad acc f32",
               extra_abs=np.abs(c_in.astype(np.float64) + ref) * 2.0 ** -23)
    assert np.allclose(got, ogemm.wgrad_accumulate_ref(c_in, aq, a_s, bq, b_s), rtol=0,
                       atol=float((1e-2 * an[:, None] * bn[None, :]).max()))


def test_wgrad_acc_f32_layer_full_size_sampled(pf):
    """gate/up weight gradient of a Qwen3-1.7B-shaped layer at 4096 tokens, from the
    workload's BF16 tensors through the library's quantisers, accumulated onto a nonzero
    FP32 main gradient; sampled against the oracle."""
    T = 4096
    (name, x, w) = wl.layer_forward(1, T, DEV)[2]
    (_, dy) = wl.layer_grads(2, T, DEV)[2]
    dyt, dyst = pf.quantize_1x128_transposed(dy)
    xt, xst = pf.quantize_1x128_transposed(x)
    n_out, k_in = w.shape
    main = torch.randn(n_out, k_in, device=DEV) * 1e-3
    start = main.clone()
    pf.puro_fp8_gemm_wgrad_acc_f32(dyt, dyst, xt, xst, main)
    rows, nblocks = _sample(n_out, 48, 4), _sample(k_in // 128, 2, 5)
    c_ref, cols, an, bn = oracle_gemm_sampled("wgrad", dy, x, rows, nblocks)
    ri, ci = torch.as_tensor(rows, device=DEV), torch.as_tensor(cols, device=DEV)
    added = (main[ri][:, ci].double() - start[ri][:, ci].double()).cpu().numpy()
    check_gemm(added, c_ref, an, bn, f"{name} wgrad acc f32",
               extra_abs=np.abs(start[ri][:, ci].double().cpu().numpy() + c_ref) * 2.0 ** -23)
