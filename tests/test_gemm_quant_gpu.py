"""GPU parity of the GEMM whose epilogue also quantises its output (puro_fp8_gemm_blockwise_quant).

The entry point writes C (BF16) and the 1x128 quantisation of that C along N, the input of
a following linear layer.

* Exact-integer operands (codes in {0, +-0.5, +-1, +-2}, power-of-two scales): every FP32
  partial and sum is exact, so the oracle knows C exactly. It rounds its own exact C to
  BF16 and quantises that with its 1x128 routine; C, the codes and the scales must match
  bit for bit. Both layouts, single-CTA and CTA-pair tiles, ragged M.
* Random codes over several tiles: C within the GEMM tolerance of the FP64 oracle, and the
  codes and scales identical to the library's separate 1x128 quantiser applied to that C
  (itself checked bit-exactly against the oracle in test_quant_gpu.py).
* Full size (the benchmarked step's QKV fprop and gate/up dgrad at 8192 tokens, through the
  library's quantisers): C sampled against the oracle, codes and scales compared in full
  with the separate quantiser of C.
"""

import numpy as np
import pytest
import torch

from oracle import gemm as ogemm
from oracle import quant as oquant
from tests.parity import bf16_to_f64, check_gemm, oracle_gemm_sampled
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _b_scale_shape(layout, n, k):
    nb, kb = -(-n // 128), k // 128
    return {"fprop": (nb, kb), "dgrad": (kb, nb)}[layout]


def _to_dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in arrays]


def _bits(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _eq(got, want, what):
    got = got.cpu().numpy()
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), np.asarray(want).view(np.uint32)
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{what}: {len(mism)} mismatches, first at {mism[:4].tolist()}"


@pytest.mark.parametrize("layout", ["fprop", "dgrad"])
@pytest.mark.parametrize("m,n,k", [(100, 256, 256), (200, 384, 384), (300, 512, 1024)])
def test_exact_integer_case_bitexact(pf, layout, m, n, k):
    rng = np.random.default_rng(3 * m + n + k)
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    aq = codes[rng.integers(0, 7, size=(m, k))]
    bq = codes[rng.integers(0, 7, size=(n, k))]
    a_s = (2.0 ** rng.integers(-3, 3, size=(k // 128, m))).astype(np.float32)
    b_s = (2.0 ** rng.integers(-3, 3, size=_b_scale_shape(layout, n, k))).astype(np.float32)
    aq[rng.random(m) < 0.1] = 0  # some all-zero rows of A: all-zero output groups (s = 0)
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)  # exact in float64 and in FP32
    assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))
    c_bf16 = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16)   # the oracle's own rounding
    q_ref, s_ref = oquant.quant_1x128(_bits(c_bf16))
    c, cq, cs = pf.gemm_quant(*_to_dev(aq, a_s, bq, b_s), layout)
    pf.puro_fp8_sync_status()
    _eq(c.view(torch.int16), c_bf16.view(torch.int16).numpy(), "C")
    _eq(cq, q_ref, "codes")
    _eq(cs, s_ref, "scales")


@pytest.mark.parametrize("layout", ["fprop", "dgrad"])
@pytest.mark.parametrize("m,n,k", [(130, 256, 640), (512, 768, 2048), (77, 1024, 256)])
def test_random_codes_match_separate_quantiser(pf, layout, m, n, k):
    rng = np.random.default_rng(11 * m + n)
    aq = rng.integers(0, 256, size=(m, k)).astype(np.uint8)
    bq = rng.integers(0, 256, size=(n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x38
    bq[(bq & 0x7F) == 0x7F] = 0xB8
    a_s = (rng.random((k // 128, m)) * 2.0 ** -6).astype(np.float32)
    b_s = (rng.random(_b_scale_shape(layout, n, k)) * 2.0 ** -6).astype(np.float32)
    ops = _to_dev(aq, a_s, bq, b_s)
    c, cq, cs = pf.gemm_quant(*ops, layout)
    plain = pf.gemm(*ops, layout)
    q2, s2 = pf.quantize_1x128(c)
    pf.puro_fp8_sync_status()
    ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)
    an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, layout)
    check_gemm(bf16_to_f64(c), ref, an, bn, f"{layout} {m}x{n}x{k}")
    _eq(c.view(torch.int16), plain.view(torch.int16).cpu().numpy(), "C vs the plain GEMM")
    _eq(cq, q2.cpu().numpy(), "codes vs the separate quantiser")
    _eq(cs, s2.cpu().numpy(), "scales vs the separate quantiser")


def test_full_size_step_shapes(pf):
    T = 8192
    (name, x, w) = wl.layer_forward(4, T, DEV, layer=0)[0]       # QKV: fprop N = 4096
    (name2, x2, w2) = wl.layer_forward(4, T, DEV, layer=0)[2]    # gate/up weight: dgrad N = 2048
    (_, dy2) = wl.layer_grads(4, T, DEV, layer=0)[2]
    xq, xs = pf.quantize_1x128(x)
    wq, wqt, ws = pf.quantize_128x128(w)
    dyq, dys = pf.quantize_1x128(dy2)
    _, w2t, w2s = pf.quantize_128x128(w2)
    rows = np.sort(np.random.default_rng(1).choice(T, size=32, replace=False))
    for layout, (a, a_s, bq, b_s), a_bf, b_bf, nb in (
            ("fprop", (xq, xs, wq, ws), x, w, [0, 17, 31]),
            ("dgrad", (dyq, dys, w2t, w2s), dy2, w2, [0, 9, 15])):
        c, cq, cs = pf.gemm_quant(a, a_s, bq, b_s, layout)
        q2, s2 = pf.quantize_1x128(c)
        pf.puro_fp8_sync_status()
        assert torch.equal(cq, q2), f"{layout}: codes differ from the separate quantiser"
        assert torch.equal(cs.view(torch.int32), s2.view(torch.int32)), f"{layout}: scales differ"
        c_ref, cols, an, bn = oracle_gemm_sampled(layout, a_bf, b_bf, rows, nb)
        got = bf16_to_f64(c[torch.as_tensor(rows, device=DEV)][:, torch.as_tensor(cols, device=DEV)])
        check_gemm(got, c_ref, an, bn, f"{layout} fused, 8192 tokens")
        del c, cq, cs, q2, s2
