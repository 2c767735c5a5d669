"""GPU parity of the grouped GEMM launch (puro_fp8_gemm_blockwise_grouped).

* Every problem of a group gives bit for bit what puro_fp8_gemm_blockwise gives for it
  alone, when both use the same kernel shape (all problems with more than 128 output rows:
  CTA pairs): the same tiles, with the same order of additions, only scheduled together.
  Groups of 1 to 4 problems of different M, N and K (so tiles of different length share
  the launch), all three layouts.
* A group with a problem of at most 128 rows runs on single CTAs; every problem is then
  checked against the FP64 oracle within the GEMM tolerance, and an exact-integer group
  bit for bit against the oracle rounded to BF16.
* Full size: the four weight gradients of a Qwen3-1.7B-shaped block at 8192 tokens (the
  benchmarked step's wgrads of one layer) in one launch, identical to four separate calls.
"""

import numpy as np
import pytest
import torch

from oracle import gemm as ogemm
from tests.parity import bf16_to_f64, check_gemm
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _b_scale_shape(layout, n, k):
    nb, kb = -(-n // 128), k // 128
    return {"fprop": (nb, kb), "dgrad": (kb, nb), "wgrad": (kb, n)}[layout]


def _random_problem(rng, layout, m, n, k):
    aq = rng.integers(0, 256, size=(m, k)).astype(np.uint8)
    bq = rng.integers(0, 256, size=(n, k)).astype(np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0x38
    bq[(bq & 0x7F) == 0x7F] = 0xB8
    a_s = (rng.random((k // 128, m)) * 2.0 ** -6).astype(np.float32)
    b_s = (rng.random(_b_scale_shape(layout, n, k)) * 2.0 ** -6).astype(np.float32)
    return aq, a_s, bq, b_s


def _dev(arrays):
    return tuple(torch.from_numpy(np.ascontiguousarray(a)).to(DEV) for a in arrays)


SHAPES = [(512, 768, 2048), (300, 256, 640), (1024, 520, 384), (256, 1024, 1152)]


@pytest.mark.parametrize("layout", ["fprop", "dgrad", "wgrad"])
@pytest.mark.parametrize("count", [1, 2, 4])
def test_grouped_equals_separate_calls(pf, layout, count):
    rng = np.random.default_rng(count * 7 + len(layout))
    host = [_random_problem(rng, layout, *SHAPES[i]) for i in range(count)]
    ops = [_dev(h) for h in host]
    outs = [torch.zeros((h[0].shape[0], h[2].shape[0]), dtype=torch.bfloat16, device=DEV) for h in host]
    pf.puro_fp8_gemm_blockwise_grouped([(*o, c) for o, c in zip(ops, outs)], layout)
    singles = [pf.gemm(*o, layout) for o in ops]
    pf.puro_fp8_sync_status()
    for i, (c, s) in enumerate(zip(outs, singles)):
        assert torch.equal(c.view(torch.int16), s.view(torch.int16)), f"problem {i} differs from its single call"
    # and the group against the oracle
    for (aq, a_s, bq, b_s), c in zip(host, outs):
        ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)
        an, bn = ogemm.row_col_norms(aq, a_s, bq, b_s, layout)
        check_gemm(bf16_to_f64(c), ref, an, bn, f"grouped {layout}")


@pytest.mark.parametrize("layout", ["fprop", "wgrad"])
def test_group_with_small_problem_on_single_ctas(pf, layout):
    """A problem of 77 rows sends the whole group to the single-CTA kernel; exact-integer
    operands make every output the oracle's exact value rounded to BF16."""
    rng = np.random.default_rng(21)
    codes = np.array([0x00, 0x30, 0xB0, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)
    host = []
    for m, n, k in ((77, 264, 384), (300, 512, 1024), (128, 8, 128)):
        aq = codes[rng.integers(0, 7, size=(m, k))]
        bq = codes[rng.integers(0, 7, size=(n, k))]
        a_s = (2.0 ** rng.integers(-3, 3, size=(k // 128, m))).astype(np.float32)
        b_s = (2.0 ** rng.integers(-3, 3, size=_b_scale_shape(layout, n, k))).astype(np.float32)
        host.append((aq, a_s, bq, b_s))
    ops = [_dev(h) for h in host]
    outs = [torch.zeros((h[0].shape[0], h[2].shape[0]), dtype=torch.bfloat16, device=DEV) for h in host]
    pf.puro_fp8_gemm_blockwise_grouped([(*o, c) for o, c in zip(ops, outs)], layout)
    pf.puro_fp8_sync_status()
    for (aq, a_s, bq, b_s), c in zip(host, outs):
        ref = ogemm.gemm_ref(aq, a_s, bq, b_s, layout)
        assert np.array_equal(ref, ref.astype(np.float32).astype(np.float64))
        want = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
        assert torch.equal(c.cpu().view(torch.int16), want)


def test_layer_wgrads_grouped_at_8192_tokens(pf):
    T = 8192
    fwd = wl.layer_forward(4, T, DEV, layer=1)
    grads = wl.layer_grads(4, T, DEV, layer=1)
    problems, singles = [], []
    for (name, x, w), (_, dy) in zip(fwd, grads):
        dyt, dyst = pf.quantize_1x128_transposed(dy)
        xt, xst = pf.quantize_1x128_transposed(x)
        out = torch.empty(w.shape, dtype=torch.bfloat16, device=DEV)
        problems.append((dyt, dyst, xt, xst, out))
        singles.append(pf.gemm(dyt, dyst, xt, xst, "wgrad"))
    pf.puro_fp8_gemm_blockwise_grouped(problems, "wgrad")
    pf.puro_fp8_sync_status()
    for (_, _, _, _, out), s, (name, _, _) in zip(problems, singles, fwd):
        assert torch.equal(out.view(torch.int16), s.view(torch.int16)), f"{name} wgrad differs"
