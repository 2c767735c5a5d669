"""GPU parity at the benchmarked micro-step's own sizes: 8192 tokens (2 x 4096), the
benchmark's input seed, the first and the last of the 28 Qwen3-1.7B-shaped blocks.

For every linear of those blocks the six library calls of the step run through the C ABI
in the step's order: the weight's 128x128 quantisation with its transposed codes, the
activation's dual 1x128 quantisation (row-wise for fprop, along the tokens for wgrad),
fprop, the output gradient's dual quantisation, dgrad and wgrad. Codes and scales are
checked bit for bit on sampled rows, columns and weight blocks that the oracle quantises
from the same BF16 input; the three GEMMs on sampled rows and 128-column blocks against
the oracle's FP64 contraction, within the GEMM tolerance of tests/parity.py. The step's
M = 8192 fprop/dgrad grids and K = 8192 wgrads are the shapes covered here.
"""

import numpy as np
import pytest
import torch

from oracle import quant as oquant
from tests.parity import as_np, bf16_to_f64, check_gemm, host_bits, oracle_gemm_sampled
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOKENS = 8192
STEP_SEED = 4          # the benchmark's seed for rank 0
LAYERS = (0, wl.LAYERS - 1)


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(n, k), replace=False))


def _bits_eq(got, want, what):
    got = as_np(got)
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), np.asarray(want).view(np.uint32)
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{what}: {len(mism)} mismatches, first at {mism[:4].tolist()}"


def _check_dual(out, t, rows, cols, what):
    """(XqT, ST, Xq, S) of a dual quantisation of t [T, C] against the oracle."""
    qt, st, q, s = out
    ci = torch.as_tensor(cols, device=DEV)
    qt_ref, st_ref = oquant.quant_1x128_transposed(host_bits(t[:, ci].contiguous()))
    _bits_eq(qt[ci], qt_ref, f"{what} codes along tokens")
    _bits_eq(st[:, ci], st_ref, f"{what} scales along tokens")
    ri = torch.as_tensor(rows, device=DEV)
    q_ref, s_ref = oquant.quant_1x128(host_bits(t[ri]))
    _bits_eq(q[ri], q_ref, f"{what} row-wise codes")
    _bits_eq(s[:, ri], s_ref, f"{what} row-wise scales")


def _check_gemm_sampled(c_gpu, layout, a, b, rows, nblocks, what):
    c_ref, cols, an, bn = oracle_gemm_sampled(layout, a, b, rows, nblocks)
    got = bf16_to_f64(c_gpu[torch.as_tensor(rows, device=DEV)][:, torch.as_tensor(cols, device=DEV)])
    check_gemm(got, c_ref, an, bn, what)


@pytest.mark.parametrize("layer", LAYERS)
def test_step_layer_at_8192_tokens(pf, layer):
    fwd = wl.layer_forward(STEP_SEED, TOKENS, DEV, layer=layer)
    grads = wl.layer_grads(STEP_SEED, TOKENS, DEV, layer=layer)
    for (name, x, w), (_, dy) in zip(fwd, grads):
        what = f"L{layer}.{name}"
        n_out, k_in = w.shape
        wq, wqt, ws = pf.quantize_128x128(w)
        xqt, xst, xq, xs = pf.quantize_1x128_transposed(x, dual=True)
        y = pf.gemm(xq, xs, wq, ws, "fprop")
        dyqt, dyst, dyq, dys = pf.quantize_1x128_transposed(dy, dual=True)
        dx = pf.gemm(dyq, dys, wqt, ws, "dgrad")
        dw = pf.gemm(dyqt, dyst, xqt, xst, "wgrad")
        torch.cuda.synchronize()
        pf.puro_fp8_sync_status()

        for rb in _sample(-(-n_out // 128), 3, seed=layer + 1):
            q_ref, _, s_ref = oquant.quant_128x128(host_bits(w[rb * 128:(rb + 1) * 128]))
            _bits_eq(wq[rb * 128:(rb + 1) * 128], q_ref, f"{what} Wq block row {rb}")
            _bits_eq(wqt[:, rb * 128:(rb + 1) * 128], q_ref.T, f"{what} WqT block row {rb}")
            _bits_eq(ws[rb], s_ref[0], f"{what} W scales block row {rb}")
        _check_dual((xqt, xst, xq, xs), x, _sample(TOKENS, 48, 2), _sample(k_in, 48, 3), f"{what} X")
        _check_dual((dyqt, dyst, dyq, dys), dy, _sample(TOKENS, 48, 4), _sample(n_out, 48, 5), f"{what} dY")

        rows_t = _sample(TOKENS, 32, seed=6)
        _check_gemm_sampled(y, "fprop", x, w, rows_t, _sample(n_out // 128, 2, 7), f"{what} fprop")
        _check_gemm_sampled(dx, "dgrad", dy, w, rows_t, _sample(k_in // 128, 2, 8), f"{what} dgrad")
        _check_gemm_sampled(dw, "wgrad", dy, x, _sample(n_out, 32, 9), _sample(k_in // 128, 2, 10),
                            f"{what} wgrad")
        del wq, wqt, ws, xqt, xst, xq, xs, y, dyqt, dyst, dyq, dys, dx, dw
