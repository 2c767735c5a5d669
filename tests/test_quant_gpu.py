"""GPU parity of the three quantisers against the oracle: codes and scales bit-exact.

Small cases run the oracle on the whole tensor: hand-built edge blocks (zeros, signed
zeros, BF16 subnormals, a lone outlier, E4M3 ties from the worked example, tiny and
huge magnitudes), ragged row counts, strided rows, several tiles. Full-size workloads
(a Qwen3-1.7B-shaped layer at 4096 tokens, the LM head, the dlogits at 8192 tokens)
are checked on sampled rows, columns and blocks that the oracle quantises from the
same BF16 input.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import quant as oquant
from tests.conftest import GOLDEN
from tests.parity import as_np, host_bits
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _edge_matrix(rows, cols, seed):
    """BF16 [rows, cols] whose 128-blocks cycle through hand-built edge cases."""
    g = torch.Generator().manual_seed(seed)
    x = wl.heavy_tailed((rows, cols), 1.0, g, "cpu")
    with open(os.path.join(GOLDEN, "quant_1x128_worked.json")) as f:
        worked = np.zeros(128, dtype=np.float32)
        for e in json.load(f)["elements"]:
            worked[e["index"]] = e["x"]
    for r in range(rows):
        for j in range(cols // 128):
            kind = (r * 7 + j) % 8
            blk = x[r, j * 128:(j + 1) * 128]
            if kind == 0:
                blk.zero_()
            elif kind == 1:
                blk.zero_()
                blk[::3] = -0.0
            elif kind == 2:
                blk.mul_(2.0 ** -130)  # BF16 subnormals
            elif kind == 3:
                blk.mul_(1e-3)
                blk[17] = -7e4
            elif kind == 4:
                blk.copy_(torch.from_numpy(worked))
            elif kind == 5:
                blk.mul_(3e38 / blk.abs().max())  # near the top of the finite BF16 range
            elif kind == 6:
                blk.fill_(0.3)
    return wl.bf16(x)


def _check_rows(pf, x_dev):
    xq, s = pf.quantize_1x128(x_dev)
    q_ref, s_ref = oquant.quant_1x128(host_bits(x_dev))
    np.testing.assert_array_equal(as_np(xq), q_ref)
    np.testing.assert_array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("rows", [1, 3, 64, 65, 130])
def test_1x128_edge_blocks(pf, rows):
    _check_rows(pf, _edge_matrix(rows, 1024, seed=rows).to(DEV))


def test_1x128_strided_rows_and_codes(pf):
    x = _edge_matrix(70, 512, seed=1).to(DEV)
    wide = torch.zeros((70, 520), dtype=torch.bfloat16, device=DEV)
    wide[:, :512] = x
    view = wide[:, :512]
    xq_wide = torch.full((70, 528), 0xAB, dtype=torch.uint8, device=DEV)
    s = torch.empty((4, 70), dtype=torch.float32, device=DEV)
    pf.puro_fp8_quantize_1x128(view, xq_wide[:, :512], s)
    q_ref, s_ref = oquant.quant_1x128(host_bits(x))
    np.testing.assert_array_equal(as_np(xq_wide[:, :512]), q_ref)
    assert torch.all(xq_wide[:, 512:] == 0xAB), "wrote past the row"
    np.testing.assert_array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))


def test_1x128_small_gemm_operand(pf):
    a, _ = wl.small_gemm(seed=0)
    _check_rows(pf, a.to(DEV))


@pytest.mark.parametrize("T,C,dual", [(128, 8, False), (384, 136, False), (256, 384, True),
                                      (512, 1000, False), (640, 256, True)])
def test_transposed_small(pf, T, C, dual):
    x = _edge_matrix(T, max(C, 128) if C % 128 == 0 else C // 128 * 128 + 128, seed=T + C)[:, :C]
    x = x.contiguous().to(DEV)
    out = pf.quantize_1x128_transposed(x, dual=dual)
    qt_ref, st_ref = oquant.quant_1x128_transposed(host_bits(x))
    np.testing.assert_array_equal(as_np(out[0]), qt_ref)
    np.testing.assert_array_equal(as_np(out[1]).view(np.uint32), st_ref.view(np.uint32))
    if dual:
        q_ref, s_ref = oquant.quant_1x128(host_bits(x))
        np.testing.assert_array_equal(as_np(out[2]), q_ref)
        np.testing.assert_array_equal(as_np(out[3]).view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("R,C,transposed", [(1, 128, False), (300, 256, False), (304, 384, True),
                                            (128, 128, True), (1040, 512, True)])
def test_128x128_small(pf, R, C, transposed):
    w = (_edge_matrix(R, C, seed=R) * 0.02).to(torch.bfloat16).to(DEV)
    wq, wqt, s = pf.quantize_128x128(w, transposed=transposed)
    q_ref, qt_ref, s_ref = oquant.quant_128x128(host_bits(w))
    np.testing.assert_array_equal(as_np(wq), q_ref)
    np.testing.assert_array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))
    if transposed:
        np.testing.assert_array_equal(as_np(wqt), qt_ref)


def _slow_and_zero_groups():
    """BF16 [256, 512]: heavy-tailed, with groups that leave the kernels' fast path (tiny
    maxima: scales below 2^-90, and below 2^-100 where the scale itself needs IEEE
    division) or take it with r = 0 (all-zero groups), placed so that a warp or a tile
    mixes them with ordinary groups.

    Tile (0, 0): column 5 holds BF16 subnormals only, column 6 signed zeros, column 7
    values scaled by 2^-95; the other columns are ordinary. Tile (0, 1) is all zero, with
    signed zeros. Tile (1, 2) holds subnormals only. In tile (1, 3), row 140 is scaled by
    2^-110 while the other rows stay ordinary."""
    g = torch.Generator().manual_seed(77)
    x = wl.heavy_tailed((256, 512), 1.0, g, "cpu")
    x[:128, 5] *= 2.0 ** -130
    x[:128, 6] = 0.0
    x[1:128:3, 6] = -0.0
    x[:128, 7] *= 2.0 ** -95
    x[:128, 128:256] = 0.0
    x[:128:5, 128:256] = -0.0
    x[128:256, 256:384] *= 2.0 ** -130
    x[140, 384:512] *= 2.0 ** -110
    return wl.bf16(x)


def test_slow_and_zero_groups_in_every_mode(pf):
    x = _slow_and_zero_groups().to(DEV)
    bits = host_bits(x)
    _check_rows(pf, x)
    qt, st, q, s = pf.quantize_1x128_transposed(x, dual=True)
    qt_ref, st_ref = oquant.quant_1x128_transposed(bits)
    q_ref, s_ref = oquant.quant_1x128(bits)
    np.testing.assert_array_equal(as_np(qt), qt_ref)
    np.testing.assert_array_equal(as_np(st).view(np.uint32), st_ref.view(np.uint32))
    np.testing.assert_array_equal(as_np(q), q_ref)
    np.testing.assert_array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))
    qt2, st2 = pf.quantize_1x128_transposed(x, dual=False)
    np.testing.assert_array_equal(as_np(qt2), qt_ref)
    np.testing.assert_array_equal(as_np(st2).view(np.uint32), st_ref.view(np.uint32))
    wq, wqt, ws = pf.quantize_128x128(x, transposed=True)
    wq_ref, wqt_ref, ws_ref = oquant.quant_128x128(bits)
    np.testing.assert_array_equal(as_np(wq), wq_ref)
    np.testing.assert_array_equal(as_np(wqt), wqt_ref)
    np.testing.assert_array_equal(as_np(ws).view(np.uint32), ws_ref.view(np.uint32))
    # the constructed groups are what the docstring says
    st_np = st_ref.view(np.float32)
    assert st_np[0, 6] == 0.0 and 0.0 < st_np[0, 5] < 2.0 ** -90 and 0.0 < st_np[0, 7] < 2.0 ** -90
    assert ws_ref[0, 1] == 0.0 and 0.0 < ws_ref[1, 2] < 2.0 ** -90
    s_np = s_ref.view(np.float32)
    assert 0.0 < s_np[3, 140] < 2.0 ** -100 / 448 * 2 and s_np[3, 141] > 2.0 ** -90


# ------------------------------------------------------------------ full-size workloads

def _sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(n, k), replace=False))


def test_layer_operands_full_size(pf):
    """Every quantiser call of one block's forward and backward at 4096 tokens."""
    T = 4096
    fwd = wl.layer_forward(1, T, DEV)
    grads = wl.layer_grads(2, T, DEV)
    for (name, x, w), (_, dy) in zip(fwd, grads):
        # activations, row-wise: full comparison
        _check_rows(pf, x)
        # weights: every block, both code layouts
        wq, wqt, s = pf.quantize_128x128(w)
        q_ref, _, s_ref = oquant.quant_128x128(host_bits(w))
        np.testing.assert_array_equal(as_np(wq), q_ref, err_msg=name)
        np.testing.assert_array_equal(as_np(wqt), q_ref.T, err_msg=name)
        np.testing.assert_array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))
        # activations along tokens (wgrad B) and dY dual (dgrad A + wgrad A): sampled columns
        for t, dual in ((x, False), (dy, True)):
            out = pf.quantize_1x128_transposed(t, dual=dual)
            cols = _sample(t.shape[1], 96, seed=3)
            sub = host_bits(t[:, torch.as_tensor(cols, device=DEV)].contiguous())
            qt_ref, st_ref = oquant.quant_1x128_transposed(sub)
            np.testing.assert_array_equal(as_np(out[0])[cols], qt_ref, err_msg=name)
            np.testing.assert_array_equal(as_np(out[1])[:, cols].view(np.uint32), st_ref.view(np.uint32))
            if dual:
                rows = _sample(T, 64, seed=4)
                q_ref, s_ref = oquant.quant_1x128(host_bits(t[torch.as_tensor(rows, device=DEV)]))
                np.testing.assert_array_equal(as_np(out[2])[rows], q_ref)
                np.testing.assert_array_equal(as_np(out[3])[:, rows].view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("tokens", [4096, 8192])
def test_lm_head_operands_full_size(pf, tokens):
    h, w, dl = wl.lm_head(3, tokens, DEV)
    # weight: sampled row blocks, both layouts
    wq, wqt, s = pf.quantize_128x128(w)
    for rb in _sample(w.shape[0] // 128, 6, seed=5):
        q_ref, _, s_ref = oquant.quant_128x128(host_bits(w[rb * 128:(rb + 1) * 128]))
        np.testing.assert_array_equal(as_np(wq[rb * 128:(rb + 1) * 128]), q_ref)
        np.testing.assert_array_equal(as_np(wqt[:, rb * 128:(rb + 1) * 128]), q_ref.T)
        np.testing.assert_array_equal(as_np(s[rb]).view(np.uint32), s_ref[0].view(np.uint32))
    del wq, wqt
    # dlogits: dual transposed quantisation, sampled rows and columns
    qt, st, q, sr = pf.quantize_1x128_transposed(dl, dual=True)
    rows = _sample(tokens, 24, seed=6)
    q_ref, s_ref = oquant.quant_1x128(host_bits(dl[torch.as_tensor(rows, device=DEV)]))
    np.testing.assert_array_equal(as_np(q[torch.as_tensor(rows, device=DEV)]), q_ref)
    np.testing.assert_array_equal(as_np(sr[:, torch.as_tensor(rows, device=DEV)]).view(np.uint32),
                                  s_ref.view(np.uint32))
    cols = _sample(dl.shape[1], 64, seed=7)
    cols_t = torch.as_tensor(cols, device=DEV)
    qt_ref, st_ref = oquant.quant_1x128_transposed(host_bits(dl[:, cols_t].contiguous()))
    np.testing.assert_array_equal(as_np(qt[cols_t]), qt_ref)
    np.testing.assert_array_equal(as_np(st[:, cols_t]).view(np.uint32), st_ref.view(np.uint32))
    # hidden states, row-wise and along tokens
    _check_rows(pf, h)
    ht, hst = pf.quantize_1x128_transposed(h)
    qt_ref, st_ref = oquant.quant_1x128_transposed(host_bits(h))
    np.testing.assert_array_equal(as_np(ht), qt_ref)
    np.testing.assert_array_equal(as_np(hst).view(np.uint32), st_ref.view(np.uint32))
