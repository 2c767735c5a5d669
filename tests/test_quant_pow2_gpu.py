"""GPU parity of the power-of-two (UE8M0) scale quantisers against oracle.mx: codes and
scale bytes bit-exact.

Edge groups (zeros, signed zeros, BF16 subnormals, groups below the clamp, lone outliers,
values exactly at 448 * 2^e and just above it, near the top of the BF16 range), ragged row
counts and strided rows, all three geometries (rows, along tokens with the dual output,
128x128 weights with the transposed codes), and a full-size Qwen3-1.7B-shaped layer's
operands at 8192 tokens on sampled rows, columns and blocks.
"""

import numpy as np
import pytest
import torch

from oracle import mx
from tests.parity import as_np, host_bits
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _edge_matrix(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = wl.heavy_tailed((rows, cols), 1.0, g, "cpu")
    for r in range(rows):
        for j in range(cols // 128):
            kind = (3 * r + j) % 9
            blk = x[r, j * 128:(j + 1) * 128]
            if kind == 0:
                blk.zero_()
            elif kind == 1:
                blk.zero_()
                blk[1::4] = -0.0
            elif kind == 2:
                blk.mul_(2.0 ** -130)          # BF16 subnormals: below the exponent clamp
            elif kind == 3:
                blk.mul_(2.0 ** -125)          # near the clamp
            elif kind == 4:
                blk.mul_(1e-3)
                blk[5] = -448.0 * 2.0 ** -3    # amax exactly 448 * 2^e
            elif kind == 5:
                blk.mul_(1e-3)
                blk[9] = 449.0 * 2.0 ** -3     # just above it
            elif kind == 6:
                blk.mul_(3e38 / blk.abs().max())
            elif kind == 7:
                blk.fill_(-0.75)
    return wl.bf16(x)


def _eq(got, want, what):
    got = as_np(got)
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{what}: {len(mism)} mismatches, first at {mism[:4].tolist()}"


@pytest.mark.parametrize("rows", [1, 3, 65, 130, 256])
def test_rows_edge_groups(pf, rows):
    x = _edge_matrix(rows, 512, rows)
    xd = x.to(DEV)
    xq = torch.empty((rows, 512), dtype=torch.uint8, device=DEV)
    s = torch.empty((4, rows), dtype=torch.uint8, device=DEV)
    pf.puro_fp8_quantize_1x128_pow2(xd, xq, s)
    q_ref, s_ref = mx.quant_1x128_pow2(host_bits(x))
    _eq(xq, q_ref, "codes")
    _eq(s, s_ref, "scale bytes")


def test_rows_strided(pf):
    x = _edge_matrix(70, 640, 5)
    big = torch.zeros((70, 768), dtype=torch.bfloat16)
    big[:, :640] = x
    xd = big.to(DEV)[:, :640]
    xq_big = torch.full((70, 784), 0xAB, dtype=torch.uint8, device=DEV)
    s = torch.empty((5, 70), dtype=torch.uint8, device=DEV)
    pf.puro_fp8_quantize_1x128_pow2(xd, xq_big[:, :640], s)
    q_ref, s_ref = mx.quant_1x128_pow2(host_bits(x))
    _eq(xq_big[:, :640], q_ref, "codes")
    assert torch.all(xq_big[:, 640:] == 0xAB), "wrote past the row"
    _eq(s, s_ref, "scale bytes")


@pytest.mark.parametrize("t,c", [(256, 384), (384, 136), (128, 8)])
def test_along_tokens_and_dual(pf, t, c):
    x = _edge_matrix(t, 384 if c % 128 else c, t + c)[:, :c].contiguous()
    xd = x.to(DEV)
    qt = torch.empty((c, t), dtype=torch.uint8, device=DEV)
    st = torch.empty((t // 128, c), dtype=torch.uint8, device=DEV)
    dual = c % 128 == 0
    q = torch.empty((t, c), dtype=torch.uint8, device=DEV) if dual else None
    s = torch.empty((c // 128, t), dtype=torch.uint8, device=DEV) if dual else None
    pf.puro_fp8_quantize_1x128_transposed_pow2(xd, qt, st, q, s)
    qt_ref, st_ref = mx.quant_1x128_transposed_pow2(host_bits(x))
    _eq(qt, qt_ref, "codes along tokens")
    _eq(st, st_ref, "scale bytes along tokens")
    if dual:
        q_ref, s_ref = mx.quant_1x128_pow2(host_bits(x))
        _eq(q, q_ref, "row-wise codes")
        _eq(s, s_ref, "row-wise scale bytes")


@pytest.mark.parametrize("r,c", [(256, 256), (304, 384), (16, 128)])
def test_weight_blocks(pf, r, c):
    w = _edge_matrix(r, c, 3 * r + c)
    wd = w.to(DEV)
    wq = torch.empty((r, c), dtype=torch.uint8, device=DEV)
    wqt = torch.empty((c, r), dtype=torch.uint8, device=DEV)
    s = torch.empty(((r + 127) // 128, c // 128), dtype=torch.uint8, device=DEV)
    pf.puro_fp8_quantize_128x128_pow2(wd, wq, wqt, s)
    q_ref, qt_ref, s_ref = mx.quant_128x128_pow2(host_bits(w))
    _eq(wq, q_ref, "codes")
    _eq(wqt, qt_ref, "transposed codes")
    _eq(s, s_ref, "scale bytes")


def test_layer_operands_full_size(pf):
    T = 8192
    (name, x, w) = wl.layer_forward(4, T, DEV, layer=0)[2]   # gate/up: X [8192, 2048], W [12288, 2048]
    (_, dy) = wl.layer_grads(4, T, DEV, layer=0)[2]           # dY [8192, 12288]
    rng = np.random.default_rng(3)
    wq = torch.empty(w.shape, dtype=torch.uint8, device=DEV)
    wqt = torch.empty((w.shape[1], w.shape[0]), dtype=torch.uint8, device=DEV)
    ws = torch.empty((w.shape[0] // 128, w.shape[1] // 128), dtype=torch.uint8, device=DEV)
    pf.puro_fp8_quantize_128x128_pow2(w, wq, wqt, ws)
    for rb in rng.choice(w.shape[0] // 128, 3, replace=False):
        q_ref, qt_ref, s_ref = mx.quant_128x128_pow2(host_bits(w[rb * 128:(rb + 1) * 128]))
        _eq(wq[rb * 128:(rb + 1) * 128], q_ref, "weight codes")
        _eq(ws[rb], s_ref[0], "weight scale bytes")
    for t in (x, dy):
        c = t.shape[1]
        qt = torch.empty((c, T), dtype=torch.uint8, device=DEV)
        st = torch.empty((T // 128, c), dtype=torch.uint8, device=DEV)
        q = torch.empty((T, c), dtype=torch.uint8, device=DEV)
        s = torch.empty((c // 128, T), dtype=torch.uint8, device=DEV)
        pf.puro_fp8_quantize_1x128_transposed_pow2(t, qt, st, q, s)
        rows = np.sort(rng.choice(T, 40, replace=False))
        q_ref, s_ref = mx.quant_1x128_pow2(host_bits(t[torch.as_tensor(rows, device=DEV)]))
        _eq(q[torch.as_tensor(rows, device=DEV)], q_ref, "row-wise codes")
        _eq(s[:, torch.as_tensor(rows, device=DEV)], s_ref, "row-wise bytes")
        cols = np.sort(rng.choice(c, 40, replace=False))
        ci = torch.as_tensor(cols, device=DEV)
        qt_ref, st_ref = mx.quant_1x128_transposed_pow2(host_bits(t[:, ci].contiguous()))
        _eq(qt[ci], qt_ref, "codes along tokens")
        _eq(st[:, ci], st_ref, "bytes along tokens")
    pf.puro_fp8_sync_status()
