"""GPU parity of the grouped weight quantiser (puro_fp8_quantize_128x128_grouped).

* Every weight of a group gets bit for bit the codes, transposed codes and scales that
  puro_fp8_quantize_128x128 gives it alone, and those match the oracle: weights of
  different shapes in one launch (partial last row blocks, strided rows, with and without
  the transposed codes, all-zero and tiny-scale blocks);
* more weights than one launch takes (two launches), each weight still exact;
* full size: the 113 weights of the benchmarked step (28 Qwen3-1.7B-shaped blocks and the
  LM head) in one call, identical to 113 single calls.
"""

import numpy as np
import pytest
import torch

from oracle import quant as oquant
from tests.parity import as_np, host_bits
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def _weight(r, c, ld, seed):
    g = torch.Generator().manual_seed(seed)
    w = wl.heavy_tailed((r, ld), 0.02, g, "cpu")
    if r > 128 and c >= 256:
        w[:128, 128:256] = 0.0                 # an all-zero block
        w[128:, :128] *= 2.0 ** -120           # tiny scales (off the fast division path)
    return wl.bf16(w).to(DEV)[:, :c]


def _outputs(r, c, with_t, fill):
    wq = torch.full((r, c), fill, dtype=torch.uint8, device=DEV)
    wqt = torch.full((c, r), fill, dtype=torch.uint8, device=DEV) if with_t else None
    s = torch.full(((r + 127) // 128, c // 128), -1.0, dtype=torch.float32, device=DEV)
    return wq, wqt, s


def _check_group(pf, shapes, seed):
    ws = [_weight(r, c, ld, seed + i) for i, (r, c, ld, _) in enumerate(shapes)]
    grouped = [_outputs(r, c, t, 0xAB) for (r, c, _, t) in shapes]
    single = [_outputs(r, c, t, 0xCD) for (r, c, _, t) in shapes]
    pf.puro_fp8_quantize_128x128_grouped([(w, *o) for w, o in zip(ws, grouped)])
    for w, (wq, wqt, s) in zip(ws, single):
        pf.puro_fp8_quantize_128x128(w, wq, wqt, s)
    pf.puro_fp8_sync_status()
    for i, (g, o) in enumerate(zip(grouped, single)):
        for a, b, name in zip(g, o, ("Wq", "WqT", "S")):
            if a is not None:
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"weight {i}: {name} differs"
    return ws, grouped


def test_mixed_shapes_match_single_calls_and_oracle(pf):
    shapes = [(256, 256, 256, True), (130, 384, 512, False), (304, 128, 128, True), (16, 256, 256, True),
              (1, 128, 128, False), (1008, 640, 648, True), (384, 1024, 1024, True)]
    ws, outs = _check_group(pf, shapes, seed=11)
    for w, (wq, wqt, s) in zip(ws, outs):
        q_ref, qt_ref, s_ref = oquant.quant_128x128(host_bits(w.contiguous()))
        assert np.array_equal(as_np(wq), q_ref)
        if wqt is not None:
            assert np.array_equal(as_np(wqt), qt_ref)
        assert np.array_equal(as_np(s).view(np.uint32), s_ref.view(np.uint32))


def test_more_weights_than_one_launch(pf):
    rng = np.random.default_rng(3)
    shapes = [(int(16 * rng.integers(1, 25)), int(128 * rng.integers(1, 3)), 0, bool(rng.integers(0, 2)))
              for _ in range(70)]
    shapes = [(r, c, c, t) for r, c, _, t in shapes]
    _check_group(pf, shapes, seed=100)


def test_step_weights_full_size(pf):
    """The weights the benchmarked step quantises, one grouped call against single calls."""
    ws = []
    for layer in range(28):
        ws += [w for (_, _, w) in wl.layer_forward(4, 128, DEV, layer=layer)]
    ws.append(wl.lm_head(4, 128, DEV)[1])
    grouped, single = [], []
    for w in ws:
        r, c = w.shape
        grouped.append(_outputs(r, c, True, 0))
        single.append(_outputs(r, c, True, 0))
    pf.puro_fp8_quantize_128x128_grouped([(w, *o) for w, o in zip(ws, grouped)])
    for w, (wq, wqt, s) in zip(ws, single):
        pf.puro_fp8_quantize_128x128(w, wq, wqt, s)
    pf.puro_fp8_sync_status()
    for i, (g, o) in enumerate(zip(grouped, single)):
        for a, b, name in zip(g, o, ("Wq", "WqT", "S")):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"weight {i}: {name} differs"
    # and one block of each of a few weights against the oracle
    for i in (0, 57, 112):
        w = ws[i]
        q_ref, _, s_ref = oquant.quant_128x128(host_bits(w[:128]))
        assert np.array_equal(as_np(grouped[i][0][:128]), q_ref)
        assert np.array_equal(as_np(grouped[i][2][:1]).view(np.uint32), s_ref.view(np.uint32))
