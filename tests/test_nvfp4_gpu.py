"""NVFP4 mode on the GPU against the oracle (oracle/nvfp4.py), through the C ABI.

- quantisers: packed codes, UE4M3 factors and the tensor amax bit-exact, row-wise,
  transposed and both from one call (dual), on ragged and strided shapes, all-zero groups, negative zeros, a tiny tensor
  (subnormal factors) and the hand-worked row of tests/golden/nvfp4_blocks_worked.json;
- GEMM: the benchmark spec's tolerance (relative Frobenius <= 2e-3, elementwise <= 1e-2 ||a_m|| ||b_n||)
  against the FP64 oracle, including a half K block (K % 256 == 128), single CTAs and CTA
  pairs, M / N tails; an exact-integer case compared bit for bit; the step's full sizes on
  sampled rows.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4 as onv
from oracle.quant import bf16_bits_to_f32

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def pf():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8


def bits_of(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, seed, scale=1.0, tails=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * scale
    if tails:
        t = torch.distributions.StudentT(3.0).sample(shape) * scale
        m = torch.rand(shape, generator=g) < 0.01
        x = torch.where(m, t * 10, x)
    return x.to(torch.bfloat16)


def unblocked(f_blocked, groups):
    """[ceil(K/256), R, 16] -> [R, K/16] (the defined bytes)."""
    nb, r, _ = f_blocked.shape
    return f_blocked.transpose(1, 0, 2).reshape(r, nb * 16)[:, :groups]


def check_rows(pf, x, ldq_pad=0, ldx_pad=0):
    R, C = x.shape
    xs = torch.zeros((R, C + ldx_pad), dtype=torch.bfloat16, device="cuda")
    xs[:, :C] = x.cuda()
    X = xs[:, :C]
    q_full = torch.zeros((R, C // 2 + ldq_pad), dtype=torch.uint8, device="cuda")
    f = torch.zeros(((C + 255) // 256, R, 16), dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), -1.0, device="cuda")
    pf.puro_nvfp4_quantize_1x16(X, q_full[:, :C // 2], f, amax)
    sync(pf)
    wq, wf, wa = onv.quant_1x16(bits_of(x))
    assert amax.item() == float(wa) or (amax.item() == 0 and wa == 0)
    assert np.array_equal(unblocked(f.cpu().numpy(), C // 16), wf)
    assert np.array_equal(q_full[:, :C // 2].cpu().numpy(), wq)
    if ldq_pad:
        assert not q_full[:, C // 2:].any(), "nothing written past a row's codes"


def check_cols(pf, x):
    R, C = x.shape
    X = x.cuda()
    q = torch.zeros((C, R // 2), dtype=torch.uint8, device="cuda")
    f = torch.zeros(((R + 255) // 256, C, 16), dtype=torch.uint8, device="cuda")
    amax = torch.zeros(1, device="cuda")
    pf.puro_nvfp4_quantize_1x16_transposed(X, q, f, amax)
    wq, wf, wa = onv.quant_1x16_transposed(bits_of(x))
    assert amax.item() == float(wa)
    assert np.array_equal(unblocked(f.cpu().numpy(), R // 16), wf)
    assert np.array_equal(q.cpu().numpy(), wq)


def sync(pf):
    st = pf._lib.puro_fp8_sync_status(pf._stream(None))
    assert st == 0, st


@pytest.mark.parametrize("shape,seed,pads", [((1, 16), 0, (0, 0)), ((3, 48), 1, (16, 8)), ((100, 2048), 2, (0, 0)),
                                             ((257, 384), 3, (32, 24)), ((64, 4096), 4, (0, 0))])
def test_quant_rows_bit_exact(pf, shape, seed, pads):
    check_rows(pf, rand_bf16(shape, seed), ldq_pad=pads[0], ldx_pad=pads[1])
    sync(pf)


def test_quant_rows_special_groups(pf):
    x = rand_bf16((8, 256), 5)
    x[1, :16] = 0.0
    x[2, 16:32] = -0.0
    x[3, 32:48] = 1e-30  # tiny against the tensor amax: factor rounds to zero or a subnormal
    x[4, :] = x[4, :] * 1e-3
    x[5, 7] = 3000.0  # the tensor amax
    check_rows(pf, x)
    tiny = (torch.randn((4, 64)) * 1e-38).to(torch.bfloat16)  # s_t underflows
    check_rows(pf, tiny)
    check_rows(pf, torch.zeros((2, 32), dtype=torch.bfloat16))
    sync(pf)


def test_quant_rows_worked_row(pf):
    g = json.load(open(os.path.join(HERE, "golden", "nvfp4_blocks_worked.json")))
    x = torch.tensor(g["x"], dtype=torch.float32).reshape(1, 64).to(torch.bfloat16)
    q, f, a = pf.nvfp4_quantize(x.cuda())
    sync(pf)
    assert a.item() == g["tensor_amax"]
    assert unblocked(f.cpu().numpy(), 4).reshape(-1).tolist() == g["factors"]
    assert onv.unpack(q.cpu().numpy()).reshape(4, 16).tolist() == g["codes"]


@pytest.mark.parametrize("shape,seed", [((64, 8), 10), ((128, 48), 11), ((256, 264), 12), ((4096, 512), 13)])
def test_quant_cols_bit_exact(pf, shape, seed):
    check_cols(pf, rand_bf16(shape, seed))
    sync(pf)


def _operands(pf, m, n, k, seed, b_scale=0.02):
    a = rand_bf16((m, k), seed)
    b = rand_bf16((n, k), seed + 1, scale=b_scale, tails=False)
    aq, af, aa = pf.nvfp4_quantize(a.cuda())
    bq, bf, ba = pf.nvfp4_quantize(b.cuda())
    return (aq, af, aa, bq, bf, ba)


def _tolerance_check(got, want, na, nb):
    err = got - want
    rel = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-300)
    assert rel <= 2e-3, rel
    bound = 1e-2 * np.outer(na, nb)
    assert np.all(np.abs(err) <= bound + 1e-30), float(np.max(np.abs(err) - bound))


@pytest.mark.parametrize("m,n,k,seed", [(128, 256, 256, 20), (300, 520, 384, 21), (512, 1024, 2048, 22),
                                        (128, 8, 128, 23), (96, 264, 640, 24), (640, 256, 1152, 25)])
def test_gemm_within_tolerance(pf, m, n, k, seed):
    ops = _operands(pf, m, n, k, seed)
    c = pf.nvfp4_gemm(*ops)
    sync(pf)
    host = [t.cpu().numpy() for t in ops]
    aq, af, aa, bq, bf, ba = host
    af, bf = unblocked(af, k // 16), unblocked(bf, k // 16)
    want = onv.gemm_ref(aq, af, aa[0], bq, bf, ba[0])
    na, nb = onv.row_col_norms(aq, af, aa[0], bq, bf, ba[0])
    _tolerance_check(c.float().cpu().numpy().astype(np.float64), want, na, nb)


def test_gemm_exact_integers(pf):
    """Values 0, +-1, +-2 with a 6 in every group (factor E4M3(1) = 1, S = 1) and one planted
    2688 per operand (tensor amax 2688, so s_t = 1 exactly): every dequantised value is an
    integer, every partial sum is an integer well inside FP32, so the GEMM is exact and its
    BF16 rounding is compared bit for bit with the oracle's."""
    m, n, k = 256, 512, 640
    g = torch.Generator().manual_seed(30)
    vals = torch.tensor([0.0, 1.0, -1.0, 2.0, -2.0])
    a = vals[torch.randint(0, 5, (m, k), generator=g)]
    b = vals[torch.randint(0, 5, (n, k), generator=g)]
    a[:, ::16] = 6.0
    b[:, 1::16] = -6.0
    a[0, 5] = 2688.0
    b[3, 100] = -2688.0
    A, B = a.to(torch.bfloat16).cuda(), b.to(torch.bfloat16).cuda()
    aq, af, aa = pf.nvfp4_quantize(A)
    bq, bf, ba = pf.nvfp4_quantize(B)
    c = pf.nvfp4_gemm(aq, af, aa, bq, bf, ba)
    sync(pf)
    assert aa.item() == 2688.0 and ba.item() == 2688.0
    fa, fb = unblocked(af.cpu().numpy(), k // 16), unblocked(bf.cpu().numpy(), k // 16)
    want = onv.gemm_ref(aq.cpu().numpy(), fa, 2688.0, bq.cpu().numpy(), fb, 2688.0)
    assert fa[0, 0] == 0x7E and fb[3, 6] == 0x7E
    fa, fb = fa.copy(), fb.copy()
    fa[0, 0] = fb[3, 6] = 0x38
    assert (fa == 0x38).all() and (fb == 0x38).all()
    assert np.array_equal(want, np.round(want)), "the oracle's result is integral"
    want_bf16 = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(c.cpu(), want_bf16)


@pytest.mark.parametrize("m,n,k", [(8192, 4096, 2048), (8192, 2048, 6144)])
def test_full_size_quantiser_and_sampled_gemm_rows(pf, m, n, k):
    a = rand_bf16((m, k), 40)
    b = rand_bf16((n, k), 41, scale=0.02, tails=False)
    aq, af, aa = pf.nvfp4_quantize(a.cuda())
    bq, bf, ba = pf.nvfp4_quantize(b.cuda())
    c = pf.nvfp4_gemm(aq, af, aa, bq, bf, ba)
    sync(pf)
    wq, wf, wa = onv.quant_1x16(bits_of(a))
    assert aa.item() == float(wa)
    assert np.array_equal(unblocked(af.cpu().numpy(), k // 16), wf) and np.array_equal(aq.cpu().numpy(), wq)
    rows = np.sort(np.random.default_rng(42).choice(m, size=48, replace=False))
    aqh, afh = wq[rows], wf[rows]
    bqh, bfh = bq.cpu().numpy(), unblocked(bf.cpu().numpy(), k // 16)
    want = onv.gemm_ref(aqh, afh, wa, bqh, bfh, ba.item())
    na, nb = onv.row_col_norms(aqh, afh, wa, bqh, bfh, ba.item())
    _tolerance_check(c.float().cpu().numpy()[rows].astype(np.float64), want, na, nb)


def run_dual(pf, X, pads=(0, 0)):
    R, C = X.shape
    q = torch.zeros((R, C // 2 + pads[0]), dtype=torch.uint8, device="cuda")
    qt = torch.zeros((C, R // 2 + pads[1]), dtype=torch.uint8, device="cuda")
    f = torch.zeros(((C + 255) // 256, R, 16), dtype=torch.uint8, device="cuda")
    ft = torch.zeros(((R + 255) // 256, C, 16), dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), -1.0, device="cuda")
    pf.puro_nvfp4_quantize_1x16_dual(X, q[:, :C // 2], f, qt[:, :R // 2], ft, amax)
    sync(pf)
    if pads[0]:
        assert not q[:, C // 2:].any()
    if pads[1]:
        assert not qt[:, R // 2:].any()
    return q[:, :C // 2], f, qt[:, :R // 2], ft, amax


@pytest.mark.parametrize("shape,seed,pads", [((64, 16), 20, (0, 0)), ((128, 272), 21, (8, 16)),
                                             ((192, 512), 22, (0, 0)), ((256, 2064), 23, (24, 32)),
                                             ((640, 768), 24, (0, 0)), ((128, 80), 28, (0, 0))])
def test_quant_dual_bit_exact(pf, shape, seed, pads):
    """One call, both layouts: each equal to its oracle routine byte for byte, with tiles that end
    inside a 256-column block (272, 2064, 80), padded output rows, and code rows that are only
    8-byte aligned (C = 80: a row stride of 40 bytes)."""
    R, C = shape
    x = rand_bf16(shape, seed)
    xs = torch.zeros((R, C + 8), dtype=torch.bfloat16, device="cuda")
    xs[:, :C] = x.cuda()
    q, f, qt, ft, amax = run_dual(pf, xs[:, :C], pads)
    wq, wf, wa = onv.quant_1x16(bits_of(x))
    tq, tf, ta = onv.quant_1x16_transposed(bits_of(x))
    assert amax.item() == float(wa) == float(ta)
    assert np.array_equal(q.cpu().numpy(), wq) and np.array_equal(unblocked(f.cpu().numpy(), C // 16), wf)
    assert np.array_equal(qt.cpu().numpy(), tq) and np.array_equal(unblocked(ft.cpu().numpy(), R // 16), tf)


def test_quant_dual_special_groups(pf):
    x = rand_bf16((64, 256), 25)
    x[1, :16] = 0.0
    x[:16, 3] = -0.0
    x[2, 32:48] = 1e-30
    x[16:32, 40] = 1e-30
    x[5, 7] = -3000.0  # the tensor amax
    # s_t >= 2^-81 with groups below 2^-100 (the all-fast path); s_t between 2^-90 and 2^-81 (the
    # per-group path); s_t below 2^-90 (IEEE division)
    small = (torch.randn((64, 64)) * 1e-20).to(torch.bfloat16)
    small[3, :16] = 1e-32
    small[:16, 40] = -1e-33
    mid = (torch.randn((64, 32)) * 1e-24).to(torch.bfloat16)
    for t in (x, torch.zeros((64, 32), dtype=torch.bfloat16), (torch.randn((64, 48)) * 1e-38).to(torch.bfloat16),
              small, mid):
        q, f, qt, ft, amax = run_dual(pf, t.cuda())
        wq, wf, wa = onv.quant_1x16(bits_of(t))
        tq, tf, _ = onv.quant_1x16_transposed(bits_of(t))
        assert amax.item() == float(wa)
        assert np.array_equal(q.cpu().numpy(), wq) and np.array_equal(unblocked(f.cpu().numpy(), t.shape[1] // 16), wf)
        assert np.array_equal(qt.cpu().numpy(), tq) and np.array_equal(unblocked(ft.cpu().numpy(), t.shape[0] // 16), tf)


@pytest.mark.parametrize("R,C", [(8192, 2048), (8192, 151936)])
def test_quant_dual_full_size(pf, R, C):
    """The step's activation (8192 x 2048) and LM-head dlogits (8192 x 151936) shapes: the dual
    call equals the two single calls byte for byte; sampled rows and columns equal the oracle's
    groups under the tensor's exact amax."""
    x = rand_bf16((R, C), 26, tails=C < 100000).cuda()
    q, f, qt, ft, amax = run_dual(pf, x)
    q1, f1, a1 = pf.nvfp4_quantize(x)
    q2, f2, a2 = pf.nvfp4_quantize(x, transposed=True)
    sync(pf)
    assert amax.item() == a1.item() == a2.item()
    assert torch.equal(q, q1) and torch.equal(f, f1) and torch.equal(qt, q2) and torch.equal(ft, f2)
    xb = bits_of(x)
    wa = onv.tensor_amax(xb)
    assert amax.item() == float(wa)
    rng = np.random.default_rng(27)
    rows = np.sort(rng.choice(R, size=16, replace=False))
    codes, fac = onv.quantize_groups(bf16_bits_to_f32(xb[rows]).reshape(16, C // 16, 16), wa)
    assert np.array_equal(q[rows].cpu().numpy(), onv.pack(codes.reshape(16, C)))
    assert np.array_equal(unblocked(f.cpu().numpy(), C // 16)[rows], fac)
    cols = np.sort(rng.choice(C, size=16, replace=False))
    codes, fac = onv.quantize_groups(bf16_bits_to_f32(np.ascontiguousarray(xb[:, cols].T)).reshape(16, R // 16, 16), wa)
    assert np.array_equal(qt[cols].cpu().numpy(), onv.pack(codes.reshape(16, R)))
    assert np.array_equal(unblocked(ft.cpu().numpy(), R // 16)[cols], fac)


def test_linear_pass_on_dual_operands(pf):
    """One linear's three GEMMs as the NVFP4 step runs them, every operand from the dual
    quantiser: fprop X . W^T, dgrad dY . W (W quantised along N_out), wgrad dY^T . X (both along
    the tokens), each within the tolerance of the oracle's contraction of the oracle's own
    quantisation of the same BF16 tensors."""
    T, K, N = 256, 512, 384
    x = rand_bf16((T, K), 50)
    w = rand_bf16((N, K), 51, scale=0.02, tails=False)
    dy = rand_bf16((T, N), 52, scale=1e-3)
    (xq, xf), (xqt, xft), xa = pf.nvfp4_quantize_dual(x.cuda())
    (wq, wf), (wqt, wft), wa = pf.nvfp4_quantize_dual(w.cuda())
    (dq, df), (dqt, dft), da = pf.nvfp4_quantize_dual(dy.cuda())
    got = {"fprop": pf.nvfp4_gemm(xq, xf, xa, wq, wf, wa),
           "dgrad": pf.nvfp4_gemm(dq, df, da, wqt, wft, wa),
           "wgrad": pf.nvfp4_gemm(dqt, dft, da, xqt, xft, xa)}
    sync(pf)
    rows, cols = onv.quant_1x16, onv.quant_1x16_transposed
    ops = {"fprop": (rows(bits_of(x)), rows(bits_of(w))),
           "dgrad": (rows(bits_of(dy)), cols(bits_of(w))),
           "wgrad": (cols(bits_of(dy)), cols(bits_of(x)))}
    for name, ((aq, af, aa), (bq, bf, ba)) in ops.items():
        want = onv.gemm_ref(aq, af, aa, bq, bf, ba)
        na, nb = onv.row_col_norms(aq, af, aa, bq, bf, ba)
        c = got[name].float().cpu().numpy().astype(np.float64)
        assert c.shape == want.shape, name
        _tolerance_check(c, want, na, nb)


def test_argument_errors(pf):
    lib = pf.library()
    st = pf._stream(None)
    x = torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((4, 16), dtype=torch.uint8, device="cuda")
    f = torch.zeros((4, 2), dtype=torch.uint8, device="cuda")
    a = torch.zeros(1, device="cuda")
    p = lambda t: t.data_ptr()
    assert lib.puro_nvfp4_quantize_1x16(None, 4, 32, 32, p(q), 16, p(f), p(a), st) == -1   # NULL
    assert lib.puro_nvfp4_quantize_1x16(p(x), 4, 24, 32, p(q), 16, p(f), p(a), st) == -2   # C % 16
    assert lib.puro_nvfp4_quantize_1x16(p(x), 4, 32, 32, p(q), 8, p(f), p(a), st) == -2    # ldq < C/2
    assert lib.puro_nvfp4_quantize_1x16(p(x), 4, 32, 32, p(q) + 1, 16, p(f), p(a), st) == -3  # alignment
    assert lib.puro_nvfp4_quantize_1x16_transposed(p(x), 4, 32, 32, p(q), 16, p(f), p(a), st) == -2  # R % 64
    assert lib.puro_nvfp4_quantize_1x16_dual(p(x), 4, 32, 32, p(q), 16, p(f), p(q), 16, p(f), p(a), st) == -2
    x64 = torch.zeros((64, 32), dtype=torch.bfloat16, device="cuda")
    q64, qt64 = torch.zeros((64, 16), dtype=torch.uint8, device="cuda"), torch.zeros((32, 32), dtype=torch.uint8, device="cuda")
    f64 = torch.zeros((1, 64, 16), dtype=torch.uint8, device="cuda")
    assert lib.puro_nvfp4_quantize_1x16_dual(p(x64), 64, 32, 32, p(q64), 16, p(f64), p(qt64), 32, p(f64), p(a), st) == 0
    assert lib.puro_nvfp4_quantize_1x16_dual(p(x64), 64, 32, 32, p(q64), 16, p(f64), p(qt64), 40, p(f64), p(a), st) == -3
    assert lib.puro_nvfp4_quantize_1x16_dual(p(x64), 64, 32, 32, p(q64), 16, None, p(qt64), 32, p(f64), p(a), st) == -1
    c = torch.zeros((128, 8), dtype=torch.bfloat16, device="cuda")
    ops = torch.zeros((128, 64), dtype=torch.uint8, device="cuda")
    fs = torch.zeros((128, 8), dtype=torch.uint8, device="cuda")
    assert lib.puro_nvfp4_gemm(p(ops), p(fs), p(a), p(ops), p(fs), p(a), p(c), 128, 8, 96, st) == -2  # K % 128
    assert lib.puro_nvfp4_gemm(p(ops), p(fs), None, p(ops), p(fs), p(a), p(c), 128, 8, 128, st) == -1
    assert lib.puro_nvfp4_gemm(p(ops), p(fs), p(a), p(ops), p(fs), p(a), p(c), 128, 12, 128, st) == -2  # N % 8
