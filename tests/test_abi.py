"""The C-ABI library builds, loads and exports every entry point include/puro_fp8.h declares,
and rejects bad arguments on the host with the documented status codes.

No call here carries arguments that pass validation, so nothing is ever launched: these
tests are safe with or without a GPU (the fake pointers never reach a kernel).
"""

import ctypes
import os
import re

import pytest
import torch

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "puro_fp8.h")

OK, ENULL, ESHAPE, EALIGN, ELAYOUT, ECUDA = 0, -1, -2, -3, -4, -8
A16 = 0x10000  # a 16-byte-aligned fake address (never dereferenced)


@pytest.fixture(scope="module")
def lib():
    from fp8_blockwise_scaled_e4m3_b200 import build
    build.build()
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8
    return puro_fp8.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"PURO_API\s+[\w\s\*]+?\b(puro_\w+)\s*\(", text)))


def exported_symbols(path):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    return sorted({line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("puro_")})


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted([
        "puro_fp8_quantize_1x128", "puro_fp8_quantize_1x128_transposed", "puro_fp8_quantize_128x128",
        "puro_fp8_gemm_blockwise", "puro_fp8_gemm_wgrad_acc_f32", "puro_fp8_gemm_blockwise_quant",
        "puro_fp8_gemm_blockwise_grouped", "puro_fp8_quantize_1x128_pow2",
        "puro_fp8_quantize_1x128_transposed_pow2", "puro_fp8_quantize_128x128_pow2", "puro_fp8_mx_gemm",
        "puro_fp8_quantize_128x128_grouped",
        "puro_nvfp4_quantize_1x16", "puro_nvfp4_quantize_1x16_transposed", "puro_nvfp4_quantize_1x16_dual",
        "puro_nvfp4_gemm", "puro_fp8_sync_status", "puro_strerror"])


def test_library_exports_exactly_the_declared_symbols(lib):
    from fp8_blockwise_scaled_e4m3_b200.build import LIB
    assert exported_symbols(LIB) == declared_functions()
    for name in declared_functions():
        assert hasattr(lib, name)


def test_strerror_covers_every_status(lib):
    for s in range(-9, 1):
        assert lib.puro_strerror(s) and lib.puro_strerror(s) != b"unknown status"
    assert lib.puro_strerror(-1234) == b"unknown status"


def test_quantize_1x128_validation(lib):
    f = lib.puro_fp8_quantize_1x128
    assert f(None, 4, 128, 128, A16, 128, A16, None) == ENULL
    assert f(A16, 0, 128, 128, A16, 128, A16, None) == ESHAPE
    assert f(A16, 4, 100, 128, A16, 128, A16, None) == ESHAPE      # C % 128
    assert f(A16, 4, 256, 128, A16, 256, A16, None) == ESHAPE      # ldx < C
    assert f(A16 + 2, 4, 128, 128, A16, 128, A16, None) == EALIGN  # X not 16-byte aligned
    assert f(A16, 4, 128, 132, A16, 128, A16, None) == EALIGN      # ldx % 8
    assert f(A16, 4, 128, 128, A16, 136, A16, None) == EALIGN      # ldq % 16


def test_quantize_transposed_validation(lib):
    f = lib.puro_fp8_quantize_1x128_transposed
    assert f(A16, 256, 64, 64, None, A16, None, None, None) == ENULL
    assert f(A16, 256, 64, 64, A16, A16, A16, None, None) == ENULL   # Xq without S
    assert f(A16, 200, 64, 64, A16, A16, None, None, None) == ESHAPE  # T % 128
    assert f(A16, 256, 60, 64, A16, A16, None, None, None) == ESHAPE  # C % 8
    assert f(A16, 256, 64, 64, A16, A16, A16, A16, None) == ESHAPE    # dual needs C % 128
    assert f(A16, 256, 64, 64, A16 + 8, A16, None, None, None) == EALIGN


def test_quantize_128x128_validation(lib):
    f = lib.puro_fp8_quantize_128x128
    assert f(A16, 300, 256, 256, None, None, A16, None) == ENULL
    assert f(A16, 300, 200, 256, A16, None, A16, None) == ESHAPE
    assert f(A16, 300, 256, 256, A16, A16, A16, None) == ESHAPE      # WqT needs R % 16
    assert f(A16, 304, 256, 256, A16, A16 + 4, A16, None) == EALIGN


def test_gemm_validation(lib):
    f = lib.puro_fp8_gemm_blockwise
    args = [A16, A16, A16, A16, A16]
    assert f(None, *args[1:], 128, 256, 256, 0, None, 0, None) == ENULL
    assert f(*args, 128, 256, 256, 7, None, 0, None) == ELAYOUT
    assert f(*args, 0, 256, 256, 0, None, 0, None) == ESHAPE
    assert f(*args, 128, 250, 256, 0, None, 0, None) == ESHAPE       # N % 8
    assert f(*args, 128, 256, 200, 0, None, 0, None) == ESHAPE       # K % 128
    assert f(A16 + 1, *args[1:], 128, 256, 256, 0, None, 0, None) == EALIGN
    assert f(*args[:3], A16 + 2, A16, 128, 256, 256, 2, None, 0, None) == EALIGN  # Bs
    assert f(A16, A16 + 1, *args[2:], 128, 256, 256, 1, None, 0, None) == EALIGN  # As


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_without_gpu_calls_report_cuda_error(lib):
    assert lib.puro_fp8_sync_status(None) == ECUDA


def test_wgrad_acc_f32_rejects_bad_arguments(lib):
    f = lib.puro_fp8_gemm_wgrad_acc_f32
    args = [A16, A16, A16, A16, A16]
    assert f(None, *args[1:], 128, 256, 256, None) == ENULL
    assert f(*args, 0, 256, 256, None) == ESHAPE
    assert f(*args, 128, 250, 256, None) == ESHAPE       # N % 8
    assert f(*args, 128, 256, 200, None) == ESHAPE       # K % 128
    assert f(*args[:4], A16 + 4, 128, 256, 256, None) == EALIGN   # C not 16-byte aligned


def test_empty_and_negative_dimensions_are_shape_errors(lib):
    """Every entry point rejects zero and negative sizes on the host, before any launch."""
    q1 = lib.puro_fp8_quantize_1x128
    assert q1(A16, -4, 128, 128, A16, 128, A16, None) == ESHAPE
    assert q1(A16, 4, 0, 128, A16, 128, A16, None) == ESHAPE
    qt = lib.puro_fp8_quantize_1x128_transposed
    assert qt(A16, 0, 64, 64, A16, A16, None, None, None) == ESHAPE
    assert qt(A16, -128, 64, 64, A16, A16, None, None, None) == ESHAPE
    assert qt(A16, 256, 0, 64, A16, A16, None, None, None) == ESHAPE
    qw = lib.puro_fp8_quantize_128x128
    assert qw(A16, 0, 256, 256, A16, None, A16, None) == ESHAPE
    assert qw(A16, -1, 256, 256, A16, None, A16, None) == ESHAPE
    assert qw(A16, 300, 0, 256, A16, None, A16, None) == ESHAPE
    g = lib.puro_fp8_gemm_blockwise
    args = [A16, A16, A16, A16, A16]
    for layout in (0, 1, 2):
        assert g(*args, 128, 0, 256, layout, None, 0, None) == ESHAPE
        assert g(*args, 128, 256, 0, layout, None, 0, None) == ESHAPE
        assert g(*args, -128, 256, 256, layout, None, 0, None) == ESHAPE
    acc = lib.puro_fp8_gemm_wgrad_acc_f32
    assert acc(*args, 128, 0, 256, None) == ESHAPE
    assert acc(*args, 128, 256, 0, None) == ESHAPE


def test_tile_counts_beyond_32_bit_indices_are_shape_errors(lib):
    """Sizes that pass every per-dimension bound but whose tile count would overflow the
    kernels' 32-bit tile indices are rejected on the host."""
    big = (1 << 31) - 256
    g = lib.puro_fp8_gemm_blockwise
    args = [A16, A16, A16, A16, A16]
    assert g(*args, big, big, 128, 0, None, 0, None) == ESHAPE
    assert lib.puro_fp8_gemm_wgrad_acc_f32(*args, big, big, 128, None) == ESHAPE
    q1 = lib.puro_fp8_quantize_1x128
    c = 65535 * 128
    assert q1(A16, (1 << 31) - 1, c, c, A16, c, A16, None) == ESHAPE
    qt = lib.puro_fp8_quantize_1x128_transposed
    assert qt(A16, 65535 * 128, 1 << 30, 1 << 30, A16, A16, None, None, None) == ESHAPE
    qw = lib.puro_fp8_quantize_128x128
    assert qw(A16, 65535 * 128, 1 << 30, 1 << 30, A16, None, A16, None) == ESHAPE


def test_binding_refuses_tensors_of_the_wrong_shape(lib):
    """The Python wrappers check every output and scale tensor against the extents the C
    declaration gives before anything reaches the device (CPU tensors suffice)."""
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8 as pf
    bf, u8, f32 = torch.bfloat16, torch.uint8, torch.float32
    z = lambda *s, dt=f32: torch.zeros(s, dtype=dt)
    X = z(256, 384, dt=bf)
    cases = [
        (lambda: pf.puro_fp8_quantize_1x128(X, z(256, 256, dt=u8), z(3, 256)), "Xq"),
        (lambda: pf.puro_fp8_quantize_1x128(X, z(256, 384, dt=u8), z(256, 3)), "S"),
        (lambda: pf.puro_fp8_quantize_1x128(z(2, 256, 384, dt=bf), z(256, 384, dt=u8), z(3, 256)), "2-D"),
        (lambda: pf.puro_fp8_quantize_1x128_transposed(X, z(256, 384, dt=u8), z(2, 384)), "XqT"),
        (lambda: pf.puro_fp8_quantize_1x128_transposed(X, z(384, 256, dt=u8), z(384, 2)), "ST"),
        (lambda: pf.puro_fp8_quantize_1x128_transposed(X, z(384, 256, dt=u8), z(2, 384),
                                                       z(256, 128, dt=u8), z(3, 256)), "Xq"),
        (lambda: pf.puro_fp8_quantize_128x128(X, z(256, 384, dt=u8), z(256, 384, dt=u8), z(2, 3)), "WqT"),
        (lambda: pf.puro_fp8_quantize_128x128(X, z(256, 384, dt=u8), None, z(3, 2)), "S"),
    ]
    M, N, K = 256, 384, 512
    Aq, Bq, C = z(M, K, dt=u8), z(N, K, dt=u8), z(M, N, dt=bf)
    As = z(K // 128, M)
    cases += [
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, z(N, 256, dt=u8), z(3, 4), C, "fprop"), "Bq"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, Bq, z(4, 3), C, "fprop"), "Bs"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, Bq, z(3, 4), C, "dgrad"), "Bs"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, Bq, z(4, 3), C, "wgrad"), "Bs"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, z(M, K // 128), Bq, z(3, 4), C, "fprop"), "As"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, Bq, z(3, 4), z(N, M, dt=bf), "fprop"), "C"),
        (lambda: pf.puro_fp8_gemm_blockwise(Aq, As, Bq, z(3, 4), C, 7), "layout"),
        (lambda: pf.puro_fp8_gemm_wgrad_acc_f32(Aq, As, Bq, z(K // 128, N - 8), z(M, N)), "Bs"),
        (lambda: pf.puro_fp8_gemm_wgrad_acc_f32(Aq, As, Bq, z(K // 128, N), z(M, N - 8)), "C"),
    ]
    for call, what in cases:
        with pytest.raises(ValueError, match=what):
            call()


def test_gemm_quant_rejects_bad_arguments(lib):
    """The fused-quantisation GEMM: fprop / dgrad only, N a multiple of 128 (the groups run
    along N), every output present and aligned; all checked before any launch."""
    f = lib.puro_fp8_gemm_blockwise_quant
    ops = [A16, A16, A16, A16, A16, A16, A16]
    assert f(None, *ops[1:], 128, 256, 256, 0, None) == ENULL
    assert f(*ops[:5], None, A16, 128, 256, 256, 0, None) == ENULL      # Cq
    assert f(*ops[:6], None, 128, 256, 256, 0, None) == ENULL           # Cs
    assert f(*ops, 128, 256, 256, 2, None) == ELAYOUT                   # wgrad has no fused form
    assert f(*ops, 128, 256, 256, 7, None) == ELAYOUT
    assert f(*ops, 128, 200, 256, 0, None) == ESHAPE                    # N % 128
    assert f(*ops, 0, 256, 256, 1, None) == ESHAPE
    assert f(*ops, 128, 256, 200, 0, None) == ESHAPE                    # K % 128
    assert f(*ops[:5], A16 + 8, A16, 128, 256, 256, 0, None) == EALIGN  # Cq not 16-byte aligned
    assert f(*ops[:6], A16 + 2, 128, 256, 256, 0, None) == EALIGN       # Cs not 4-byte aligned


def test_gemm_grouped_rejects_bad_arguments(lib):
    """The grouped GEMM checks the count, the layout and every problem as the single call
    does, before anything is launched; one bad problem rejects the whole group."""
    from fp8_blockwise_scaled_e4m3_b200.puro_fp8 import GROUP_MAX, GemmProblem
    f = lib.puro_fp8_gemm_blockwise_grouped
    good = GemmProblem(A16, A16, A16, A16, A16, 128, 256, 256)
    arr = (GemmProblem * (GROUP_MAX + 1))(*([good] * (GROUP_MAX + 1)))
    ptr = ctypes.cast(arr, ctypes.c_void_p)
    assert f(None, 2, 0, None) == ENULL
    assert f(ptr, 0, 0, None) == ESHAPE
    assert f(ptr, GROUP_MAX + 1, 0, None) == ESHAPE
    assert f(ptr, 2, 3, None) == ELAYOUT
    arr[1] = GemmProblem(A16, A16, A16, A16, A16, 128, 250, 256)     # N % 8
    assert f(ptr, 2, 0, None) == ESHAPE
    arr[1] = GemmProblem(A16, A16, None, A16, A16, 128, 256, 256)    # Bq
    assert f(ptr, 2, 2, None) == ENULL
    arr[1] = GemmProblem(A16, A16, A16, A16, A16 + 8, 128, 256, 256)  # C not 16-byte aligned
    assert f(ptr, 2, 1, None) == EALIGN


def test_quantize_grouped_rejects_bad_arguments(lib):
    """The grouped weight quantiser checks the count and every weight as the single call
    does, before anything is launched; one bad weight rejects the whole call."""
    from fp8_blockwise_scaled_e4m3_b200.puro_fp8 import WeightProblem
    f = lib.puro_fp8_quantize_128x128_grouped
    good = WeightProblem(A16, 256, 256, 256, A16, A16, A16)
    arr = (WeightProblem * 3)(good, good, good)
    ptr = ctypes.cast(arr, ctypes.c_void_p)
    assert f(None, 2, None) == ENULL
    assert f(ptr, 0, None) == ESHAPE
    arr[2] = WeightProblem(A16, 100, 256, 256, A16, A16, A16)    # WqT needs R % 16
    assert f(ptr, 3, None) == ESHAPE
    arr[2] = WeightProblem(A16, 128, 200, 256, A16, None, A16)   # C % 128
    assert f(ptr, 3, None) == ESHAPE
    arr[2] = WeightProblem(A16, 128, 256, 256, None, None, A16)  # Wq
    assert f(ptr, 3, None) == ENULL
    arr[2] = WeightProblem(A16, 128, 256, 252, A16, None, A16)   # ldw < C
    assert f(ptr, 3, None) == ESHAPE
    arr[2] = WeightProblem(A16, 128, 256, 256, A16, None, A16 + 2)  # S not 4-byte aligned
    assert f(ptr, 3, None) == EALIGN


def test_pow2_quantisers_reject_bad_arguments(lib):
    """The power-of-two scale mode checks its arguments like the FP32-scale quantisers; byte
    scales need no alignment."""
    q = lib.puro_fp8_quantize_1x128_pow2
    assert q(None, 4, 128, 128, A16, 128, A16, None) == ENULL
    assert q(A16, 4, 100, 128, A16, 128, A16, None) == ESHAPE
    assert q(A16 + 2, 4, 128, 128, A16, 128, A16, None) == EALIGN
    qt = lib.puro_fp8_quantize_1x128_transposed_pow2
    assert qt(A16, 100, 64, 64, A16, A16, None, None, None) == ESHAPE        # T % 128
    assert qt(A16, 256, 64, 64, A16, A16, A16, None, None) == ENULL          # Xq without S
    qw = lib.puro_fp8_quantize_128x128_pow2
    assert qw(A16, 100, 256, 256, A16, A16, A16, None) == ESHAPE             # WqT needs R % 16
    assert qw(A16, 128, 256, 256, A16 + 4, None, A16, None) == EALIGN


def test_mx_gemm_rejects_bad_arguments(lib):
    f = lib.puro_fp8_mx_gemm
    ops = [A16, A16, A16, A16, A16]
    assert f(None, *ops[1:], 128, 256, 256, 0, None) == ENULL
    assert f(*ops, 128, 256, 256, 5, None) == ELAYOUT
    assert f(*ops, 128, 250, 256, 0, None) == ESHAPE
    assert f(*ops, 128, 256, 200, 2, None) == ESHAPE
    assert f(*ops[:4], A16 + 2, 128, 256, 256, 1, None) == EALIGN
    assert f(*ops[:3], A16 + 4, A16, 128, 256, 256, 2, None) == EALIGN   # wgrad Bs 8-byte aligned


def test_nvfp4_entry_points_reject_bad_arguments(lib):
    """NVFP4 quantisers and GEMM: NULL pointers, shapes and alignment are refused on the host,
    before any device work."""
    q = lib.puro_nvfp4_quantize_1x16
    assert q(None, 4, 32, 32, A16, 16, A16, A16, None) == ENULL
    assert q(A16, 4, 32, 32, A16, 16, A16, None, None) == ENULL              # amax
    assert q(A16, 4, 24, 32, A16, 16, A16, A16, None) == ESHAPE              # C % 16
    assert q(A16, 4, 32, 32, A16, 8, A16, A16, None) == ESHAPE               # ldq < C / 2
    assert q(A16, 4, 32, 32, A16 + 8, 16, A16, A16, None) == EALIGN          # Xq 16-byte aligned
    assert q(A16, 4, 32, 36, A16, 16, A16, A16, None) == EALIGN              # ldx % 8
    assert q(A16, 4, 32, 32, A16, 16, A16, A16 + 2, None) == EALIGN          # amax 4-byte aligned
    qt = lib.puro_nvfp4_quantize_1x16_transposed
    assert qt(A16, 100, 64, 64, A16, 64, A16, A16, None) == ESHAPE           # R % 64
    assert qt(A16, 128, 60, 64, A16, 64, A16, A16, None) == ESHAPE           # C % 8
    assert qt(A16, 128, 64, 64, A16, 32, A16, A16, None) == ESHAPE           # ldq < R / 2
    assert qt(A16, 128, 64, 64, A16, 72, A16, A16, None) == EALIGN           # ldq % 16
    d = lib.puro_nvfp4_quantize_1x16_dual
    assert d(A16, 128, 64, 64, A16, 32, A16, None, 64, A16, A16, None) == ENULL      # XqT
    assert d(A16, 100, 64, 64, A16, 32, A16, A16, 64, A16, A16, None) == ESHAPE      # R % 64
    assert d(A16, 128, 56, 64, A16, 32, A16, A16, 64, A16, A16, None) == ESHAPE      # C % 16
    assert d(A16, 128, 64, 64, A16, 32, A16, A16, 48, A16, A16, None) == ESHAPE      # ldqt < R / 2
    assert d(A16, 128, 64, 64, A16, 32, A16, A16, 72, A16, A16, None) == EALIGN      # ldqt % 16
    assert d(A16, 128, 64, 64, A16, 36, A16, A16, 64, A16, A16, None) == EALIGN      # ldq % 8
    assert d(A16, 128, 64, 64, A16, 32, A16, A16, 64, A16 + 4, A16, None) == EALIGN  # FT 16-byte aligned
    g = lib.puro_nvfp4_gemm
    ops = [A16, A16, A16, A16, A16, A16, A16]
    assert g(None, *ops[1:], 128, 256, 256, None) == ENULL
    assert g(*ops[:2], None, *ops[3:], 128, 256, 256, None) == ENULL        # a_amax
    assert g(*ops, 128, 250, 256, None) == ESHAPE                            # N % 8
    assert g(*ops, 128, 256, 200, None) == ESHAPE                            # K % 128
    assert g(*ops, 0, 256, 256, None) == ESHAPE
    assert g(A16, A16 + 8, *ops[2:], 128, 256, 256, None) == EALIGN          # As 16-byte aligned
    assert g(*ops[:6], A16 + 2, 128, 256, 256, None) == EALIGN               # C
