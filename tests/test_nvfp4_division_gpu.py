"""The NVFP4 quantisers' group arithmetic equals IEEE division over its whole domain.

The kernels form a group's factor RN(RN(amax_g / 6) / s_t) and every code's quotient RN(x / S)
with Markstein's FMA correction of a product by a correctly rounded reciprocal (IEEE division
where a value could leave the normal range). Because every input is a BF16 number and S is
built from a BF16 tensor amax and one of 127 factor bytes, the domain is finite, and
tests/cuda/nvfp4_exhaustive.cu checks all of it against __fdiv_rn:
- every positive finite BF16 tensor amax with every BF16 group amax not above it (the factor
  byte and S bit for bit; the decode of each factor byte against CUDA's E4M3 conversion);
- every tensor amax and factor byte with every BF16 x of either sign in [S/32, 16 S], plus zero
  and the smallest subnormal (the E2M1 codes of the packed helpers the kernels call).
"""

import ctypes
import os
import subprocess

import numpy as np
import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu

SRC = os.path.join(ROOT, "tests", "cuda", "nvfp4_exhaustive.cu")
HDRS = [os.path.join(ROOT, "fp8_blockwise_scaled_e4m3_b200", "csrc", h)
        for h in ("nvfp4_math.cuh", "quant_math.cuh", "ptx.cuh")]
LIB = os.path.join(ROOT, "tests", "cuda", "_build", "libnvfp4_check.so")


def _build():
    if os.path.exists(LIB) and os.path.getmtime(LIB) > max(os.path.getmtime(p) for p in [SRC] + HDRS):
        return
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-prec-div=true",
                    "-ftz=false", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-o", LIB, SRC], check=True)


def test_group_factor_matches_ieee_division_exhaustively():
    """Both the general path and, for tensors with s_t >= 2^-81, the all-fast path."""
    _build()
    lib = ctypes.CDLL(LIB)
    counts = (ctypes.c_ulonglong * 3)()
    first = ctypes.c_uint(0)
    assert lib.run_nvfp4_factor_check(counts, ctypes.byref(first)) == 0
    bad, checked, checked_all_fast = list(counts)
    n_t = 0x7F7F
    assert checked == n_t * (n_t + 1) // 2 + n_t  # group amax 0 .. tensor amax, per tensor amax
    tb = np.arange(1, n_t + 1, dtype=np.uint32)
    s_t = (tb << 16).view(np.float32) / np.float32(2688.0)  # IEEE float32 division
    assert checked_all_fast == int((tb[s_t >= np.float32(2.0 ** -81)].astype(np.int64) + 1).sum())
    assert bad == 0, f"{bad} factor mismatches, first (tensor amax << 16 | group amax) = {first.value:#010x}"


def test_codes_match_ieee_division_exhaustively():
    _build()
    lib = ctypes.CDLL(LIB)
    counts = (ctypes.c_ulonglong * 3)()
    first = ctypes.c_uint(0)
    assert lib.run_nvfp4_codes_check(counts, ctypes.byref(first)) == 0
    bad, checked, _ = list(counts)
    print(f"values checked: {checked}")
    # 0x7F7F tensor amaxes x 126 non-zero factors x (about 9 binades of 128 values, 2 signs)
    assert checked > 0x7F7F * 126 * 1500
    assert bad == 0, f"{bad} code mismatches, first (tensor amax << 16 | x) = {first.value:#010x}"
