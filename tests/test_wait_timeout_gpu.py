"""Failure detection without a GPU fault: the bounded mbarrier wait every kernel uses.

A wait on a barrier phase that nothing completes (the "flag that nothing sets") must give
up after its limit, return false and leave the context usable; a completed phase must be
seen at once. The kernels turn such a give-up into the device status word that
puro_fp8_sync_status() reports as PURO_ERR_TIMEOUT; the status must be clean after
normal runs.
"""

import ctypes
import os
import subprocess

import pytest
import torch

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu

SRC = os.path.join(ROOT, "tests", "cuda", "wait_timeout.cu")
HDR = os.path.join(ROOT, "fp8_blockwise_scaled_e4m3_b200", "csrc", "ptx.cuh")
LIB = os.path.join(ROOT, "tests", "cuda", "_build", "libwait_check.so")


def _build():
    if os.path.exists(LIB) and os.path.getmtime(LIB) > max(os.path.getmtime(SRC), os.path.getmtime(HDR)):
        return
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared",
                    "-Xcompiler", "-fPIC", "-o", LIB, SRC], check=True)


def test_bounded_wait_gives_up_and_context_survives():
    _build()
    lib = ctypes.CDLL(LIB)
    out = (ctypes.c_ulonglong * 4)()
    timeout_ns = 20_000_000  # 20 ms
    assert lib.run_wait_check(ctypes.c_ulonglong(timeout_ns), out) == 0
    never_ok, never_ns, done_ok, done_ns = list(out)
    assert never_ok == 0, "a wait on a phase nothing completes must give up"
    assert timeout_ns <= never_ns < 50 * timeout_ns, never_ns
    assert done_ok == 1 and done_ns < timeout_ns
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_status_word_clean_after_normal_runs():
    from fp8_blockwise_scaled_e4m3_b200 import puro_fp8 as pf
    x = torch.randn(256, 512, device="cuda").to(torch.bfloat16)
    pf.quantize_1x128(x)
    pf.puro_fp8_sync_status()  # raises PuroError(PURO_ERR_TIMEOUT) if any wait gave up
