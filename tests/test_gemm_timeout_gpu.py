"""Failure detection inside a product kernel, without a GPU fault.

A test-only build of the library (the product sources compiled with PURO_TEST_HOOKS, a
flag libpuro_fp8.so never sets) can make the GEMM's promotion warps withhold one hand-back
of a TMEM buffer. On a one-tile grid the MMA warp's bounded wait for that buffer then runs
out. The test checks, in a child process whose wait limit is 20 ms:

* the call itself is accepted (the give-up happens on the device, after the launch);
* puro_fp8_sync_status() reports PURO_ERR_TIMEOUT: the give-up raised the CTA's abort
  flag and the device status word, the other warp roles left their loops, in-flight TMA
  loads and MMAs were waited for and TMEM was freed before the CTA exited;
* the status word is clear again after that read;
* with the hook off, the same GEMM on the same context runs clean and gives the exact
  result of an exact-integer case, so the context and the library stay usable.
Both promotion shapes are covered, fprop (32x32b TMEM loads) and wgrad (16x256b), on a
single-CTA tile (M = 128) and on one CTA pair's tile (M = 256: the withheld hand-back is
owed to the leader's barrier by both CTAs, and each CTA gives up on its own bounded waits).
"""

import os
import subprocess
import sys

import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu

sys.path.insert(0, ROOT)
from fp8_blockwise_scaled_e4m3_b200 import build as pbuild  # noqa: E402

LIB = os.path.join(ROOT, "tests", "cuda", "_build", "libpuro_fp8_testhooks.so")


def _build():
    deps = [os.path.join(pbuild.CSRC, f) for f in pbuild.SOURCES + pbuild.HEADERS]
    deps.append(os.path.join(ROOT, "include", "puro_fp8.h"))
    if os.path.exists(LIB) and os.path.getmtime(LIB) > max(os.path.getmtime(d) for d in deps):
        return
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    objs = []
    for src in pbuild.SOURCES:
        obj = os.path.join(os.path.dirname(LIB), "hooks_" + src.replace(".cu", ".o"))
        subprocess.run([pbuild.NVCC, *pbuild.ARCH, *pbuild.FLAGS, "-DPURO_TEST_HOOKS",
                        "-I", os.path.join(ROOT, "include"), "-c", os.path.join(pbuild.CSRC, src),
                        "-o", obj], check=True)
        objs.append(obj)
    subprocess.run([pbuild.NVCC, *pbuild.ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs], check=True)
    for o in objs:
        os.remove(o)


CHILD = r"""
import ctypes, sys
import numpy as np
import torch
lib = ctypes.CDLL(sys.argv[1])
layout = int(sys.argv[2])
M = int(sys.argv[3])
p, i64 = ctypes.c_void_p, ctypes.c_int64
lib.puro_fp8_gemm_blockwise.argtypes = [p, p, p, p, p, i64, i64, i64, ctypes.c_int, p, ctypes.c_size_t, p]
lib.puro_fp8_sync_status.argtypes = [p]
N, K = 256, 1024                  # one output tile (128 x 256, or a CTA pair's 256 x 256), 8 K blocks
rng = np.random.default_rng(1)
codes = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)    # 0, +-1, +-2
aq = codes[rng.integers(0, 5, size=(M, K))]
bq = codes[rng.integers(0, 5, size=(N, K))]
nb = (N + 127) // 128
bs_shape = {0: (nb, K // 128), 2: (K // 128, N)}[layout]
a_s = np.ones((K // 128, M), np.float32)
b_s = np.ones(bs_shape, np.float32)
dec = {0x00: 0, 0x38: 1, 0xB8: -1, 0x40: 2, 0xC0: -2}
want = np.vectorize(dec.get)(aq).astype(np.int64) @ np.vectorize(dec.get)(bq).astype(np.int64).T
dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
A, As, B, Bs = dev(aq), dev(a_s), dev(bq), dev(b_s)
C = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
args = [A.data_ptr(), As.data_ptr(), B.data_ptr(), Bs.data_ptr(), C.data_ptr(), M, N, K, layout, None, 0, st]
out = []
out.append(lib.puro_test_set_skip_release(1))
out.append(lib.puro_fp8_gemm_blockwise(*args))        # accepted: the give-up happens on the device
out.append(lib.puro_fp8_sync_status(st))              # -> PURO_ERR_TIMEOUT
out.append(lib.puro_fp8_sync_status(st))              # cleared by the read -> PURO_OK
out.append(lib.puro_test_set_skip_release(0))
C.zero_()
out.append(lib.puro_fp8_gemm_blockwise(*args))
out.append(lib.puro_fp8_sync_status(st))
want_bf16 = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16).float().numpy()  # |C| <= 4096: FP32 exact, BF16 rounds once
exact = bool(np.array_equal(C.float().cpu().numpy(), want_bf16))
print("RESULT", *out, int(exact), flush=True)
"""


@pytest.mark.parametrize("m", [128, 256], ids=["single_cta", "cta_pair"])
@pytest.mark.parametrize("layout", [0, 2], ids=["fprop", "wgrad"])
def test_gemm_wait_gives_up_reports_timeout_and_context_survives(layout, m):
    _build()
    env = dict(os.environ, PURO_WAIT_TIMEOUT_MS="20")
    r = subprocess.run([sys.executable, "-c", CHILD, LIB, str(layout), str(m)], capture_output=True, text=True,
                       env=env, timeout=300)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT")]
    assert r.returncode == 0 and lines, r.stdout + r.stderr
    hook_on, launch, first, second, hook_off, relaunch, final, exact = map(int, lines[-1].split()[1:])
    assert hook_on == 0 and hook_off == 0
    assert launch == 0, "the call is accepted; the give-up happens on the device"
    assert first == -6, f"sync_status after the withheld release: {first} (want PURO_ERR_TIMEOUT)"
    assert second == 0, "reading the status word clears it"
    assert relaunch == 0 and final == 0, "the context and the library stay usable"
    assert exact == 1, "the GEMM after the timeout gives the exact result"
