"""Failure detection inside the block-scaled GEMM and the quantisers, without a GPU fault.

The test-only build of the library (tests/test_gemm_timeout_gpu.py builds it with
PURO_TEST_HOOKS, a flag libpuro_fp8.so never sets) has two more hooks:

* the block-scaled GEMM's scale writers withhold their arrival for the first K block, so
  the MMA issuer's bounded wait for the scale factors runs out (single CTA and CTA pair,
  fprop and wgrad);
* the quantiser skips the load of each CTA's first tile, so the bounded wait for it runs
  out (row-wise, dual and grouped weight launches), and so does the NVFP4 dual quantiser.

In a child process whose wait limit is 20 ms, each call is accepted (the give-up happens on
the device), puro_fp8_sync_status() reports PURO_ERR_TIMEOUT and clears the status word,
and with the hook off the same call on the same context gives the exact result.
"""

import os
import subprocess
import sys

import pytest

from tests.conftest import ROOT
from tests.test_gemm_timeout_gpu import LIB, _build

pytestmark = pytest.mark.gpu

CHILD_MX = r"""
import ctypes, sys
import numpy as np
import torch
lib = ctypes.CDLL(sys.argv[1])
layout, M = int(sys.argv[2]), int(sys.argv[3])
p, i64 = ctypes.c_void_p, ctypes.c_int64
lib.puro_fp8_mx_gemm.argtypes = [p, p, p, p, p, i64, i64, i64, ctypes.c_int, p]
lib.puro_fp8_sync_status.argtypes = [p]
N, K = 256, 1024
rng = np.random.default_rng(2)
codes = np.array([0x00, 0x38, 0xB8, 0x40, 0xC0], dtype=np.uint8)    # 0, +-1, +-2
aq = codes[rng.integers(0, 5, size=(M, K))]
bq = codes[rng.integers(0, 5, size=(N, K))]
bs_shape = {0: ((N + 127) // 128, K // 128), 2: (K // 128, N)}[layout]
a_b = np.full((K // 128, M), 127, np.uint8)                        # scale 1
b_b = np.full(bs_shape, 127, np.uint8)
dec = {0x00: 0, 0x38: 1, 0xB8: -1, 0x40: 2, 0xC0: -2}
want = np.vectorize(dec.get)(aq).astype(np.int64) @ np.vectorize(dec.get)(bq).astype(np.int64).T
dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
A, As, B, Bs = dev(aq), dev(a_b), dev(bq), dev(b_b)
C = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
args = [A.data_ptr(), As.data_ptr(), B.data_ptr(), Bs.data_ptr(), C.data_ptr(), M, N, K, layout, st]
out = [lib.puro_test_set_mx_skip_sf(1), lib.puro_fp8_mx_gemm(*args), lib.puro_fp8_sync_status(st),
       lib.puro_fp8_sync_status(st), lib.puro_test_set_mx_skip_sf(0)]
C.zero_()
out += [lib.puro_fp8_mx_gemm(*args), lib.puro_fp8_sync_status(st)]
want_bf16 = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16).float().numpy()
out.append(int(np.array_equal(C.float().cpu().numpy(), want_bf16)))
print("RESULT", *out, flush=True)
"""

CHILD_QUANT = r"""
import ctypes, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[3])
from oracle import quant as oq
lib = ctypes.CDLL(sys.argv[1])
mode = sys.argv[2]
p, i64 = ctypes.c_void_p, ctypes.c_int64
lib.puro_fp8_quantize_1x128.argtypes = [p, i64, i64, i64, p, i64, p, p]
lib.puro_fp8_quantize_1x128_transposed.argtypes = [p, i64, i64, i64, p, p, p, p, p]
lib.puro_fp8_quantize_128x128_grouped.argtypes = [p, ctypes.c_int, p]
lib.puro_fp8_sync_status.argtypes = [p]
T, Cn = 512, 384
g = torch.Generator().manual_seed(3)
x = (torch.randn((T, Cn), generator=g) * 2.0).to(torch.bfloat16)
bits = x.view(torch.int16).numpy().view(np.uint16)
xd = x.cuda()
st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
u8, f32 = torch.uint8, torch.float32
if mode == "rows":
    q = torch.zeros((T, Cn), dtype=u8, device="cuda"); s = torch.zeros((Cn // 128, T), dtype=f32, device="cuda")
    call = lambda: lib.puro_fp8_quantize_1x128(xd.data_ptr(), T, Cn, Cn, q.data_ptr(), Cn, s.data_ptr(), st)
    outs = lambda: [(q, oq.quant_1x128(bits)[0]), (s, oq.quant_1x128(bits)[1])]
elif mode == "dual":
    qt = torch.zeros((Cn, T), dtype=u8, device="cuda"); s_t = torch.zeros((T // 128, Cn), dtype=f32, device="cuda")
    q = torch.zeros((T, Cn), dtype=u8, device="cuda"); s = torch.zeros((Cn // 128, T), dtype=f32, device="cuda")
    call = lambda: lib.puro_fp8_quantize_1x128_transposed(xd.data_ptr(), T, Cn, Cn, qt.data_ptr(), s_t.data_ptr(),
                                                          q.data_ptr(), s.data_ptr(), st)
    outs = lambda: [(qt, oq.quant_1x128_transposed(bits)[0]), (s_t, oq.quant_1x128_transposed(bits)[1]),
                    (q, oq.quant_1x128(bits)[0]), (s, oq.quant_1x128(bits)[1])]
else:  # grouped weights: the same matrix twice
    class WeightProblem(ctypes.Structure):  # puro_weight_problem
        _fields_ = [("W", p), ("R", i64), ("C", i64), ("ldw", i64), ("Wq", p), ("WqT", p), ("S", p)]
    bufs = [(torch.zeros((T, Cn), dtype=u8, device="cuda"), torch.zeros((Cn, T), dtype=u8, device="cuda"),
             torch.zeros((T // 128, Cn // 128), dtype=f32, device="cuda")) for _ in range(2)]
    arr = (WeightProblem * 2)(*[WeightProblem(xd.data_ptr(), T, Cn, Cn, b[0].data_ptr(), b[1].data_ptr(), b[2].data_ptr())
                                for b in bufs])
    call = lambda: lib.puro_fp8_quantize_128x128_grouped(ctypes.cast(arr, p), 2, st)
    ref = oq.quant_128x128(bits)
    outs = lambda: [(b[j], ref[j]) for b in bufs for j in range(3)]
out = [lib.puro_test_set_quant_skip_load(1), call(), lib.puro_fp8_sync_status(st), lib.puro_fp8_sync_status(st),
       lib.puro_test_set_quant_skip_load(0), call(), lib.puro_fp8_sync_status(st)]
exact = True
for got, want in outs():
    got = got.cpu().numpy()
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), np.asarray(want).view(np.uint32)
    exact = exact and np.array_equal(got, want)
out.append(int(exact))
print("RESULT", *out, flush=True)
"""


CHILD_NV = r"""
import ctypes, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[2])
from oracle import nvfp4 as onv
lib = ctypes.CDLL(sys.argv[1])
p, i64 = ctypes.c_void_p, ctypes.c_int64
lib.puro_nvfp4_quantize_1x16_dual.argtypes = [p, i64, i64, i64, p, i64, p, p, i64, p, p, p]
lib.puro_fp8_sync_status.argtypes = [p]
R, Cn = 512, 384
x = (torch.randn((R, Cn), generator=torch.Generator().manual_seed(4)) * 2.0).to(torch.bfloat16)
bits = x.view(torch.int16).numpy().view(np.uint16)
xd = x.cuda()
st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
u8 = torch.uint8
q = torch.zeros((R, Cn // 2), dtype=u8, device="cuda"); f = torch.zeros(((Cn + 255) // 256, R, 16), dtype=u8, device="cuda")
qt = torch.zeros((Cn, R // 2), dtype=u8, device="cuda"); ft = torch.zeros(((R + 255) // 256, Cn, 16), dtype=u8, device="cuda")
amax = torch.zeros(1, device="cuda")
call = lambda: lib.puro_nvfp4_quantize_1x16_dual(xd.data_ptr(), R, Cn, Cn, q.data_ptr(), Cn // 2, f.data_ptr(),
                                                  qt.data_ptr(), R // 2, ft.data_ptr(), amax.data_ptr(), st)
out = [lib.puro_test_set_nv_skip_load(1), call(), lib.puro_fp8_sync_status(st), lib.puro_fp8_sync_status(st),
       lib.puro_test_set_nv_skip_load(0), call(), lib.puro_fp8_sync_status(st)]
by_row = lambda fb, groups: fb.transpose(1, 0, 2).reshape(fb.shape[1], -1)[:, :groups]  # [K blocks, rows, 16]
wq, wf, _ = onv.quant_1x16(bits)
tq, tf, _ = onv.quant_1x16_transposed(bits)
exact = (np.array_equal(q.cpu().numpy(), wq) and np.array_equal(by_row(f.cpu().numpy(), Cn // 16), wf)
         and np.array_equal(qt.cpu().numpy(), tq) and np.array_equal(by_row(ft.cpu().numpy(), R // 16), tf))
out.append(int(exact))
print("RESULT", *out, flush=True)
"""


def _run(child, *args):
    env = dict(os.environ, PURO_WAIT_TIMEOUT_MS="20")
    r = subprocess.run([sys.executable, "-c", child, LIB, *map(str, args)], capture_output=True, text=True,
                       env=env, timeout=300)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT")]
    assert r.returncode == 0 and lines, r.stdout + r.stderr
    hook_on, launch, first, second, hook_off, relaunch, final, exact = map(int, lines[-1].split()[1:])
    assert hook_on == 0 and hook_off == 0
    assert launch == 0, "the call is accepted; the give-up happens on the device"
    assert first == -6, f"sync_status after the withheld arrival: {first} (want PURO_ERR_TIMEOUT)"
    assert second == 0, "reading the status word clears it"
    assert relaunch == 0 and final == 0, "the context and the library stay usable"
    assert exact == 1, "the call after the timeout gives the exact result"


@pytest.mark.parametrize("m", [128, 256], ids=["single_cta", "cta_pair"])
@pytest.mark.parametrize("layout", [0, 2], ids=["fprop", "wgrad"])
def test_mx_gemm_wait_gives_up_reports_timeout_and_context_survives(layout, m):
    _build()
    _run(CHILD_MX, layout, m)


@pytest.mark.parametrize("mode", ["rows", "dual", "grouped_weights"])
def test_quantiser_wait_gives_up_reports_timeout_and_context_survives(mode):
    _build()
    _run(CHILD_QUANT, mode, ROOT)


def test_nvfp4_dual_quantiser_wait_gives_up_reports_timeout_and_context_survives():
    _build()
    _run(CHILD_NV, ROOT)
