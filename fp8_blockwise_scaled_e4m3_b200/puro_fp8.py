"""Python binding of libpuro_fp8.so: argument marshalling only.

Every function with a ``puro_`` name mirrors the C entry point of the same name in
``include/puro_fp8.h``: it takes torch tensors that already live on the GPU, checks that
each has the dtype and exact shape the declaration gives (``ValueError`` otherwise, so a
kernel never writes past a tensor), passes their device pointers, sizes and the current
CUDA stream, and raises ``PuroError`` on a non-zero status. The convenience functions below them allocate the outputs with torch
and call the same entry points. Nothing here computes: every step runs in the CUDA
kernels, and importing this module fails if the library has not been built.
"""

import ctypes
import os

import torch

from .build import LIB

PURO_FPROP, PURO_DGRAD, PURO_WGRAD = 0, 1, 2
LAYOUTS = {"fprop": PURO_FPROP, "dgrad": PURO_DGRAD, "wgrad": PURO_WGRAD}

_p = ctypes.c_void_p
_i64 = ctypes.c_int64


GROUP_MAX = 4  # PURO_GROUP_MAX


class GemmProblem(ctypes.Structure):
    """puro_gemm_problem: one GEMM of a grouped launch."""
    _fields_ = [("Aq", _p), ("As", _p), ("Bq", _p), ("Bs", _p), ("C", _p),
                ("M", _i64), ("N", _i64), ("K", _i64)]


class WeightProblem(ctypes.Structure):
    """puro_weight_problem: one weight of a grouped 128x128 quantisation."""
    _fields_ = [("W", _p), ("R", _i64), ("C", _i64), ("ldw", _i64),
                ("Wq", _p), ("WqT", _p), ("S", _p)]


class PuroError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status} ({strerror(status)})")


def _load():
    if not os.path.exists(LIB):
        raise ImportError(
            f"{LIB} is missing: build it with `python -m fp8_blockwise_scaled_e4m3_b200.build`")
    lib = ctypes.CDLL(LIB)
    sig = {
        "puro_fp8_quantize_1x128": [_p, _i64, _i64, _i64, _p, _i64, _p, _p],
        "puro_fp8_quantize_1x128_transposed": [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
        "puro_fp8_quantize_128x128": [_p, _i64, _i64, _i64, _p, _p, _p, _p],
        "puro_fp8_gemm_blockwise": [_p, _p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_int, _p,
                                    ctypes.c_size_t, _p],
        "puro_fp8_gemm_wgrad_acc_f32": [_p, _p, _p, _p, _p, _i64, _i64, _i64, _p],
        "puro_fp8_gemm_blockwise_quant": [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_int, _p],
        "puro_fp8_gemm_blockwise_grouped": [_p, ctypes.c_int, ctypes.c_int, _p],
        "puro_fp8_quantize_128x128_grouped": [_p, ctypes.c_int, _p],
        "puro_fp8_quantize_1x128_pow2": [_p, _i64, _i64, _i64, _p, _i64, _p, _p],
        "puro_fp8_mx_gemm": [_p, _p, _p, _p, _p, _i64, _i64, _i64, ctypes.c_int, _p],
        "puro_fp8_quantize_1x128_transposed_pow2": [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p],
        "puro_fp8_quantize_128x128_pow2": [_p, _i64, _i64, _i64, _p, _p, _p, _p],
        "puro_nvfp4_quantize_1x16": [_p, _i64, _i64, _i64, _p, _i64, _p, _p, _p],
        "puro_nvfp4_quantize_1x16_transposed": [_p, _i64, _i64, _i64, _p, _i64, _p, _p, _p],
        "puro_nvfp4_quantize_1x16_dual": [_p, _i64, _i64, _i64, _p, _i64, _p, _p, _i64, _p, _p, _p],
        "puro_nvfp4_gemm": [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p],
        "puro_fp8_sync_status": [_p],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.puro_strerror.argtypes = [ctypes.c_int]
    lib.puro_strerror.restype = ctypes.c_char_p
    return lib


_lib = _load()


def library():
    """The loaded ctypes.CDLL (for ABI tests)."""
    return _lib


def strerror(status: int) -> str:
    return _lib.puro_strerror(int(status)).decode()


# With PURO_CHECK_EACH_CALL=1 every call below is followed by puro_fp8_sync_status(), so a
# device-side wait that gave up is reported by the call whose kernel gave up (and the call
# becomes synchronous). Off by default: the calls then stay asynchronous, and a caller that
# needs valid outputs calls puro_fp8_sync_status() itself after the calls it depends on.
CHECK_EACH_CALL = os.environ.get("PURO_CHECK_EACH_CALL", "0") == "1"


def _check(status: int, where: str, stream=None):
    if status != 0:
        raise PuroError(status, where)
    if CHECK_EACH_CALL and stream is not None:
        st = _lib.puro_fp8_sync_status(stream)
        if st != 0:
            raise PuroError(st, f"{where} (status after the call)")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, rows_contig=True):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if rows_contig and t.dim() == 2 and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit column stride")


def _dense(t, name):
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape(t, shape, name):
    """The kernels write (and read) exactly the extents the C declaration gives; a tensor of
    any other shape would be overrun or misread, so it is refused here."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _matrix(t, name):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got {t.dim()}-D")
    return t.shape


# ------------------------------------------------------------------ C-ABI mirrors

def puro_fp8_quantize_1x128(X, Xq, S, stream=None):
    R, C = _matrix(X, "X")
    _shape(Xq, (R, C), "Xq"); _shape(S, (C // 128, R), "S")
    _need(X, torch.bfloat16, "X"); _need(Xq, torch.uint8, "Xq"); _need(S, torch.float32, "S")
    _dense(S, "S")
    with torch.cuda.device(X.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_1x128(_ptr(X), R, C, X.stride(0), _ptr(Xq), Xq.stride(0),
                                            _ptr(S), st), "puro_fp8_quantize_1x128", st)


def puro_fp8_quantize_1x128_transposed(X, XqT, ST, Xq=None, S=None, stream=None):
    T, C = _matrix(X, "X")
    _shape(XqT, (C, T), "XqT"); _shape(ST, (T // 128, C), "ST")
    _shape(Xq, (T, C), "Xq"); _shape(S, (C // 128, T), "S")
    _need(X, torch.bfloat16, "X"); _need(XqT, torch.uint8, "XqT"); _need(ST, torch.float32, "ST")
    _need(Xq, torch.uint8, "Xq"); _need(S, torch.float32, "S")
    for t, n in ((XqT, "XqT"), (ST, "ST"), (Xq, "Xq"), (S, "S")):
        _dense(t, n)
    with torch.cuda.device(X.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_1x128_transposed(_ptr(X), T, C, X.stride(0), _ptr(XqT), _ptr(ST),
                                                       _ptr(Xq), _ptr(S), st), "puro_fp8_quantize_1x128_transposed", st)


def puro_fp8_quantize_128x128(W, Wq, WqT, S, stream=None):
    R, C = _matrix(W, "W")
    _shape(Wq, (R, C), "Wq"); _shape(WqT, (C, R), "WqT"); _shape(S, ((R + 127) // 128, C // 128), "S")
    _need(W, torch.bfloat16, "W"); _need(Wq, torch.uint8, "Wq"); _need(WqT, torch.uint8, "WqT")
    _need(S, torch.float32, "S")
    for t, n in ((Wq, "Wq"), (WqT, "WqT"), (S, "S")):
        _dense(t, n)
    with torch.cuda.device(W.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_128x128(_ptr(W), R, C, W.stride(0), _ptr(Wq), _ptr(WqT), _ptr(S),
                                              st), "puro_fp8_quantize_128x128", st)


def puro_fp8_quantize_128x128_grouped(problems, stream=None):
    """problems: sequence of (W, Wq, WqT or None, S) tensor tuples, each checked as for
    puro_fp8_quantize_128x128; quantised in one launch per 64 weights (see the C declaration)."""
    if len(problems) < 1:
        raise ValueError("at least one weight")
    arr = (WeightProblem * len(problems))()
    dev = problems[0][0].device
    for i, (W, Wq, WqT, S) in enumerate(problems):
        R, C = _matrix(W, "W")
        _shape(Wq, (R, C), "Wq"); _shape(WqT, (C, R), "WqT"); _shape(S, ((R + 127) // 128, C // 128), "S")
        _need(W, torch.bfloat16, "W"); _need(Wq, torch.uint8, "Wq"); _need(WqT, torch.uint8, "WqT")
        _need(S, torch.float32, "S")
        for t, n in ((W, "W"), (Wq, "Wq"), (WqT, "WqT"), (S, "S")):
            if t is not None and t.device != dev:
                raise ValueError("all weights of a group must be on one device")
            if n != "W":
                _dense(t, n)
        arr[i] = WeightProblem(W.data_ptr(), R, C, W.stride(0), Wq.data_ptr(), _ptr(WqT), S.data_ptr())
    with torch.cuda.device(dev):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_128x128_grouped(ctypes.cast(arr, _p), len(problems), st),
               "puro_fp8_quantize_128x128_grouped", st)


def _gemm_shapes(Aq, As, Bq, Bs, C, bs_shape):
    M, K = _matrix(Aq, "Aq")
    N = _matrix(Bq, "Bq")[0]
    _shape(Bq, (N, K), "Bq"); _shape(C, (M, N), "C"); _shape(As, (K // 128, M), "As")
    _shape(Bs, bs_shape(N, K), "Bs")
    return M, N, K


def puro_fp8_gemm_blockwise(Aq, As, Bq, Bs, C, layout, workspace=None, stream=None):
    layout = int(LAYOUTS.get(layout, layout))
    if layout not in (PURO_FPROP, PURO_DGRAD, PURO_WGRAD):
        raise ValueError(f"unknown layout {layout}")
    bs_shape = {PURO_FPROP: lambda n, k: ((n + 127) // 128, k // 128),
                PURO_DGRAD: lambda n, k: (k // 128, (n + 127) // 128),
                PURO_WGRAD: lambda n, k: (k // 128, n)}[layout]
    M, N, K = _gemm_shapes(Aq, As, Bq, Bs, C, bs_shape)
    _need(Aq, torch.uint8, "Aq"); _need(Bq, torch.uint8, "Bq"); _need(C, torch.bfloat16, "C")
    _need(As, torch.float32, "As"); _need(Bs, torch.float32, "Bs")
    for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs"), (C, "C")):
        _dense(t, n)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(Aq.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_gemm_blockwise(_ptr(Aq), _ptr(As), _ptr(Bq), _ptr(Bs), _ptr(C), M, N, K,
                                            layout, _ptr(workspace), ws_bytes, st), "puro_fp8_gemm_blockwise", st)


def puro_fp8_quantize_1x128_pow2(X, Xq, S, stream=None):
    """As puro_fp8_quantize_1x128, power-of-two scales as bytes: S uint8 [C/128, R]."""
    R, C = _matrix(X, "X")
    _shape(Xq, (R, C), "Xq"); _shape(S, (C // 128, R), "S")
    _need(X, torch.bfloat16, "X"); _need(Xq, torch.uint8, "Xq"); _need(S, torch.uint8, "S")
    _dense(S, "S")
    with torch.cuda.device(X.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_1x128_pow2(_ptr(X), R, C, X.stride(0), _ptr(Xq), Xq.stride(0), _ptr(S), st),
               "puro_fp8_quantize_1x128_pow2", st)


def puro_fp8_quantize_1x128_transposed_pow2(X, XqT, ST, Xq=None, S=None, stream=None):
    """As puro_fp8_quantize_1x128_transposed, power-of-two scales as bytes."""
    T, C = _matrix(X, "X")
    _shape(XqT, (C, T), "XqT"); _shape(ST, (T // 128, C), "ST")
    _shape(Xq, (T, C), "Xq"); _shape(S, (C // 128, T), "S")
    _need(X, torch.bfloat16, "X"); _need(XqT, torch.uint8, "XqT"); _need(ST, torch.uint8, "ST")
    _need(Xq, torch.uint8, "Xq"); _need(S, torch.uint8, "S")
    for t, n in ((XqT, "XqT"), (ST, "ST"), (Xq, "Xq"), (S, "S")):
        _dense(t, n)
    with torch.cuda.device(X.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_1x128_transposed_pow2(_ptr(X), T, C, X.stride(0), _ptr(XqT), _ptr(ST),
                                                            _ptr(Xq), _ptr(S), st),
               "puro_fp8_quantize_1x128_transposed_pow2", st)


def puro_fp8_quantize_128x128_pow2(W, Wq, WqT, S, stream=None):
    """As puro_fp8_quantize_128x128, power-of-two scales as bytes: S uint8 [ceil(R/128), C/128]."""
    R, C = _matrix(W, "W")
    _shape(Wq, (R, C), "Wq"); _shape(WqT, (C, R), "WqT"); _shape(S, ((R + 127) // 128, C // 128), "S")
    _need(W, torch.bfloat16, "W"); _need(Wq, torch.uint8, "Wq"); _need(WqT, torch.uint8, "WqT")
    _need(S, torch.uint8, "S")
    for t, n in ((Wq, "Wq"), (WqT, "WqT"), (S, "S")):
        _dense(t, n)
    with torch.cuda.device(W.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_quantize_128x128_pow2(_ptr(W), R, C, W.stride(0), _ptr(Wq), _ptr(WqT), _ptr(S), st),
               "puro_fp8_quantize_128x128_pow2", st)


def puro_fp8_mx_gemm(Aq, As, Bq, Bs, C, layout, stream=None):
    """The block-scaled GEMM of power-of-two scale bytes (see the C declaration): As, Bs uint8
    laid out as the float scales of puro_fp8_gemm_blockwise for the same layout."""
    layout = int(LAYOUTS.get(layout, layout))
    if layout not in (PURO_FPROP, PURO_DGRAD, PURO_WGRAD):
        raise ValueError(f"unknown layout {layout}")
    bs_shape = {PURO_FPROP: lambda n, k: ((n + 127) // 128, k // 128),
                PURO_DGRAD: lambda n, k: (k // 128, (n + 127) // 128),
                PURO_WGRAD: lambda n, k: (k // 128, n)}[layout]
    M, N, K = _gemm_shapes(Aq, As, Bq, Bs, C, bs_shape)
    _need(Aq, torch.uint8, "Aq"); _need(Bq, torch.uint8, "Bq"); _need(C, torch.bfloat16, "C")
    _need(As, torch.uint8, "As"); _need(Bs, torch.uint8, "Bs")
    for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs"), (C, "C")):
        _dense(t, n)
    with torch.cuda.device(Aq.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_mx_gemm(_ptr(Aq), _ptr(As), _ptr(Bq), _ptr(Bs), _ptr(C), M, N, K, layout, st),
               "puro_fp8_mx_gemm", st)


def mx_gemm(Aq, As, Bq, Bs, layout, stream=None):
    """C [M, N] bf16 from the block-scaled GEMM (allocating helper)."""
    C = torch.empty((Aq.shape[0], Bq.shape[0]), dtype=torch.bfloat16, device=Aq.device)
    puro_fp8_mx_gemm(Aq, As, Bq, Bs, C, layout, stream)
    return C


def puro_nvfp4_quantize_1x16(X, Xq, F, amax, stream=None):
    """NVFP4 1x16 quantisation along the columns of X [R, C] bf16 (see the C declaration):
    Xq uint8 [R, C/2] packed codes (row stride may exceed C/2), F uint8 [ceil(C/256), R, 16]
    (factors by 256-element K block), amax float32 [1] (the tensor's max |x|, written by the call)."""
    _need(X, torch.bfloat16, "X"); _need(Xq, torch.uint8, "Xq"); _need(F, torch.uint8, "F")
    _need(amax, torch.float32, "amax")
    R, C = X.shape
    if tuple(Xq.shape) != (R, C // 2) or tuple(F.shape) != ((C + 255) // 256, R, 16) or amax.numel() != 1:
        raise ValueError("Xq must be [R, C/2], F [ceil(C/256), R, 16] and amax one float")
    _dense(F, "F")
    with torch.cuda.device(X.device):
        st = _stream(stream)
        _check(_lib.puro_nvfp4_quantize_1x16(_ptr(X), R, C, X.stride(0), _ptr(Xq), Xq.stride(0), _ptr(F),
                                             _ptr(amax), st), "puro_nvfp4_quantize_1x16", st)


def puro_nvfp4_quantize_1x16_transposed(X, XqT, FT, amax, stream=None):
    """NVFP4 1x16 quantisation along the rows (tokens) of X [R, C] bf16, written transposed:
    XqT uint8 [C, R/2] packed codes, FT uint8 [ceil(R/256), C, 16], amax float32 [1]."""
    _need(X, torch.bfloat16, "X"); _need(XqT, torch.uint8, "XqT"); _need(FT, torch.uint8, "FT")
    _need(amax, torch.float32, "amax")
    R, C = X.shape
    if tuple(XqT.shape) != (C, R // 2) or tuple(FT.shape) != ((R + 255) // 256, C, 16) or amax.numel() != 1:
        raise ValueError("XqT must be [C, R/2], FT [ceil(R/256), C, 16] and amax one float")
    _dense(FT, "FT")
    with torch.cuda.device(X.device):
        st = _stream(stream)
        _check(_lib.puro_nvfp4_quantize_1x16_transposed(_ptr(X), R, C, X.stride(0), _ptr(XqT), XqT.stride(0),
                                                        _ptr(FT), _ptr(amax), st),
               "puro_nvfp4_quantize_1x16_transposed", st)


def puro_nvfp4_quantize_1x16_dual(X, Xq, F, XqT, FT, amax, stream=None):
    """Both NVFP4 layouts of X [R, C] bf16 from one read (see the C declaration): Xq [R, C/2] and
    F [ceil(C/256), R, 16] along the columns, XqT [C, R/2] and FT [ceil(R/256), C, 16] along the
    rows, amax float32 [1]."""
    _need(X, torch.bfloat16, "X"); _need(Xq, torch.uint8, "Xq"); _need(F, torch.uint8, "F")
    _need(XqT, torch.uint8, "XqT"); _need(FT, torch.uint8, "FT"); _need(amax, torch.float32, "amax")
    R, C = X.shape
    if (tuple(Xq.shape) != (R, C // 2) or tuple(F.shape) != ((C + 255) // 256, R, 16)
            or tuple(XqT.shape) != (C, R // 2) or tuple(FT.shape) != ((R + 255) // 256, C, 16) or amax.numel() != 1):
        raise ValueError("Xq must be [R, C/2], F [ceil(C/256), R, 16], XqT [C, R/2], FT [ceil(R/256), C, 16] "
                         "and amax one float")
    _dense(F, "F"); _dense(FT, "FT")
    with torch.cuda.device(X.device):
        st = _stream(stream)
        _check(_lib.puro_nvfp4_quantize_1x16_dual(_ptr(X), R, C, X.stride(0), _ptr(Xq), Xq.stride(0), _ptr(F),
                                                  _ptr(XqT), XqT.stride(0), _ptr(FT), _ptr(amax), st),
               "puro_nvfp4_quantize_1x16_dual", st)


def puro_nvfp4_gemm(Aq, As, a_amax, Bq, Bs, b_amax, C, stream=None):
    """NVFP4 GEMM C [M, N] bf16 = A . B^T of two operands quantised along K (see the C
    declaration): Aq [M, K/2], Bq [N, K/2] packed codes, As [ceil(K/256), M, 16], Bs
    [ceil(K/256), N, 16] factors, uint8, dense; the amax arguments float32 [1] on the device."""
    for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs")):
        _need(t, torch.uint8, n)
        _dense(t, n)
    _need(C, torch.bfloat16, "C"); _dense(C, "C")
    _need(a_amax, torch.float32, "a_amax"); _need(b_amax, torch.float32, "b_amax")
    M, K = Aq.shape[0], 2 * Aq.shape[1]
    N = Bq.shape[0]
    kb = (K + 255) // 256
    if (tuple(As.shape) != (kb, M, 16) or tuple(Bq.shape) != (N, K // 2) or tuple(Bs.shape) != (kb, N, 16)
            or tuple(C.shape) != (M, N)):
        raise ValueError("operand shapes do not match: Aq [M, K/2], As [ceil(K/256), M, 16], Bq [N, K/2], "
                         "Bs [ceil(K/256), N, 16], C [M, N]")
    with torch.cuda.device(Aq.device):
        st = _stream(stream)
        _check(_lib.puro_nvfp4_gemm(_ptr(Aq), _ptr(As), _ptr(a_amax), _ptr(Bq), _ptr(Bs), _ptr(b_amax), _ptr(C),
                                    M, N, K, st), "puro_nvfp4_gemm", st)


def nvfp4_quantize(X, transposed=False, stream=None):
    """(packed codes, factors, amax) of X along its columns, or along its rows written
    transposed (allocating helper)."""
    R, C = X.shape
    amax = torch.empty(1, dtype=torch.float32, device=X.device)
    if transposed:
        q = torch.empty((C, R // 2), dtype=torch.uint8, device=X.device)
        f = torch.zeros(((R + 255) // 256, C, 16), dtype=torch.uint8, device=X.device)
        puro_nvfp4_quantize_1x16_transposed(X, q, f, amax, stream)
    else:
        q = torch.empty((R, C // 2), dtype=torch.uint8, device=X.device)
        f = torch.zeros(((C + 255) // 256, R, 16), dtype=torch.uint8, device=X.device)
        puro_nvfp4_quantize_1x16(X, q, f, amax, stream)
    return q, f, amax


def nvfp4_quantize_dual(X, stream=None):
    """((Xq, F), (XqT, FT), amax): both NVFP4 layouts of X from one call (allocating helper)."""
    R, C = X.shape
    amax = torch.empty(1, dtype=torch.float32, device=X.device)
    q = torch.empty((R, C // 2), dtype=torch.uint8, device=X.device)
    f = torch.zeros(((C + 255) // 256, R, 16), dtype=torch.uint8, device=X.device)
    qt = torch.empty((C, R // 2), dtype=torch.uint8, device=X.device)
    ft = torch.zeros(((R + 255) // 256, C, 16), dtype=torch.uint8, device=X.device)
    puro_nvfp4_quantize_1x16_dual(X, q, f, qt, ft, amax, stream)
    return (q, f), (qt, ft), amax


def nvfp4_gemm(Aq, As, a_amax, Bq, Bs, b_amax, stream=None):
    """C [M, N] bf16 from the NVFP4 GEMM (allocating helper)."""
    C = torch.empty((Aq.shape[0], Bq.shape[0]), dtype=torch.bfloat16, device=Aq.device)
    puro_nvfp4_gemm(Aq, As, a_amax, Bq, Bs, b_amax, C, stream)
    return C


def puro_fp8_gemm_blockwise_grouped(problems, layout, stream=None):
    """problems: sequence of (Aq, As, Bq, Bs, C) tensor tuples, each checked as for
    puro_fp8_gemm_blockwise; all run in one launch (see the C declaration)."""
    layout = int(LAYOUTS.get(layout, layout))
    if layout not in (PURO_FPROP, PURO_DGRAD, PURO_WGRAD):
        raise ValueError(f"unknown layout {layout}")
    if not 1 <= len(problems) <= GROUP_MAX:
        raise ValueError(f"1 to {GROUP_MAX} problems per grouped launch, got {len(problems)}")
    bs_shape = {PURO_FPROP: lambda n, k: ((n + 127) // 128, k // 128),
                PURO_DGRAD: lambda n, k: (k // 128, (n + 127) // 128),
                PURO_WGRAD: lambda n, k: (k // 128, n)}[layout]
    arr = (GemmProblem * len(problems))()
    dev = problems[0][0].device
    for i, (Aq, As, Bq, Bs, C) in enumerate(problems):
        M, N, K = _gemm_shapes(Aq, As, Bq, Bs, C, bs_shape)
        _need(Aq, torch.uint8, "Aq"); _need(Bq, torch.uint8, "Bq"); _need(C, torch.bfloat16, "C")
        _need(As, torch.float32, "As"); _need(Bs, torch.float32, "Bs")
        for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs"), (C, "C")):
            _dense(t, n)
            if t.device != dev:
                raise ValueError("all problems of a group must be on one device")
        arr[i] = GemmProblem(Aq.data_ptr(), As.data_ptr(), Bq.data_ptr(), Bs.data_ptr(), C.data_ptr(), M, N, K)
    with torch.cuda.device(dev):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_gemm_blockwise_grouped(ctypes.cast(arr, _p), len(problems), layout, st),
               "puro_fp8_gemm_blockwise_grouped", st)


def puro_fp8_gemm_blockwise_quant(Aq, As, Bq, Bs, C, Cq, Cs, layout, stream=None):
    """fprop / dgrad into C (bf16 [M, N]) plus the 1x128 quantisation of C along N: Cq
    (uint8 [M, N]) and Cs (float32 [N/128, M]); see the C declaration."""
    layout = int(LAYOUTS.get(layout, layout))
    if layout not in (PURO_FPROP, PURO_DGRAD):
        raise ValueError(f"layout must be fprop or dgrad, got {layout}")
    bs_shape = {PURO_FPROP: lambda n, k: ((n + 127) // 128, k // 128),
                PURO_DGRAD: lambda n, k: (k // 128, (n + 127) // 128)}[layout]
    M, N, K = _gemm_shapes(Aq, As, Bq, Bs, C, bs_shape)
    _shape(Cq, (M, N), "Cq"); _shape(Cs, (N // 128, M), "Cs")
    _need(Aq, torch.uint8, "Aq"); _need(Bq, torch.uint8, "Bq"); _need(C, torch.bfloat16, "C")
    _need(As, torch.float32, "As"); _need(Bs, torch.float32, "Bs")
    _need(Cq, torch.uint8, "Cq"); _need(Cs, torch.float32, "Cs")
    for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs"), (C, "C"), (Cq, "Cq"), (Cs, "Cs")):
        _dense(t, n)
    with torch.cuda.device(Aq.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_gemm_blockwise_quant(_ptr(Aq), _ptr(As), _ptr(Bq), _ptr(Bs), _ptr(C), _ptr(Cq),
                                                  _ptr(Cs), M, N, K, layout, st),
               "puro_fp8_gemm_blockwise_quant", st)


def gemm_quant(Aq, As, Bq, Bs, layout, stream=None):
    """(C bf16 [M, N], Cq uint8 [M, N], Cs float32 [N/128, M]) = the GEMM and its output's
    1x128 quantisation from one launch (see puro_fp8_gemm_blockwise_quant)."""
    M, N = Aq.shape[0], Bq.shape[0]
    C = torch.empty((M, N), dtype=torch.bfloat16, device=Aq.device)
    Cq = torch.empty((M, N), dtype=torch.uint8, device=Aq.device)
    Cs = torch.empty((N // 128, M), dtype=torch.float32, device=Aq.device)
    puro_fp8_gemm_blockwise_quant(Aq, As, Bq, Bs, C, Cq, Cs, layout, stream)
    return C, Cq, Cs


def puro_fp8_gemm_wgrad_acc_f32(Aq, As, Bq, Bs, C, stream=None):
    """C (float32 [M, N]) += the wgrad product of the operands (see the C declaration)."""
    M, N, K = _gemm_shapes(Aq, As, Bq, Bs, C, lambda n, k: (k // 128, n))
    _need(Aq, torch.uint8, "Aq"); _need(Bq, torch.uint8, "Bq"); _need(C, torch.float32, "C")
    _need(As, torch.float32, "As"); _need(Bs, torch.float32, "Bs")
    for t, n in ((Aq, "Aq"), (As, "As"), (Bq, "Bq"), (Bs, "Bs"), (C, "C")):
        _dense(t, n)
    with torch.cuda.device(Aq.device):
        st = _stream(stream)  # the current stream of the tensors' device
        _check(_lib.puro_fp8_gemm_wgrad_acc_f32(_ptr(Aq), _ptr(As), _ptr(Bq), _ptr(Bs), _ptr(C), M, N, K,
                                                st), "puro_fp8_gemm_wgrad_acc_f32", st)


def puro_fp8_sync_status(stream=None):
    _check(_lib.puro_fp8_sync_status(_stream(stream)), "puro_fp8_sync_status")


# ------------------------------------------------------------------ allocating helpers

def quantize_1x128(X, stream=None):
    """X [R, C] bf16 -> (Xq uint8 [R, C], S float32 [C/128, R])."""
    R, C = X.shape
    Xq = torch.empty((R, C), dtype=torch.uint8, device=X.device)
    S = torch.empty((C // 128, R), dtype=torch.float32, device=X.device)
    puro_fp8_quantize_1x128(X, Xq, S, stream)
    return Xq, S


def quantize_1x128_transposed(X, dual=False, stream=None):
    """X [T, C] bf16 -> (XqT [C, T], ST [T/128, C]) and, if dual, also (Xq, S) row-wise."""
    T, C = X.shape
    XqT = torch.empty((C, T), dtype=torch.uint8, device=X.device)
    ST = torch.empty((T // 128, C), dtype=torch.float32, device=X.device)
    Xq = S = None
    if dual:
        Xq = torch.empty((T, C), dtype=torch.uint8, device=X.device)
        S = torch.empty((C // 128, T), dtype=torch.float32, device=X.device)
    puro_fp8_quantize_1x128_transposed(X, XqT, ST, Xq, S, stream)
    return (XqT, ST, Xq, S) if dual else (XqT, ST)


def quantize_128x128(W, transposed=True, stream=None):
    """W [R, C] bf16 -> (Wq [R, C], WqT [C, R] or None, S [ceil(R/128), C/128])."""
    R, C = W.shape
    Wq = torch.empty((R, C), dtype=torch.uint8, device=W.device)
    WqT = torch.empty((C, R), dtype=torch.uint8, device=W.device) if transposed else None
    S = torch.empty(((R + 127) // 128, C // 128), dtype=torch.float32, device=W.device)
    puro_fp8_quantize_128x128(W, Wq, WqT, S, stream)
    return Wq, WqT, S


def quantize_1x128_pow2(X, stream=None):
    """X [R, C] bf16 -> (Xq [R, C], UE8M0 bytes [C/128, R])."""
    R, C = X.shape
    Xq = torch.empty((R, C), dtype=torch.uint8, device=X.device)
    S = torch.empty((C // 128, R), dtype=torch.uint8, device=X.device)
    puro_fp8_quantize_1x128_pow2(X, Xq, S, stream)
    return Xq, S


def quantize_1x128_transposed_pow2(X, dual=False, stream=None):
    """X [T, C] bf16 -> (XqT [C, T], bytes [T/128, C]) and, if dual, also (Xq, bytes) row-wise."""
    T, C = X.shape
    XqT = torch.empty((C, T), dtype=torch.uint8, device=X.device)
    ST = torch.empty((T // 128, C), dtype=torch.uint8, device=X.device)
    Xq = S = None
    if dual:
        Xq = torch.empty((T, C), dtype=torch.uint8, device=X.device)
        S = torch.empty((C // 128, T), dtype=torch.uint8, device=X.device)
    puro_fp8_quantize_1x128_transposed_pow2(X, XqT, ST, Xq, S, stream)
    return (XqT, ST, Xq, S) if dual else (XqT, ST)


def quantize_128x128_pow2(W, transposed=True, stream=None):
    """W [R, C] bf16 -> (Wq, WqT or None, bytes [ceil(R/128), C/128])."""
    R, C = W.shape
    Wq = torch.empty((R, C), dtype=torch.uint8, device=W.device)
    WqT = torch.empty((C, R), dtype=torch.uint8, device=W.device) if transposed else None
    S = torch.empty(((R + 127) // 128, C // 128), dtype=torch.uint8, device=W.device)
    puro_fp8_quantize_128x128_pow2(W, Wq, WqT, S, stream)
    return Wq, WqT, S


def gemm(Aq, As, Bq, Bs, layout, out=None, stream=None):
    """C [M, N] bf16 = blockwise GEMM of the given operands (see puro_fp8_gemm_blockwise)."""
    M, N = Aq.shape[0], Bq.shape[0]
    C = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=Aq.device)
    puro_fp8_gemm_blockwise(Aq, As, Bq, Bs, C, layout, None, stream)
    return C
