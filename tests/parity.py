"""Shared helpers of the GPU parity tests: oracle calls on BF16 inputs and the GEMM
tolerance check. The oracle only ever receives BF16 inputs (or hand-built codes and
scales); it never receives anything the CUDA path produced.

GEMM tolerance (fixed by the method's target accuracy): against the FP64 oracle result
C_ref, unrounded,
    ||C_gpu - C_ref||_F / ||C_ref||_F <= 2e-3
    |C_gpu - C_ref|[m, n] <= 1e-2 * ||A_deq[m, :]||_2 * ||B_deq[n, :]||_2
BF16 rounding of the output alone contributes about 1.5e-3 relative Frobenius error
(half an ulp of an 8-bit significand, uniformly spread), so the first bound leaves
room only for FP32-exact accumulation; the second is loose per element but catches
any single wrong output.
"""

import numpy as np
import torch

from oracle import gemm as ogemm
from oracle import mx as omx
from oracle import quant as oquant
from fp8_blockwise_scaled_e4m3_b200 import workloads as wl

REL_FRO = 2e-3
ELEM = 1e-2


def host_bits(t):
    return wl.bf16_bits(t)


def as_np(t):
    return t.detach().cpu().numpy()


def bf16_to_f64(t):
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def check_gemm(c_gpu, c_ref, a_norm, b_norm, what="", extra_abs=0.0):
    """c_gpu, c_ref [m, n] float64 arrays; a_norm [m], b_norm [n]. extra_abs: an additional
    elementwise allowance (the one FP32 rounding of an accumulation into an FP32 buffer)."""
    diff = c_gpu - c_ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(c_ref), 1e-300)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    bound = ELEM * np.outer(a_norm, b_norm) + extra_abs
    worst = np.max(np.abs(diff) - bound)
    assert worst <= 0, f"{what}: elementwise bound exceeded by {worst:.3e}"
    return rel


def oracle_rows_1x128(x_bits_rows):
    """Row-wise 1x128 codes and scales of some rows (rows are independent)."""
    return oquant.quant_1x128(x_bits_rows)


class _Pow2Quant:
    """The power-of-two scale quantisers of oracle.mx, with their bytes turned into the float
    scales 2^(byte - 127) so that oracle.gemm applies unchanged."""

    @staticmethod
    def quant_1x128(x):
        q, b = omx.quant_1x128_pow2(x)
        return q, omx.scales_from_ue8m0(b)

    @staticmethod
    def quant_1x128_transposed(x):
        q, b = omx.quant_1x128_transposed_pow2(x)
        return q, omx.scales_from_ue8m0(b)

    @staticmethod
    def quant_128x128(w):
        q, qt, b = omx.quant_128x128_pow2(w)
        return q, qt, omx.scales_from_ue8m0(b)


QUANTISERS = {"fp32": oquant, "pow2": _Pow2Quant}


def oracle_gemm_sampled(layout, a_bf16, b_bf16, rows, nblocks, scales="fp32"):
    """Oracle C[rows, n] for n in the 128-wide column blocks `nblocks`, from BF16 inputs,
    quantised with FP32 scales (oracle.quant) or power-of-two scales (oracle.mx).

    fprop: a = X [T, K_in],  b = W [N_out, K_in]   -> C = X W^T      [T, N_out]
    dgrad: a = dY [T, N_out], b = W [N_out, K_in]  -> C = dY W       [T, K_in]
    wgrad: a = dY [T, N_out], b = X [T, K_in]      -> C = dY^T X     [N_out, K_in]
    Returns (c_ref [len(rows), len(cols)], cols, a_norm, b_norm).
    """
    rows = np.asarray(rows)
    oquant = QUANTISERS[scales]
    if layout == "fprop":
        a_rows = host_bits(a_bf16[torch.as_tensor(rows, device=a_bf16.device)])
        aq, a_s = oquant.quant_1x128(a_rows)
        n_total = b_bf16.shape[0]
        cols = np.concatenate([np.arange(nb * 128, min(n_total, nb * 128 + 128)) for nb in nblocks])
        bq_parts, bs_parts = [], []
        for nb in nblocks:
            w_blk = host_bits(b_bf16[nb * 128:nb * 128 + 128])
            q, _, s = oquant.quant_128x128(w_blk)
            bq_parts.append(q)
            bs_parts.append(s)
        bq, bs = np.concatenate(bq_parts), np.concatenate(bs_parts)
        c = ogemm.gemm_ref(aq, a_s, bq, bs, "fprop")
        an, bn = ogemm.row_col_norms(aq, a_s, bq, bs, "fprop")
        return c, cols, an, bn
    if layout == "dgrad":
        a_rows = host_bits(a_bf16[torch.as_tensor(rows, device=a_bf16.device)])
        aq, a_s = oquant.quant_1x128(a_rows)
        cols = np.concatenate([np.arange(nb * 128, nb * 128 + 128) for nb in nblocks])
        bq_parts, bs_parts = [], []
        for nb in nblocks:
            w_cols = host_bits(b_bf16[:, nb * 128:nb * 128 + 128].contiguous())  # [N_out, 128]
            q, qt, s = oquant.quant_128x128(w_cols)  # s [N_out/128, 1]
            bq_parts.append(qt)  # [128, N_out]
            bs_parts.append(s)
        bq = np.concatenate(bq_parts)
        bs = np.concatenate(bs_parts, axis=1)  # [K/128, len(nblocks)]
        c = ogemm.gemm_ref(aq, a_s, bq, bs, "dgrad")
        an, bn = ogemm.row_col_norms(aq, a_s, bq, bs, "dgrad")
        return c, cols, an, bn
    if layout == "wgrad":
        rows_t = torch.as_tensor(rows, device=a_bf16.device)
        a_cols = host_bits(a_bf16[:, rows_t].contiguous())  # [T, len(rows)]
        aq, a_s = oquant.quant_1x128_transposed(a_cols)
        cols = np.concatenate([np.arange(nb * 128, nb * 128 + 128) for nb in nblocks])
        b_cols = host_bits(b_bf16[:, torch.as_tensor(cols, device=b_bf16.device)].contiguous())
        bq, bs = oquant.quant_1x128_transposed(b_cols)
        c = ogemm.gemm_ref(aq, a_s, bq, bs, "wgrad")
        an, bn = ogemm.row_col_norms(aq, a_s, bq, bs, "wgrad")
        return c, cols, an, bn
    raise ValueError(layout)
