"""FP64 reference contraction of the oracle (test infrastructure only).

"Paper walkthrough: Puro-2B ...", section "Lever 2: use blockwise FP8 from step zero":
only the linear-layer GEMMs run in FP8, with the blockwise scales described there.
Every layout computes

    C[m, n] = sum_k A[m, k] * B[n, k]

over dequantised operands, A_deq[m, k] = E4M3(Aq[m, k]) * sA(m, k) and likewise B,
which equals the blockwise definition sum_kb sA*sB * sum_{k in kb} Aq*Bq because each
scale is constant over its 128-wide group. Dequantisation is exact in float64; the
contraction is a float64 matmul (a library primitive, used as one step).

Operand layouts (K is the reduction dim, always a multiple of 128):
  A   : Aq [M, K] codes, As [K/128, M]                (1x128 along K)
  B, "fprop": Bq = Wq [N, K], Bs [ceil(N/128), K/128]  (128x128 weight blocks)
  B, "dgrad": Bq = WqT [N, K], Bs [K/128, ceil(N/128)] (the weight's own S: its rows
              are the output features, which dgrad contracts over)
  B, "wgrad": Bq [N, K], Bs [K/128, N]                 (1x128 along the tokens)
The result is returned in float64, not rounded to BF16.
"""

import numpy as np

from . import e4m3

BLOCK = 128
LAYOUTS = ("fprop", "dgrad", "wgrad")


def dequant_1x128(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Codes [R, K] with scales [K/128, R] -> float64 [R, K]."""
    r, k = q.shape
    assert s.shape == (k // BLOCK, r)
    scale = np.repeat(np.asarray(s, dtype=np.float64).T, BLOCK, axis=1)  # [R, K]
    return e4m3.decode(q) * scale


def dequant_weight_blocks(q: np.ndarray, s_rows_by_cols: np.ndarray) -> np.ndarray:
    """Codes [R, K] with one scale per 128x128 block, s[R/128 (ceil), K/128]."""
    r, k = q.shape
    rb = -(-r // BLOCK)
    assert s_rows_by_cols.shape == (rb, k // BLOCK)
    scale = np.repeat(np.repeat(np.asarray(s_rows_by_cols, dtype=np.float64), BLOCK, axis=0)[:r],
                      BLOCK, axis=1)
    return e4m3.decode(q) * scale


def dequant_b(bq: np.ndarray, bs: np.ndarray, layout: str) -> np.ndarray:
    """Dequantise the B operand [N, K] for one of the three layouts."""
    if layout == "fprop":
        return dequant_weight_blocks(bq, bs)
    if layout == "dgrad":
        # Bs is indexed [k-block, n-block]: the transpose of fprop's indexing.
        return dequant_weight_blocks(bq, np.asarray(bs).T)
    if layout == "wgrad":
        return dequant_1x128(bq, bs)
    raise ValueError(f"unknown layout {layout!r}")


def gemm_ref(aq, a_s, bq, b_s, layout: str) -> np.ndarray:
    """C = A_deq @ B_deq^T in float64, shape [M, N]."""
    a = dequant_1x128(np.asarray(aq), np.asarray(a_s))
    b = dequant_b(np.asarray(bq), np.asarray(b_s), layout)
    assert a.shape[1] == b.shape[1]
    return a @ b.T


def gemm_ref_rows(aq, a_s, bq, b_s, layout: str, rows) -> np.ndarray:
    """The rows ``rows`` of gemm_ref, without forming the other rows of A_deq."""
    rows = np.asarray(rows)
    a_rows = e4m3.decode(np.asarray(aq)[rows]) * np.repeat(
        np.asarray(a_s, dtype=np.float64)[:, rows].T, BLOCK, axis=1)
    b = dequant_b(np.asarray(bq), np.asarray(b_s), layout)
    return a_rows @ b.T


def wgrad_accumulate_ref(c_in, aq, a_s, bq, b_s) -> np.ndarray:
    """FP32 main-gradient accumulation of a weight gradient: C_in + dW, with dW the wgrad
    contraction above (the pages keep master weights in BF16/FP32; accumulating each
    micro-step's dW into an FP32 buffer is the plain reading of that). float64 result; the
    GPU's FP32 add rounds it once."""
    return np.asarray(c_in, dtype=np.float64) + gemm_ref(aq, a_s, bq, b_s, "wgrad")


def row_col_norms(aq, a_s, bq, b_s, layout: str, rows=None):
    """||A_deq[m, :]||_2 and ||B_deq[n, :]||_2, for the elementwise error bound."""
    if rows is None:
        a = dequant_1x128(np.asarray(aq), np.asarray(a_s))
    else:
        rows = np.asarray(rows)
        a = e4m3.decode(np.asarray(aq)[rows]) * np.repeat(
            np.asarray(a_s, dtype=np.float64)[:, rows].T, BLOCK, axis=1)
    b = dequant_b(np.asarray(bq), np.asarray(b_s), layout)
    return np.linalg.norm(a, axis=1), np.linalg.norm(b, axis=1)
