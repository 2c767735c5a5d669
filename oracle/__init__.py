"""CPU oracle for the blockwise-FP8 (E4M3) linear-layer path. TEST INFRASTRUCTURE ONLY.

Only the test suite (``tests/``), ``__graft_entry__.smoke()`` and the ``cpu_baseline``
leg of ``bench.py`` (plus its ``--impl reference`` arm) may import, call or run anything
in this package. The library itself (``fp8_blockwise_scaled_e4m3_b200``) never does:
its every step runs in the CUDA kernels, and it raises if they are missing.

What it computes, and where that comes from
-------------------------------------------
The method is the one stated in "Paper walkthrough: Puro-2B — pretraining a 2B model
from scratch for $6.9K on consumer GPUs", section "Lever 2: use blockwise FP8 from step
zero": the linear-layer GEMMs run in FP8, with scales taken per local group,
activations and their gradients in groups of 128 along the reduction dimension,
weights in 128x128 blocks, and FP8 used as a compute format only (inputs and outputs
stay in BF16). The page does not spell out the number format or the scale formula;
the readings this oracle takes are:

* E4M3 (OCP 8-bit floating point, "E4M3" encoding: bias 7, largest finite 448, no
  infinities, 0x7F/0xFF are NaN) for every FP8 tensor, gradients included;
* scale ``s = amax / 448`` as a correctly rounded FP32 division, no power-of-two
  rounding and no margin, computed "just in time" from the tensor being quantised
  (no amax history: the page says FP8 is used from random initialisation);
* code ``q = E4M3(x / s)``: FP32 division (correctly rounded), then round to nearest,
  ties to even mantissa, saturating to +-448; an all-zero block has ``s = 0`` and
  sign-preserving zero codes;
* GEMM: dequantise both operands exactly in float64 and contract with an FP64 matmul.

Because a quantised code is an integer decided by floating point, the oracle takes
that decision in FP32, the precision the method fixes; only the contraction is FP64.

Modules
-------
``e4m3``        codec (decode table, nearest-value encoder), pinned by brute force,
                closed forms and PyTorch's own float8_e4m3fn conversion.
``quant``       the 1x128, transposed 1x128 and 128x128 quantisers, pinned by
                invariants, hand-worked fixtures and special cases.
``mx``          the power-of-two (UE8M0) scale mode of the same groups (scale rounded up
                to a power of two, stored as an exponent byte), pinned by its exponent
                rule in exact rationals, a hand-worked group and nearest-value checks.
``nvfp4``       the NVFP4 mode (E2M1 codes, a UE4M3 factor per 16 elements along the
                reduction dimension, an FP32 tensor scale amax / 2688), pinned by the E2M1
                table, a brute-force encoder, a hand-worked row of groups, invariants of the
                two-level scale and an exact rational contraction.
``gemm``        the FP64 reference contraction for the fprop / dgrad / wgrad operand
                layouts, pinned by exact rational brute force and an exact-integer case.
``accounting``  parameter and FLOP accounting (C = 6ND), pinned by the numbers the
                pages print.

No function here is "parity unpinned".
"""

from . import e4m3, quant, gemm, accounting, nvfp4  # noqa: F401
