/*
 * puro_fp8.h -- C ABI of the blockwise-FP8 (E4M3) linear-layer library for B200 (sm_100a).
 *
 * The method ("Paper walkthrough: Puro-2B -- pretraining a 2B model from scratch for
 * $6.9K on consumer GPUs", section "Lever 2: use blockwise FP8 from step zero"): only
 * the linear-layer GEMMs run in FP8, tensors are converted to FP8 only for the GEMM that
 * consumes them, and scales are local -- activations and their gradients get one scale per 128
 * consecutive elements along the reduction dimension, weights one scale per 128x128
 * block. Readings this library takes where the page is silent: the FP8 format is E4M3
 * (bias 7, max 448, no infinities, 0x7F/0xFF NaN); a block's scale is s = amax / 448,
 * a correctly rounded FP32 division, computed from the tensor being quantised (no
 * amax history); a code is E4M3(x / s) with a correctly rounded FP32 division, then
 * round-to-nearest-even saturating to +-448; an all-zero block has s = 0 and signed
 * zero codes. GEMM partial sums are FP32 per 128-wide K block, promoted with the two
 * scales in FP32, output BF16 (round to nearest even), or, for the accumulating weight
 * gradient, added into an FP32 buffer.
 *
 * Conventions for every entry point:
 *  - Every pointer is a DEVICE pointer to memory the caller owns and allocated; the
 *    library allocates nothing and keeps no reference after the call is enqueued.
 *  - BF16 data is passed as uint16_t bit patterns; FP8 codes as uint8_t; scales float.
 *  - Matrices are row-major. Leading dimensions are in elements.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default stream).
 *  - Arguments are checked on the host before anything is launched; a failed check
 *    returns a negative puro_status and enqueues nothing.
 *  - Inputs must be finite (no NaN / Inf); this is not checked.
 *  - Calls keep no state between them and may be made from several host threads. The
 *    one piece of global state is a status word per device: any kernel of this library,
 *    on any stream, sets it when one of its bounded device-side waits gives up (the
 *    kernel then stops early and leaves its outputs partly written). A call's outputs
 *    are therefore valid only once a puro_fp8_sync_status() issued after it has
 *    returned PURO_OK. That function joins the whole device, so it sees timeouts from
 *    every stream; if several threads call it, the first one after the timeout gets the
 *    report, because reading the word clears it.
 */
#ifndef PURO_FP8_H
#define PURO_FP8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PURO_API __attribute__((visibility("default")))
#else
#define PURO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (ABI-identical to cudaStream_t / CUstream). */
typedef struct CUstream_st *puro_stream_t;

typedef enum {
  PURO_OK = 0,
  PURO_ERR_NULL = -1,      /* a required pointer is NULL                               */
  PURO_ERR_SHAPE = -2,     /* a size is <= 0, a reduction dim is not a multiple of 128,
                              a leading dimension is smaller than the row length, or
                              the sizes are too large for 32-bit tile indices           */
  PURO_ERR_ALIGN = -3,     /* a pointer or leading dimension breaks the 16-byte rule    */
  PURO_ERR_LAYOUT = -4,    /* unknown GEMM layout                                       */
  PURO_ERR_LAUNCH = -5,    /* the CUDA launch failed (cudaGetLastError after launch)    */
  PURO_ERR_TIMEOUT = -6,   /* a bounded device-side wait gave up (see sync_status)      */
  PURO_ERR_WORKSPACE = -7, /* reserved; not returned by this version                     */
  PURO_ERR_CUDA = -8,      /* another CUDA runtime / driver call failed                 */
  PURO_ERR_DEVICE = -9     /* the current device is not sm_100 (B200-class)             */
} puro_status;

/* Operand layouts of puro_fp8_gemm_blockwise (see there). */
enum { PURO_FPROP = 0, PURO_DGRAD = 1, PURO_WGRAD = 2 };

/*
 * 1x128 quantisation along the columns (the reduction dimension) of X [R, C].
 * Source: "Lever 2: use blockwise FP8 from step zero" -- activations and their
 * gradients in groups of 128 along the reduction dimension. Used for the forward
 * activation (fprop A operand) and for dY (dgrad A operand).
 *
 *   X   [R, C] BF16, row stride ldx (>= C)         input
 *   Xq  [R, C] E4M3 codes, row stride ldq (>= C)   output
 *   S   [C/128, R] float, dense                   output; S[j*R + r] is the scale of
 *                                                  X[r, 128j .. 128j+127]
 * Requires R >= 1, C >= 128, C % 128 == 0; X, Xq 16-byte aligned, ldx % 8 == 0,
 * ldq % 16 == 0; S 4-byte aligned.
 */
PURO_API int puro_fp8_quantize_1x128(const uint16_t *X, int64_t R, int64_t C, int64_t ldx,
                            uint8_t *Xq, int64_t ldq, float *S, puro_stream_t stream);

/*
 * 1x128 quantisation along the rows (tokens) of X [T, C], written transposed.
 * Source: "Lever 2: use blockwise FP8 from step zero" -- gradients (and activations)
 * in groups of 128 along the reduction dimension; for the weight-gradient GEMM
 * dW = dY^T X that dimension is the token dimension, so both of its operands are
 * re-quantised from BF16 in 128-token groups.
 *
 *   X    [T, C] BF16, row stride ldx (>= C)   input (tokens are rows)
 *   XqT  [C, T] E4M3 codes, dense              output; XqT[c, t] is the code of X[t, c]
 *   ST   [T/128, C] float, dense               output; ST[b*C + c] is the scale of
 *                                              X[128b .. 128b+127, c]
 *   Xq, S  optional (both NULL or both set): the row-wise 1x128 quantisation of the
 *          same X (exactly what puro_fp8_quantize_1x128 writes with ldq = C), made
 *          from the same read of X. Requires C % 128 == 0 when set.
 * Requires T >= 128, T % 128 == 0, C >= 8, C % 8 == 0; X 16-byte aligned, ldx % 8 == 0;
 * XqT, Xq 16-byte aligned.
 */
PURO_API int puro_fp8_quantize_1x128_transposed(const uint16_t *X, int64_t T, int64_t C, int64_t ldx,
                                       uint8_t *XqT, float *ST, uint8_t *Xq, float *S,
                                       puro_stream_t stream);

/*
 * 128x128 block quantisation of a weight W [R, C] (R = output features, C = input
 * features, the forward reduction dimension).
 * Source: "Lever 2: use blockwise FP8 from step zero" -- weights in 128x128 blocks.
 *
 *   W    [R, C] BF16, row stride ldw (>= C)   input
 *   Wq   [R, C] E4M3 codes, dense             output (fprop B operand)
 *   WqT  [C, R] E4M3 codes, dense, optional   output: the same codes transposed (dgrad
 *                                             B operand); NULL to skip. Needs R % 16 == 0.
 *   S    [ceil(R/128), C/128] float, dense    output; S[i*(C/128) + j] is the scale of
 *                                             block (i, j). A partial last row block
 *                                             takes its amax over the rows that exist.
 * Requires R >= 1, C % 128 == 0; W, Wq, WqT 16-byte aligned, ldw % 8 == 0.
 */
PURO_API int puro_fp8_quantize_128x128(const uint16_t *W, int64_t R, int64_t C, int64_t ldw,
                              uint8_t *Wq, uint8_t *WqT, float *S, puro_stream_t stream);

/* One weight of puro_fp8_quantize_128x128_grouped: the arguments of
 * puro_fp8_quantize_128x128 for it. */
typedef struct {
  const uint16_t *W; /* [R, C] BF16, row stride ldw       */
  int64_t R, C, ldw;
  uint8_t *Wq;       /* [R, C] codes, dense               */
  uint8_t *WqT;      /* [C, R] codes, dense, or NULL      */
  float *S;          /* [ceil(R/128), C/128] scales       */
} puro_weight_problem;

/*
 * The 128x128 quantisation of `count` weights, each exactly what puro_fp8_quantize_128x128
 * with its arguments writes (bit for bit), in one persistent launch per 64 weights instead of
 * one launch per weight. Source: "Lever 2: use blockwise FP8 from step zero" -- weights in
 * 128x128 blocks, converted to FP8 for the GEMMs that consume them. All weights of a model
 * are known before its forward pass, so a step can quantise them together: the CTAs walk the
 * weights' tiles as one sequence and one weight's tiles fill the SMs another's last wave
 * leaves idle. The problem array is read during the call only (the host copies it into the
 * launches' parameters).
 * Requires count >= 1 and, for every weight, what puro_fp8_quantize_128x128 requires; the
 * outputs of different weights must not overlap. Nothing is launched unless every weight
 * passes the checks. Status codes as for puro_fp8_quantize_128x128.
 */
PURO_API int puro_fp8_quantize_128x128_grouped(const puro_weight_problem *problems, int count,
                                               puro_stream_t stream);

/*
 * Power-of-two (UE8M0) scale mode of the three quantisers above: the same groups, codes
 * written the same way, but each group's scale is the method's amax / 448 rounded up to a
 * power of two, stored as one byte. Source: "Lever 2: use blockwise FP8 from step zero"
 * (FP8 with local scales per group of 128 / 128x128 block); the pages give no scale
 * formula, and this mode is the variant whose scales the tensor cores' block-scaled FP8
 * MMAs (puro_fp8_mx_gemm) apply themselves:
 *     e    = the smallest integer with 448 * 2^e >= amax, clamped to [-127, 127]
 *            (an all-zero group: -127)
 *     byte = e + 127                     (UE8M0)
 *     code = E4M3_RNE(x * 2^-e)          (exact scaling; nothing saturates)
 * Arguments, layouts and requirements as for puro_fp8_quantize_1x128,
 * puro_fp8_quantize_1x128_transposed and puro_fp8_quantize_128x128, with every scale
 * array (S, ST) holding bytes instead of floats (no alignment requirement).
 */
PURO_API int puro_fp8_quantize_1x128_pow2(const uint16_t *X, int64_t R, int64_t C, int64_t ldx,
                                          uint8_t *Xq, int64_t ldq, uint8_t *S, puro_stream_t stream);
PURO_API int puro_fp8_quantize_1x128_transposed_pow2(const uint16_t *X, int64_t T, int64_t C, int64_t ldx,
                                                     uint8_t *XqT, uint8_t *ST, uint8_t *Xq, uint8_t *S,
                                                     puro_stream_t stream);
PURO_API int puro_fp8_quantize_128x128_pow2(const uint16_t *W, int64_t R, int64_t C, int64_t ldw,
                                            uint8_t *Wq, uint8_t *WqT, uint8_t *S, puro_stream_t stream);

/*
 * Blockwise-FP8 GEMM with power-of-two scales, on the tensor cores' block-scaled MMA:
 *     C[m, n] = sum_kb 2^(sA(kb, m) - 127) * 2^(sB(kb, n) - 127) * sum_{k in kb} A[m, k] B[n, k]
 * The operands are the power-of-two quantisers' output (puro_fp8_quantize_*_pow2); the
 * tensor core applies each power-of-two factor exactly and accumulates all of K in FP32,
 * so no scale promotion runs on the CUDA cores. Source: "Lever 2: use blockwise FP8 from
 * step zero" (the linear-layer GEMMs in FP8 with local scales), in the power-of-two scale
 * mode described above.
 *
 *   Aq  [M, K] E4M3 codes, dense      As [K/128, M] UE8M0 bytes
 *   Bq  [N, K] E4M3 codes, dense      Bs bytes, laid out as the float Bs of
 *                                     puro_fp8_gemm_blockwise for the same layout
 *   C   [M, N] BF16, dense            output (round to nearest even)
 * Requires M >= 1, N >= 8, N % 8 == 0, K >= 128, K % 128 == 0; Aq, Bq, C 16-byte aligned;
 * for PURO_WGRAD also Bs 8-byte aligned. Status codes as for puro_fp8_gemm_blockwise.
 */
PURO_API int puro_fp8_mx_gemm(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs,
                              uint16_t *C, int64_t M, int64_t N, int64_t K, int layout, puro_stream_t stream);

/*
 * NVFP4 mode: E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one UE4M3 factor per 16
 * consecutive elements along the reduction dimension, and one FP32 tensor scale. Source: the
 * pages name FP4 only as a capability of the hardware they chose (the jj-blog page, the
 * paragraph after its Table 2); the format is NVIDIA's published NVFP4, with the method's
 * choices carried over (scales from the tensor being quantised, groups along the reduction
 * dimension, correctly rounded FP32 arithmetic):
 *     s_t = amax_t / 2688                       (2688 = 6 * 448)
 *     e   = E4M3_RNE_sat((amax_g / 6) / s_t)     the group's factor, a UE4M3 byte
 *     S   = dec(e) * s_t
 *     q   = E2M1_RNE_sat(x / S)                  (S == 0: a signed zero)
 * every step correctly rounded in FP32. Two codes per byte, element 2i in the low nibble.
 * Factors are stored by 256-element K block: F[b][r][j], 16 bytes per row and block, is the
 * factor of row r's elements 256 b + 16 j .. 256 b + 16 j + 15 (the last block's bytes past
 * the row's end are not written), so the GEMM reads one K block's factors of consecutive rows
 * as one contiguous run.
 * Inputs must be finite. Each quantiser runs two kernels on `stream`: the tensor's absolute
 * maximum (written to *amax, which the call first sets to zero), then the codes, which read
 * *amax on the device. Nothing else is written and nothing is allocated.
 *
 * puro_nvfp4_quantize_1x16: groups along the columns of X.
 *   X    [R, C] BF16, row stride ldx (>= C, % 8 == 0)   input
 *   Xq   [R, C/2] bytes, row stride ldq (>= C/2, % 8)   output: packed codes
 *   F    [ceil(C/256), R, 16] bytes                       output: factors, by K block
 *   amax one float                                       output: max |X|
 *   Requires R >= 1, C >= 16, C % 16 == 0; X, Xq, F 16-byte aligned, amax 4-byte aligned.
 * puro_nvfp4_quantize_1x16_transposed: groups of 16 consecutive rows (tokens), written
 * transposed (the wgrad operands, and W along N_out for dgrad).
 *   X    [R, C] BF16, row stride ldx (>= C, % 8 == 0)   input
 *   XqT  [C, R/2] bytes, row stride ldq (>= R/2, % 16)  output: packed codes of X^T
 *   FT   [ceil(R/256), C, 16] bytes                       output: factors of X^T's rows, by K block
 *   amax one float                                       output: max |X|
 *   Requires R % 64 == 0 (R >= 64), C % 8 == 0; alignment as above.
 * puro_nvfp4_quantize_1x16_dual: both of the above from one read of X (plus the amax pass):
 * the outputs are byte for byte those of the two calls, with one amax shared by both.
 *   X, Xq, ldq, F    as for puro_nvfp4_quantize_1x16
 *   XqT, ldqt, FT    as XqT, ldq, FT of puro_nvfp4_quantize_1x16_transposed
 *   amax             one float, output: max |X|
 *   Requires R % 64 == 0 (R >= 64), C % 16 == 0 (C >= 16), ldq % 8 == 0, ldqt % 16 == 0;
 *   alignment as above.
 * Status: PURO_ERR_NULL, PURO_ERR_SHAPE, PURO_ERR_ALIGN, PURO_ERR_DEVICE, PURO_ERR_CUDA or
 * PURO_ERR_LAUNCH, checked on the host before any launch.
 */
PURO_API int puro_nvfp4_quantize_1x16(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                                      int64_t ldq, uint8_t *F, float *amax, puro_stream_t stream);
PURO_API int puro_nvfp4_quantize_1x16_transposed(const uint16_t *X, int64_t R, int64_t C, int64_t ldx,
                                                 uint8_t *XqT, int64_t ldq, uint8_t *FT, float *amax,
                                                 puro_stream_t stream);
PURO_API int puro_nvfp4_quantize_1x16_dual(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                                           int64_t ldq, uint8_t *F, uint8_t *XqT, int64_t ldqt, uint8_t *FT,
                                           float *amax, puro_stream_t stream);

/*
 * NVFP4 GEMM on the tensor cores' block-scaled FP4 MMA, which applies the UE4M3 factors
 * itself and accumulates all of K in FP32:
 *     C[m, n] = s_tA * s_tB * sum_k dec(qA[m, k]) fA[m, k/16] dec(qB[n, k]) fB[n, k/16]
 * with s_t = amax / 2688 of each operand's tensor, rounded to BF16 (nearest even) once.
 * Both operands are quantised along K (the 1x16 quantisers above): fprop takes X and W
 * row-wise, dgrad dY row-wise and W transposed, wgrad dY and X transposed.
 *   Aq [M, K/2] packed codes, dense   As [ceil(K/256), M, 16] factors   a_amax: A's tensor amax
 *   Bq [N, K/2] packed codes, dense   Bs [ceil(K/256), N, 16] factors   b_amax: B's tensor amax
 *   C  [M, N] BF16, dense               output
 * Requires M >= 1, N >= 8, N % 8 == 0, K >= 128, K % 128 == 0; Aq, As, Bq, Bs, C 16-byte
 * aligned, the amax pointers 4-byte aligned (device memory). Status codes as for
 * puro_fp8_gemm_blockwise.
 */
PURO_API int puro_nvfp4_gemm(const uint8_t *Aq, const uint8_t *As, const float *a_amax, const uint8_t *Bq,
                             const uint8_t *Bs, const float *b_amax, uint16_t *C, int64_t M, int64_t N,
                             int64_t K, puro_stream_t stream);

/*
 * Blockwise-FP8 GEMM  C[m, n] = sum_kb sA(kb, m) * sB(kb, n) * sum_{k in kb} A[m, k] B[n, k]
 * with an FP32 tensor-core partial per 128-wide K block, FP32 promotion and BF16 output.
 * Source: "Lever 2: use blockwise FP8 from step zero" (the linear-layer GEMMs in FP8
 * with local scales); forward, dgrad and wgrad of one linear layer are the three
 * layouts below.
 *
 *   Aq  [M, K] E4M3 codes, dense      As [K/128, M] float    (1x128 along K)
 *   Bq  [N, K] E4M3 codes, dense      Bs depends on layout:
 *     PURO_FPROP  Y  = X W^T:   Bq = Wq,  Bs = S of W  [ceil(N/128), K/128]
 *     PURO_DGRAD  dX = dY W:    Bq = WqT, Bs = S of W  [K/128, ceil(N/128)]
 *     PURO_WGRAD  dW = dY^T X:  Bq = XqT, Bs = ST of X [K/128, N]
 *   C   [M, N] BF16, dense            output
 *   workspace, ws_bytes   ignored: no layout of this version needs scratch memory.
 *                         Pass NULL / 0 (any value is accepted).
 * Requires M >= 1, N >= 8, N % 8 == 0, K >= 128, K % 128 == 0; Aq, Bq, C 16-byte aligned;
 * As, Bs 4-byte aligned. M and N need not be multiples of the tile size.
 */
PURO_API int puro_fp8_gemm_blockwise(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                            const float *Bs, uint16_t *C, int64_t M, int64_t N, int64_t K,
                            int layout, void *workspace, size_t ws_bytes,
                            puro_stream_t stream);

/* One GEMM of a grouped launch: the operands and output of a puro_fp8_gemm_blockwise call. */
typedef struct {
  const uint8_t *Aq; /* [M, K] codes            */
  const float *As;   /* [K/128, M] scales        */
  const uint8_t *Bq; /* [N, K] codes            */
  const float *Bs;   /* scales, layout-dependent */
  uint16_t *C;       /* [M, N] BF16 output       */
  int64_t M, N, K;
} puro_gemm_problem;

/* Largest number of problems in one puro_fp8_gemm_blockwise_grouped call. */
enum { PURO_GROUP_MAX = 4 };

/*
 * 1 to PURO_GROUP_MAX independent GEMMs of the same layout in one persistent launch: each
 * problem computes exactly what puro_fp8_gemm_blockwise with its arguments computes (bit for
 * bit: same tiles, same order of additions). Source: "Lever 2: use blockwise FP8 from step
 * zero" (the linear-layer GEMMs in FP8). A layer's weight gradients need only their own dY
 * and X, so they can share one launch: the CTAs walk the problems' tiles as one sequence
 * (the problems with the most K blocks first), and the tiles of one problem fill the SMs
 * another problem's last wave leaves idle.
 *
 *   problems  host array of `count` descriptors (read during the call, not kept); every
 *             problem obeys the requirements of puro_fp8_gemm_blockwise
 *   count     1 .. PURO_GROUP_MAX
 *   layout    PURO_FPROP, PURO_DGRAD or PURO_WGRAD, for every problem
 * Outputs of different problems must not overlap. Status codes as for
 * puro_fp8_gemm_blockwise; PURO_ERR_SHAPE also for a count outside 1 .. PURO_GROUP_MAX.
 */
PURO_API int puro_fp8_gemm_blockwise_grouped(const puro_gemm_problem *problems, int count, int layout,
                                             puro_stream_t stream);

/*
 * fprop or dgrad whose epilogue also quantises its own output for the next GEMM:
 *     C = the PURO_FPROP / PURO_DGRAD product of puro_fp8_gemm_blockwise (BF16), and
 *     Cq, Cs = the 1x128 quantisation of that BF16 C along N, exactly what
 *              puro_fp8_quantize_1x128(C, ...) with ldq = N would write from it.
 * Source: "Lever 2: use blockwise FP8 from step zero" -- tensors are converted to FP8 only
 * for the GEMM that consumes them, in groups of 128 along its reduction dimension. When
 * the output feeds another linear layer as its input, that dimension is this GEMM's N,
 * and each thread of the epilogue already holds one output row x 128 columns: the group's
 * amax, scale and codes are formed from the BF16 values in its registers, so the BF16
 * output is not read back by a separate quantiser pass.
 *
 *   Aq, As, Bq, Bs, M, N, K, layout   as for puro_fp8_gemm_blockwise (PURO_FPROP or
 *                                     PURO_DGRAD only; PURO_ERR_LAYOUT otherwise)
 *   C   [M, N] BF16, dense            output
 *   Cq  [M, N] E4M3 codes, dense      output
 *   Cs  [N/128, M] float, dense       output; Cs[j*M + m] is the scale of C[m, 128j .. +127]
 * Requires M >= 1, N >= 128, N % 128 == 0, K >= 128, K % 128 == 0; Aq, Bq, C, Cq 16-byte
 * aligned; As, Bs, Cs 4-byte aligned. Status codes as for puro_fp8_gemm_blockwise.
 */
PURO_API int puro_fp8_gemm_blockwise_quant(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                           const float *Bs, uint16_t *C, uint8_t *Cq, float *Cs,
                                           int64_t M, int64_t N, int64_t K, int layout,
                                           puro_stream_t stream);

/*
 * Weight gradient with FP32 accumulation:
 *     C[m, n] += sum_kb sA(kb, m) * sB(kb, n) * sum_{k in kb} A[m, k] B[n, k]
 * the PURO_WGRAD product of puro_fp8_gemm_blockwise (same operands, same FP32 promotion),
 * added into an FP32 main-gradient buffer instead of written as BF16. Source: "Lever 2: use
 * blockwise FP8 from step zero" (master weights and gradients stay in BF16/FP32; FP8 is the
 * compute format of the GEMMs only): each micro-step's FP8 weight gradient is accumulated
 * at FP32.
 *
 *   Aq  [M, K] E4M3 codes = dY^T quantised 1x128 along the tokens, As [K/128, M]
 *   Bq  [N, K] E4M3 codes = X^T quantised 1x128 along the tokens,  Bs [K/128, N]
 *   C   [M, N] FP32, dense, read and written: every element gets exactly one FP32 add
 *       (round to nearest) of its FP32 product per call, done by the TMA unit at L2.
 * Requires M >= 1, N >= 8, N % 8 == 0, K >= 128, K % 128 == 0; Aq, Bq, C 16-byte aligned,
 * As, Bs 4-byte aligned. Calls that add into the same C must not overlap on the GPU.
 * Status codes as for puro_fp8_gemm_blockwise.
 */
PURO_API int puro_fp8_gemm_wgrad_acc_f32(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                         const float *Bs, float *C, int64_t M, int64_t N,
                                         int64_t K, puro_stream_t stream);

/*
 * Waits for all work on the current device (every stream, not only `stream`), then
 * reads and clears the device's status word, which any kernel of this library sets
 * when a bounded wait gives up. `stream` carries the two small copies of the word.
 * Returns PURO_OK (every call enqueued before this one finished and its outputs are
 * valid), PURO_ERR_TIMEOUT (some kernel gave up; its outputs are partly written), or
 * PURO_ERR_CUDA if the synchronisation itself reported an error.
 */
PURO_API int puro_fp8_sync_status(puro_stream_t stream);

/* Human-readable text of a puro_status value (static storage, never NULL). */
PURO_API const char *puro_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* PURO_FP8_H */
