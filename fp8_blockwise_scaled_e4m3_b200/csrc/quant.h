// Internal launchers of the quantiser and GEMM kernels (host side). Arguments are
// validated by the C-ABI layer before these are called.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/puro_fp8.h"

namespace puro {

// Quantiser launchers; return 0 or a negative puro_status. With the byte pointers set (Sb,
// STb) the scales are the power-of-two (UE8M0) mode's bytes and the float pointers unused.
int launch_quant_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                      int64_t ldq, float *S, cudaStream_t stream, uint8_t *Sb = nullptr);
int launch_quant_cols(const uint16_t *X, int64_t T, int64_t C, int64_t ldx, uint8_t *XqT,
                      float *ST, uint8_t *Xq, float *S, cudaStream_t stream, uint8_t *STb = nullptr,
                      uint8_t *Sb = nullptr);
int launch_quant_weight(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, uint8_t *Wq,
                        uint8_t *WqT, float *S, cudaStream_t stream, uint8_t *Sb = nullptr);

// Many weights' 128x128 quantisations in persistent launches of up to 64 weights each.
using WeightProblem = puro_weight_problem;
int launch_quant_weight_grouped(const WeightProblem *problems, int count, cudaStream_t stream);

// NVFP4 (E2M1 codes, a UE4M3 factor per 16 elements along the reduction dimension, an FP32
// tensor amax): the row-wise and transposed 1x16 quantisers (each also writes the tensor's
// amax) and the GEMM C = A . B^T of two operands quantised along K.
int launch_nvfp4_quant_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq, int64_t ldq,
                            uint8_t *F, float *amax, cudaStream_t stream);
int launch_nvfp4_quant_cols(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *XqT, int64_t ldq,
                            uint8_t *FT, float *amax, cudaStream_t stream);
int launch_nvfp4_quant_dual(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq, int64_t ldq,
                            uint8_t *F, uint8_t *XqT, int64_t ldqt, uint8_t *FT, float *amax,
                            cudaStream_t stream);
int launch_gemm_nvfp4(const uint8_t *Aq, const uint8_t *As, const float *a_amax, const uint8_t *Bq,
                      const uint8_t *Bs, const float *b_amax, uint16_t *C, int64_t M, int64_t N, int64_t K,
                      cudaStream_t stream);
int read_and_clear_nv_status(cudaStream_t stream, int *status_out);
// NVFP4 host helpers shared by its quantisers and GEMM: the device status word its kernels
// raise when a bounded wait gives up (address cached per device), the wait limit, and a
// tensor map of a BF16 matrix [rows, cols] with row stride `ld` elements, box [box_rows x 64]
// (128 bytes per row, 128-byte swizzle), reads past the edge returning zeros.
int *nv_status_word();
unsigned long long nv_wait_timeout_ns();
bool nv_bf16_map(CUtensorMap *map, const uint16_t *X, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows);

// Reads and clears the quantisers' device status word (after a stream sync).
int read_and_clear_quant_status(cudaStream_t stream, int *status_out);

// Returns 0 on success, a negative puro_status on failure.
int launch_gemm_blockwise(const uint8_t *Aq, const float *As, const uint8_t *Bq, const float *Bs,
                          uint16_t *C, int64_t M, int64_t N, int64_t K, int layout,
                          cudaStream_t stream);

// Up to PURO_GROUP_MAX GEMMs of one layout in one persistent launch (see
// puro_fp8_gemm_blockwise_grouped).
using GroupedProblem = puro_gemm_problem;
int launch_gemm_blockwise_grouped(const GroupedProblem *problems, int count, int layout,
                                  cudaStream_t stream);

// fprop / dgrad whose epilogue also writes the 1x128 quantisation of the BF16 output along
// N: codes Cq [M, N] and scales Cs [N/128, M].
int launch_gemm_blockwise_quant(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                const float *Bs, uint16_t *C, uint8_t *Cq, float *Cs, int64_t M,
                                int64_t N, int64_t K, int layout, cudaStream_t stream);

// wgrad with FP32 accumulation: C[M, N] (FP32) += the wgrad product.
int launch_gemm_wgrad_acc_f32(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                              const float *Bs, float *C, int64_t M, int64_t N, int64_t K,
                              cudaStream_t stream);

// Blockwise GEMM with power-of-two scale bytes on the block-scaled MMA; and its status word.
int launch_gemm_mx(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs, uint16_t *C,
                   int64_t M, int64_t N, int64_t K, int layout, cudaStream_t stream);
int read_and_clear_mx_status(cudaStream_t stream, int *status_out);

// Reads and clears the device status word of the GEMM kernels (after a stream sync).
int read_and_clear_device_status(cudaStream_t stream, int *status_out);

}  // namespace puro
