// Blockwise BF16 -> E4M3 quantisers (memory-bound), sm_100a.
//
// "Paper walkthrough: Puro-2B ...", section "Lever 2: use blockwise FP8 from step zero":
// activations and their gradients get one scale per 128 elements along the reduction
// dimension, weights one scale per 128x128 block. Per block, in FP32:
//   amax = max|x|;  s = amax / 448 (IEEE division);  q = E4M3_rn_satfinite(x / s)
// and an all-zero block stores s = 0 with signed-zero codes (x / 1 keeps the sign).
//
// Kernels:
//   k_quant_rows      1x128 along the columns of X [R, C]     (fprop A, dgrad A)
//   k_quant_cols      1x128 along the rows (tokens), output transposed, optionally also
//                     the row-wise codes from the same read   (wgrad A and B)
//   k_quant_weight    128x128 blocks, optionally the transposed codes (fprop / dgrad B)
// All read BF16 with 16-byte vector loads, several in flight per thread, and reduce
// amax with warp shuffles; the transposed outputs go through a shared-memory tile so
// every global store is a full 16-byte vector of a contiguous 128-byte row.

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "quant.h"
#include "quant_math.cuh"

namespace puro {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerHalfWarp = 4;            // k_quant_rows: rows per 16-lane group
constexpr int kRowsPerCta = 16 * kRowsPerHalfWarp;
constexpr int kTile = 128;                      // transposed kernels: 128 x 128 tile
constexpr int kPitch = kTile * 2 + 16;          // BF16 tile row pitch in bytes (272)
constexpr int kCodePitch = kTile + 16;          // code tile row pitch in bytes (144)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 load_stream(const uint16_t *p) {
  return __ldcs(reinterpret_cast<const uint4 *>(p));
}

// Four quotients -> four E4M3 codes, first argument in the lowest byte.
__device__ __forceinline__ uint32_t codes4(float a, float b, float c, float d,
                                           const BlockDivider &div) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(
      make_float2(block_divide(div, a), block_divide(div, b)), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(
      make_float2(block_divide(div, c), block_divide(div, d)), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__device__ __forceinline__ float absmax8(const uint4 &v) {
  float m = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
  return m;
}

__device__ __forceinline__ uint2 codes8(const uint4 &v, const BlockDivider &div) {
  return make_uint2(codes4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y), div),
                    codes4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w), div));
}

// Scale of a block with absolute maximum `amax`, and the divider for its codes.
__device__ __forceinline__ void block_scale(float amax, float &s, BlockDivider &div) {
  s = __fdiv_rn(amax, 448.0f);
  div = amax > 0.0f ? make_divider(s) : zero_block_divider();
}

// Max over the 16 lanes of a half-warp (lanes 0-15 and 16-31 reduce separately).
__device__ __forceinline__ float halfwarp_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return v;
}

// ------------------------------------------------------------------ 1x128 along columns
// CTA = 64 rows x one 128-column block. Half-warp h handles rows base + h + 16u, lane l
// of the half-warp columns 8l .. 8l+7. All four loads are issued before any arithmetic.
__global__ void __launch_bounds__(kThreads) k_quant_rows(const uint16_t *__restrict__ X, int64_t R,
                                                         int64_t ldx, uint8_t *__restrict__ Xq,
                                                         int64_t ldq, float *__restrict__ S) {
  const int hw = threadIdx.x >> 4;
  const int l = threadIdx.x & 15;
  const int64_t j = blockIdx.y;
  const int64_t r_first = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + hw;
  uint4 v[kRowsPerHalfWarp];
#pragma unroll
  for (int u = 0; u < kRowsPerHalfWarp; ++u) {
    const int64_t r = r_first + 16 * u;
    v[u] = r < R ? load_stream(X + r * ldx + j * kTile + l * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int u = 0; u < kRowsPerHalfWarp; ++u) {
    const int64_t r = r_first + 16 * u;
    const float amax = halfwarp_max(absmax8(v[u]));
    float s;
    BlockDivider div;
    block_scale(amax, s, div);
    const uint2 q = codes8(v[u], div);
    if (r < R) {
      *reinterpret_cast<uint2 *>(Xq + r * ldq + j * kTile + l * 8) = q;
      if (l == 0) S[j * R + r] = s;
    }
  }
}

// ------------------------------------------------------------------ shared tile helpers
// The transposed kernels stage a 128-row x 128-column BF16 tile (rows = tokens for the
// activation quantiser, output features for the weight quantiser) in shared memory.
// Loading: half-warp h, lane l reads row h + 16p (p = 0..7), columns 8l .. 8l+7.

struct TileLoad {
  uint4 v[8];
};

__device__ __forceinline__ void load_tile(TileLoad &t, const uint16_t *__restrict__ X,
                                          int64_t row0, int64_t rows_valid, int64_t col0,
                                          int64_t cols, int64_t ldx) {
  const int hw = threadIdx.x >> 4;
  const int l = threadIdx.x & 15;
  const int64_t col = col0 + l * 8;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t r = hw + 16 * p;
    t.v[p] = (r < rows_valid && col < cols) ? load_stream(X + (row0 + r) * ldx + col)
                                            : make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void store_tile_smem(const TileLoad &t, uint8_t *tile) {
  const int hw = threadIdx.x >> 4;
  const int l = threadIdx.x & 15;
#pragma unroll
  for (int p = 0; p < 8; ++p)
    *reinterpret_cast<uint4 *>(tile + (hw + 16 * p) * kPitch + l * 16) = t.v[p];
}

// Column phase. Thread (cp = tid % 64, g = tid / 64) holds columns 2cp, 2cp+1 of tile
// rows 32g .. 32g+31 as BF16 pairs.
__device__ __forceinline__ void read_column_pairs(const uint8_t *tile, uint32_t (&w)[32]) {
  const int cp = threadIdx.x & 63;
  const int g = threadIdx.x >> 6;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    w[i] = *reinterpret_cast<const uint32_t *>(tile + (32 * g + i) * kPitch + cp * 4);
}

// Codes of the held column pair with divisors div0 (column 2cp) and div1 (column 2cp+1)
// into the code tile: code tile row = tile column, 128 bytes = the 128 tile rows.
__device__ __forceinline__ void column_codes_to_smem(const uint32_t (&w)[32],
                                                     const BlockDivider &div0,
                                                     const BlockDivider &div1, uint8_t *codes) {
  const int cp = threadIdx.x & 63;
  const int g = threadIdx.x >> 6;
  uint32_t q0[8], q1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    q0[i] = codes4(bf16_lo(w[4 * i]), bf16_lo(w[4 * i + 1]), bf16_lo(w[4 * i + 2]),
                   bf16_lo(w[4 * i + 3]), div0);
    q1[i] = codes4(bf16_hi(w[4 * i]), bf16_hi(w[4 * i + 1]), bf16_hi(w[4 * i + 2]),
                   bf16_hi(w[4 * i + 3]), div1);
  }
  uint8_t *row0 = codes + (2 * cp) * kCodePitch + 32 * g;
  uint8_t *row1 = row0 + kCodePitch;
  reinterpret_cast<uint4 *>(row0)[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
  reinterpret_cast<uint4 *>(row0)[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
  reinterpret_cast<uint4 *>(row1)[0] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
  reinterpret_cast<uint4 *>(row1)[1] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
}

// Code tile -> global: row c of the tile goes to out[(col0 + c) * ld_out + row0 ...],
// 16 bytes per thread, 8 threads per 128-byte row. Only columns < cols and 16-row
// chunks < rows_valid are written.
__device__ __forceinline__ void store_code_tile(const uint8_t *codes, uint8_t *__restrict__ out,
                                                int64_t ld_out, int64_t row0, int64_t rows_valid,
                                                int64_t col0, int64_t cols) {
  const int chunk = threadIdx.x & 7;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int c = (threadIdx.x >> 3) + 32 * p;
    if (col0 + c < cols && 16 * chunk < rows_valid) {
      const uint4 q = *reinterpret_cast<const uint4 *>(codes + c * kCodePitch + 16 * chunk);
      *reinterpret_cast<uint4 *>(out + (col0 + c) * ld_out + row0 + 16 * chunk) = q;
    }
  }
}

// ------------------------------------------------------------------ 1x128 along tokens
// CTA = 128 tokens x 128 columns. Optional dual output: the row-wise 1x128 codes of the
// same rows, computed from the registers of the load (16 lanes hold one row block).
__global__ void __launch_bounds__(kThreads) k_quant_cols(const uint16_t *__restrict__ X, int64_t T,
                                                         int64_t C, int64_t ldx,
                                                         uint8_t *__restrict__ XqT,
                                                         float *__restrict__ ST,
                                                         uint8_t *__restrict__ Xq,
                                                         float *__restrict__ S) {
  __shared__ __align__(16) uint8_t tile[kTile * kPitch];
  __shared__ float part[4][kTile];
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int64_t tok0 = static_cast<int64_t>(blockIdx.y) * kTile;

  TileLoad t;
  load_tile(t, X, tok0, kTile, col0, C, ldx);
  store_tile_smem(t, tile);
  if (Xq != nullptr) {  // uniform over the grid
    const int hw = threadIdx.x >> 4;
    const int l = threadIdx.x & 15;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int64_t tok = tok0 + hw + 16 * p;
      const float amax = halfwarp_max(absmax8(t.v[p]));
      float s;
      BlockDivider div;
      block_scale(amax, s, div);
      *reinterpret_cast<uint2 *>(Xq + tok * C + col0 + l * 8) = codes8(t.v[p], div);
      if (l == 0) S[blockIdx.x * T + tok] = s;
    }
  }
  __syncthreads();

  uint32_t w[32];
  read_column_pairs(tile, w);
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    a0 = fmaxf(a0, fabsf(bf16_lo(w[i])));
    a1 = fmaxf(a1, fabsf(bf16_hi(w[i])));
  }
  const int cp = threadIdx.x & 63;
  const int g = threadIdx.x >> 6;
  part[g][2 * cp] = a0;
  part[g][2 * cp + 1] = a1;
  __syncthreads();  // every thread has read its tile slice: the tile may be reused
  a0 = fmaxf(fmaxf(part[0][2 * cp], part[1][2 * cp]), fmaxf(part[2][2 * cp], part[3][2 * cp]));
  a1 = fmaxf(fmaxf(part[0][2 * cp + 1], part[1][2 * cp + 1]),
             fmaxf(part[2][2 * cp + 1], part[3][2 * cp + 1]));
  float s0, s1;
  BlockDivider d0, d1;
  block_scale(a0, s0, d0);
  block_scale(a1, s1, d1);
  uint8_t *codes = tile;  // reuse: 128 x kCodePitch bytes fit in the BF16 tile
  column_codes_to_smem(w, d0, d1, codes);
  if (g == 0) {
    const int64_t c = col0 + 2 * cp;
    if (c < C) ST[blockIdx.y * C + c] = s0;
    if (c + 1 < C) ST[blockIdx.y * C + c + 1] = s1;
  }
  __syncthreads();
  store_code_tile(codes, XqT, T, tok0, kTile, col0, C);
}

// ------------------------------------------------------------------ 128x128 weight blocks
__global__ void __launch_bounds__(kThreads) k_quant_weight(const uint16_t *__restrict__ W,
                                                           int64_t R, int64_t C, int64_t ldw,
                                                           uint8_t *__restrict__ Wq,
                                                           uint8_t *__restrict__ WqT,
                                                           float *__restrict__ S) {
  __shared__ __align__(16) uint8_t tile[kTile * kPitch];
  __shared__ float warp_max[kThreads / 32];
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * kTile;
  const int64_t rows_valid = R - row0 < kTile ? R - row0 : kTile;

  TileLoad t;
  load_tile(t, W, row0, rows_valid, col0, C, ldw);
  float m = 0.0f;
#pragma unroll
  for (int p = 0; p < 8; ++p) m = fmaxf(m, absmax8(t.v[p]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  if (WqT != nullptr) store_tile_smem(t, tile);
  __syncthreads();
  float amax = warp_max[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) amax = fmaxf(amax, warp_max[i]);
  float s;
  BlockDivider div;
  block_scale(amax, s, div);
  if (threadIdx.x == 0) S[blockIdx.y * (C / kTile) + blockIdx.x] = s;

  const int hw = threadIdx.x >> 4;
  const int l = threadIdx.x & 15;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t r = hw + 16 * p;
    if (r < rows_valid)
      *reinterpret_cast<uint2 *>(Wq + (row0 + r) * C + col0 + l * 8) = codes8(t.v[p], div);
  }
  if (WqT == nullptr) return;  // uniform over the grid

  uint32_t w[32];
  read_column_pairs(tile, w);
  __syncthreads();
  column_codes_to_smem(w, div, div, tile);
  __syncthreads();
  store_code_tile(tile, WqT, R, row0, rows_valid, col0, C);
}

}  // namespace

// ------------------------------------------------------------------ launchers
cudaError_t launch_quant_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                              int64_t ldq, float *S, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>((R + kRowsPerCta - 1) / kRowsPerCta),
            static_cast<unsigned>(C / kTile));
  k_quant_rows<<<grid, kThreads, 0, stream>>>(X, R, ldx, Xq, ldq, S);
  return cudaGetLastError();
}

cudaError_t launch_quant_cols(const uint16_t *X, int64_t T, int64_t C, int64_t ldx, uint8_t *XqT,
                              float *ST, uint8_t *Xq, float *S, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>((C + kTile - 1) / kTile), static_cast<unsigned>(T / kTile));
  k_quant_cols<<<grid, kThreads, 0, stream>>>(X, T, C, ldx, XqT, ST, Xq, S);
  return cudaGetLastError();
}

cudaError_t launch_quant_weight(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, uint8_t *Wq,
                                uint8_t *WqT, float *S, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(C / kTile), static_cast<unsigned>((R + kTile - 1) / kTile));
  k_quant_weight<<<grid, kThreads, 0, stream>>>(W, R, C, ldw, Wq, WqT, S);
  return cudaGetLastError();
}

}  // namespace puro
