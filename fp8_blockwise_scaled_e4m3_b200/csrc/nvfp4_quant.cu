// NVFP4 quantisers (memory-bound), sm_100a: BF16 -> E2M1 codes with a UE4M3 factor per 16
// elements along the reduction dimension and one FP32 tensor scale.
//
// The pages name FP4 only as a capability of the hardware they chose (the jj-blog page, the
// paragraph after its Table 2); the format is NVIDIA's published NVFP4, with the method's
// choices carried over (scales from the tensor being quantised, groups along the reduction
// dimension, correctly rounded FP32 arithmetic). Per tensor and per 16-element group:
//   s_t = RN(amax_t / 2688)          2688 = 6 * 448 (E2M1 max times E4M3 max)
//   e   = E4M3_RNE_sat(RN(RN(amax_g / 6) / s_t))      the group's UE4M3 factor
//   S   = RN(dec(e) * s_t)
//   q   = E2M1_RNE_sat(RN(x / S)), or a signed zero when S == 0
// Two codes per byte (element 2i in the low nibble). Factors are stored by 256-element K
// block: F[b][r][j] (16 bytes per row and block) is the factor of X[r, 256 b + 16 j ..], so the
// GEMM reads a K block's factors of consecutive rows as one contiguous run. Quotients are
// correctly rounded through the group's reciprocal with Markstein's correction (as in the FP8
// quantisers; IEEE division below divisors of 2^-90). The tensor amax is an output of its own
// kernel, read by the quantising kernel from device memory, so the two launches need no host
// round trip. Inputs must be finite.
//
//   k_nv_amax        max |x| over X [R, C], by atomicMax on its FP32 bit pattern (non-negative
//                    floats order like their bit patterns); the word starts at zero
//   k_nv_quant_rows  one thread per 16-element group along the columns: 32-byte loads, one
//                    8-byte store of codes and one factor byte, consecutive threads on
//                    consecutive groups of a row (16 consecutive factor bytes per K block)
//   k_nv_quant_cols  groups of 16 consecutive rows, written transposed: a thread takes two
//                    adjacent columns over 64 rows (4-byte loads, a warp reads 128 contiguous
//                    bytes of each row) and writes 32 bytes of codes and 4 factor bytes (one
//                    4-byte store into its K block's 16) per column

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>

#include "../../include/puro_fp8.h"
#include "host_cache.h"
#include "quant.h"
#include "quant_math.cuh"

namespace puro {
namespace {

constexpr float kTensorDiv = 2688.0f;  // 6 * 448
constexpr int kThreads = 256;

// two E2M1 codes in one byte: `lo` in bits 0..3, `hi` in bits 4..7 (RN, satfinite)
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t v;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(v)
      : "f"(hi), "f"(lo));
  return v & 0xFFu;
}

// value of a non-negative E4M3 byte (exact): subnormal m * 2^-9, normal (8 + m) * 2^(e - 10)
__device__ __forceinline__ float ue4m3_value(uint32_t b) {
  const uint32_t ex = (b >> 3) & 0xFu, m = b & 7u;
  return ex == 0 ? static_cast<float>(m) * 0.001953125f  // 2^-9
                 : __uint_as_float(((ex + 120u) << 23) | (m << 20));
}

// The group factor and its decoded scale S for group maximum `amax_g` (an FP32 value of a
// BF16 magnitude) and tensor scale s_t.
__device__ __forceinline__ void group_scale(float amax_g, float s_t, uint32_t &e, float &S) {
  if (s_t > 0.0f) {
    const float d = __fdiv_rn(amax_g, 6.0f);
    e = e4m3x2(__fdiv_rn(d, s_t), 0.0f) & 0xFFu;
    S = __fmul_rn(ue4m3_value(e), s_t);
  } else {
    e = 0;
    S = 0.0f;
  }
}

// the divider of a group with decoded scale S (S == 0: every quotient a signed zero)
__device__ __forceinline__ BlockDivider group_divider(float S) {
  return S > 0.0f ? make_divider(S) : zero_block_divider();
}

// codes of two elements
__device__ __forceinline__ uint32_t codes2(float x0, float x1, const BlockDivider &dv) {
  return e2m1x2(block_divide(dv, x0), block_divide(dv, x1));
}

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t m, uint32_t w) {
  w &= 0x7FFF7FFFu;
  return max(m, max(w & 0xFFFFu, w >> 16));
}

__global__ void __launch_bounds__(kThreads) k_nv_amax(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t ldx,
                                                      uint32_t *amax_bits) {
  const int64_t chunks_per_row = C / 8;  // 16-byte chunks of 8 BF16
  const int64_t total = R * chunks_per_row;
  uint32_t m = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / chunks_per_row, c = (i - r * chunks_per_row) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X + r * ldx + c));
    m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(m, v.x), v.y), v.z), v.w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax_bits, m << 16);
}

__global__ void __launch_bounds__(kThreads) k_nv_quant_rows(const uint16_t *__restrict__ X, int64_t R, int64_t C,
                                                            int64_t ldx, uint8_t *__restrict__ Xq, int64_t ldq,
                                                            uint8_t *__restrict__ F, const float *amax_t) {
  const float s_t = __fdiv_rn(*amax_t, kTensorDiv);
  const int64_t groups_per_row = C / 16;
  const int64_t total = R * groups_per_row;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = g / groups_per_row, j = g - r * groups_per_row;
    const uint4 *src = reinterpret_cast<const uint4 *>(X + r * ldx + 16 * j);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = absmax_bf16x2(m, w[i]);
    uint32_t e;
    float S;
    group_scale(__uint_as_float(m << 16), s_t, e, S);
    const BlockDivider dv = group_divider(S);
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = codes2(bf16_lo(w[i]), bf16_hi(w[i]), dv);
    uint2 out;
    out.x = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
    out.y = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
    *reinterpret_cast<uint2 *>(Xq + r * ldq + 8 * j) = out;
    F[((j >> 4) * R + r) * 16 + (j & 15)] = static_cast<uint8_t>(e);
  }
}

// X [R, C] -> XqT [C, R/2] (row stride ldq bytes), FT [R/256 (rounded up)][C][16]; R % 64 == 0,
// C % 2 == 0.
__global__ void __launch_bounds__(kThreads) k_nv_quant_cols(const uint16_t *__restrict__ X, int64_t R, int64_t C,
                                                            int64_t ldx, uint8_t *__restrict__ XqT, int64_t ldq,
                                                            uint8_t *__restrict__ FT, const float *amax_t) {
  const float s_t = __fdiv_rn(*amax_t, kTensorDiv);
  const int64_t pairs = C / 2, slabs = R / 64;
  const int64_t total = pairs * slabs;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t slab = t / pairs, c0 = 2 * (t - slab * pairs), r0 = 64 * slab;
    const uint32_t *src = reinterpret_cast<const uint32_t *>(X + r0 * ldx + c0);
    const int64_t step = ldx / 2;  // 4-byte words per row
    uint32_t w[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) w[i] = __ldg(src + i * step);
#pragma unroll
    for (int col = 0; col < 2; ++col) {
      uint32_t fac = 0;
      uint32_t out[8];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t h = col ? (w[16 * g + i] >> 16) : (w[16 * g + i] & 0xFFFFu);
          m = max(m, h & 0x7FFFu);
        }
        uint32_t e;
        float S;
        group_scale(__uint_as_float(m << 16), s_t, e, S);
        fac |= e << (8 * g);
        const BlockDivider dv = group_divider(S);
        uint32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t a = w[16 * g + 2 * i], b = w[16 * g + 2 * i + 1];
          q[i] = col ? codes2(bf16_hi(a), bf16_hi(b), dv) : codes2(bf16_lo(a), bf16_lo(b), dv);
        }
        out[2 * g] = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
        out[2 * g + 1] = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
      }
      uint8_t *dst = XqT + (c0 + col) * ldq + r0 / 2;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
      *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
      // groups 4 slab .. 4 slab + 3 of column c0 + col: K block slab / 4, bytes 4 (slab % 4) ..
      *reinterpret_cast<uint32_t *>(FT + ((slab >> 2) * C + (c0 + col)) * 16 + 4 * (slab & 3)) = fac;
    }
  }
}

int grid_for(int64_t work) {
  int sms = 0;
  if (!sm_count(sms)) return -1;
  const int64_t blocks = (work + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  return static_cast<int>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

int launch_amax(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, float *amax, cudaStream_t stream) {
  if (cudaMemsetAsync(amax, 0, sizeof(float), stream) != cudaSuccess) return PURO_ERR_CUDA;
  const int grid = grid_for(R * (C / 8));
  if (grid < 0) return PURO_ERR_CUDA;
  k_nv_amax<<<grid, kThreads, 0, stream>>>(X, R, C, ldx, reinterpret_cast<uint32_t *>(amax));
  return cudaGetLastError() == cudaSuccess ? PURO_OK : PURO_ERR_LAUNCH;
}

}  // namespace

int launch_nvfp4_quant_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq, int64_t ldq,
                            uint8_t *F, float *amax, cudaStream_t stream) {
  const int rc = launch_amax(X, R, C, ldx, amax, stream);
  if (rc != PURO_OK) return rc;
  const int grid = grid_for(R * (C / 16));
  if (grid < 0) return PURO_ERR_CUDA;
  k_nv_quant_rows<<<grid, kThreads, 0, stream>>>(X, R, C, ldx, Xq, ldq, F, amax);
  return cudaGetLastError() == cudaSuccess ? PURO_OK : PURO_ERR_LAUNCH;
}

int launch_nvfp4_quant_cols(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *XqT, int64_t ldq,
                            uint8_t *FT, float *amax, cudaStream_t stream) {
  const int rc = launch_amax(X, R, C, ldx, amax, stream);
  if (rc != PURO_OK) return rc;
  const int grid = grid_for((C / 2) * (R / 64));
  if (grid < 0) return PURO_ERR_CUDA;
  k_nv_quant_cols<<<grid, kThreads, 0, stream>>>(X, R, C, ldx, XqT, ldq, FT, amax);
  return cudaGetLastError() == cudaSuccess ? PURO_OK : PURO_ERR_LAUNCH;
}

}  // namespace puro
