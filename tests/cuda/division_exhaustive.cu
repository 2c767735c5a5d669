// Test-only kernels: the quantisers' block scale s = RN(amax / 448) against IEEE division
// for every positive finite BF16 amax, and their per-block quotient (Markstein's correction with a
// correctly rounded reciprocal, IEEE division for tiny scales) against CUDA's
// correctly rounded division, for every pair the quantisers can meet: every positive
// finite BF16 amax, its scale s = RN(amax / 448), and every BF16 x with |x| <= amax.
// Counts: [0] E4M3 code mismatches (satfinite RNE of the two quotients, and the codes of
// the packed four-value helper the kernels use), [1] pairs checked, [2] quotient bit
// mismatches where |x/s| >= 2^-11 (the range in which E4M3 rounding decisions are
// taken), [3] quotient bit mismatches anywhere.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../fp8_blockwise_scaled_e4m3_b200/csrc/quant_math.cuh"

namespace {

__device__ __forceinline__ unsigned code_of(float q) {
  return __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
}

__global__ void k_check(unsigned long long *counts, unsigned int *first_bad) {
  const uint32_t amax_bits = blockIdx.x + 1;  // 0x0001 .. 0x7F7F
  const float amax = __uint_as_float(amax_bits << 16);
  const float s = __fdiv_rn(amax, 448.0f);
  // the scale and divider as the kernels form them: branch-free when the block allows it
  float s_kernel;
  puro::BlockDivider d;
  bool ok;
  puro::block_scale_fast(amax, s_kernel, d, ok);
  if (!ok) puro::block_scale(amax, s_kernel, d);
  unsigned long long bad = 0, n = 0, qbad_big = 0, qbad = 0;
  for (uint32_t xb = threadIdx.x + blockIdx.y * blockDim.x; xb < 65536u;
       xb += blockDim.x * gridDim.y) {
    const float x = __uint_as_float(xb << 16);
    if (!(fabsf(x) <= amax)) continue;  // also skips NaN patterns
    ++n;
    const float fast = puro::block_divide(d, x);
    const float ref = __fdiv_rn(x, s);
    const uint32_t w = xb | (xb << 16);  // x in both halves of a BF16 pair
    const uint32_t packed = puro::block_codes4(w, w, d);
    const unsigned want = code_of(ref);
    const bool packed_ok = (packed & 0xFFu) == want && ((packed >> 8) & 0xFFu) == want &&
                           ((packed >> 16) & 0xFFu) == want && (packed >> 24) == want;
    if (code_of(fast) != want || !packed_ok) {
      ++bad;
      atomicCAS(first_bad, 0u, (amax_bits << 16) | xb);
    }
    if (__float_as_uint(fast) != __float_as_uint(ref)) {
      ++qbad;
      if (fabsf(ref) >= 0x1p-11f) ++qbad_big;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    n += __shfl_xor_sync(0xffffffffu, n, o);
    qbad_big += __shfl_xor_sync(0xffffffffu, qbad_big, o);
    qbad += __shfl_xor_sync(0xffffffffu, qbad, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(counts + 0, bad);
    atomicAdd(counts + 1, n);
    atomicAdd(counts + 2, qbad_big);
    atomicAdd(counts + 3, qbad);
  }
}

// Block scales: scale_of_amax(amax) against __fdiv_rn(amax, 448) for every positive finite
// BF16 amax. counts[0] = bit mismatches, counts[1] = values checked.
__global__ void k_scale_check(unsigned long long *counts, unsigned int *first_bad) {
  const uint32_t amax_bits = blockIdx.x * blockDim.x + threadIdx.x + 1;  // 0x0001 ..
  unsigned long long bad = 0, n = 0;
  if (amax_bits <= 0x7F7Fu) {
    const float amax = __uint_as_float(amax_bits << 16);
    ++n;
    float s_fast;
    puro::BlockDivider d;
    bool ok;
    puro::block_scale_fast(amax, s_fast, d, ok);
    const uint32_t want = __float_as_uint(__fdiv_rn(amax, 448.0f));
    if (__float_as_uint(puro::scale_of_amax(amax)) != want ||
        (ok && __float_as_uint(s_fast) != want)) {
      ++bad;
      atomicCAS(first_bad, 0u, amax_bits);
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    n += __shfl_xor_sync(0xffffffffu, n, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(counts + 0, bad);
    atomicAdd(counts + 1, n);
  }
}

// The branch-free reciprocal against __frcp_rn for every FP32 s in [2^-90, 2^120], and the
// all-zero block's divider on signed zeros. counts[0] = reciprocal mismatches, counts[1] =
// values checked, counts[2] = zero-block failures.
__global__ void k_rcp_check(unsigned long long *counts, unsigned int *first_bad) {
  constexpr uint32_t lo = 0x12800000u, hi = 0x7B800000u;  // 2^-90, 2^120
  unsigned long long bad = 0, n = 0;
  for (uint32_t b = lo + blockIdx.x * blockDim.x + threadIdx.x; b <= hi && b >= lo;
       b += gridDim.x * blockDim.x) {
    const float s = __uint_as_float(b);
    ++n;
    if (__float_as_uint(puro::rcp_rn_fast(s)) != __float_as_uint(__frcp_rn(s))) {
      ++bad;
      atomicCAS(first_bad, 0u, b);
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    n += __shfl_xor_sync(0xffffffffu, n, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(counts + 0, bad);
    atomicAdd(counts + 1, n);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    // +0, -0, -0, +0 through the zero block's divider, the general and the fast helper,
    // and the branch-free scale of amax = 0
    const uint32_t w0 = 0x80000000u, w1 = 0x00008000u;
    const puro::BlockDivider z = puro::zero_block_divider();
    float s0;
    puro::BlockDivider d0;
    bool ok0;
    puro::block_scale_fast(0.0f, s0, d0, ok0);
    const bool good = puro::block_codes4(w0, w1, z) == 0x00808000u &&
                      puro::block_codes4(w0, w1, d0) == 0x00808000u && ok0 &&
                      __float_as_uint(s0) == 0u && z.fast;
    if (!good) atomicAdd(counts + 2, 1ull);
  }
}

}  // namespace

extern "C" int run_scale_check(unsigned long long *host_counts, unsigned int *host_first_bad) {
  unsigned long long *counts = nullptr;
  unsigned int *first = nullptr;
  if (cudaMalloc(&counts, 2 * sizeof(unsigned long long)) != cudaSuccess) return 1;
  if (cudaMalloc(&first, sizeof(unsigned int)) != cudaSuccess) return 2;
  cudaMemset(counts, 0, 2 * sizeof(unsigned long long));
  cudaMemset(first, 0, sizeof(unsigned int));
  k_scale_check<<<(0x7F7F + 255) / 256, 256>>>(counts, first);
  if (cudaGetLastError() != cudaSuccess) return 3;
  if (cudaMemcpy(host_counts, counts, 2 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return 4;
  cudaMemcpy(host_first_bad, first, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaFree(counts);
  cudaFree(first);
  return 0;
}

extern "C" int run_division_check(unsigned long long *host_counts, unsigned int *host_first_bad) {
  unsigned long long *counts = nullptr;
  unsigned int *first = nullptr;
  if (cudaMalloc(&counts, 4 * sizeof(unsigned long long)) != cudaSuccess) return 1;
  if (cudaMalloc(&first, sizeof(unsigned int)) != cudaSuccess) return 2;
  cudaMemset(counts, 0, 4 * sizeof(unsigned long long));
  cudaMemset(first, 0, sizeof(unsigned int));
  k_check<<<dim3(0x7F7F, 16), 256>>>(counts, first);
  if (cudaGetLastError() != cudaSuccess) return 3;
  if (cudaMemcpy(host_counts, counts, 4 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return 4;
  cudaMemcpy(host_first_bad, first, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaFree(counts);
  cudaFree(first);
  return 0;
}

extern "C" int run_rcp_check(unsigned long long *host_counts, unsigned int *host_first_bad) {
  unsigned long long *counts = nullptr;
  unsigned int *first = nullptr;
  if (cudaMalloc(&counts, 3 * sizeof(unsigned long long)) != cudaSuccess) return 1;
  if (cudaMalloc(&first, sizeof(unsigned int)) != cudaSuccess) return 2;
  cudaMemset(counts, 0, 3 * sizeof(unsigned long long));
  cudaMemset(first, 0, sizeof(unsigned int));
  k_rcp_check<<<148 * 16, 256>>>(counts, first);
  if (cudaGetLastError() != cudaSuccess) return 3;
  if (cudaMemcpy(host_counts, counts, 3 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return 4;
  cudaMemcpy(host_first_bad, first, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaFree(counts);
  cudaFree(first);
  return 0;
}
