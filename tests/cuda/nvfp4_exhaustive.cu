// Test-only kernels: the NVFP4 quantisers' group arithmetic (fp8_blockwise_scaled_e4m3_b200/
// csrc/nvfp4_math.cuh) against IEEE division, over every case the quantisers can meet.
//
// Factors: for every positive finite BF16 tensor amax a_t (s_t = RN(a_t / 2688)) and every BF16
// group amax a_g <= a_t, the factor byte E4M3_RNE_sat(RN(RN(a_g / 6) / s_t)) and its decoded
// scale S = RN(dec(e) * s_t), with the divisions done by __fdiv_rn and the decode by CUDA's
// E4M3 conversion; where the tensor takes the all-fast path (s_t >= 2^-81), that path's factor too.
// counts: [0] mismatches, [1] pairs checked, [2] pairs checked on the all-fast path.
//
// Codes: for every positive finite BF16 a_t and every factor byte e (0 .. 0x7E), the scale
// S = RN(dec(e) * s_t), and every BF16 x of either sign with S / 32 <= |x| <= 16 S (every value
// a group with this factor can hold lies below 6.4 S; below S / 32 the code is a signed zero,
// checked on the smallest values and zero), the E2M1 codes of RN(x / S) (__fdiv_rn; signed
// zeros when S == 0, where x runs over every finite BF16) against the kernels' packed helpers.
// counts: [0] mismatches, [1] values checked.
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../fp8_blockwise_scaled_e4m3_b200/csrc/nvfp4_math.cuh"

using puro::pack2;

namespace {

__device__ __forceinline__ float dec_e4m3(uint32_t b) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ uint32_t e4m3_of(float v) {
  return __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ void flush(unsigned long long *counts, unsigned long long bad, unsigned long long n,
                                      unsigned long long n2 = 0) {
  for (int o = 16; o > 0; o >>= 1) {
    bad += __shfl_xor_sync(0xffffffffu, bad, o);
    n += __shfl_xor_sync(0xffffffffu, n, o);
    n2 += __shfl_xor_sync(0xffffffffu, n2, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(counts + 0, bad);
    atomicAdd(counts + 1, n);
    atomicAdd(counts + 2, n2);
  }
}

__global__ void k_factor_check(unsigned long long *counts, unsigned int *first_bad) {
  const uint32_t tb = blockIdx.x + 1;  // tensor amax bits 0x0001 .. 0x7F7F
  const float amax_t = __uint_as_float(tb << 16);
  const float s_t = __fdiv_rn(amax_t, 2688.0f);
  const puro::NvTensor t = puro::nv_tensor(amax_t);
  unsigned long long bad = 0, n = 0, n2 = 0;
  if (threadIdx.x == 0 && __float_as_uint(t.s_t) != __float_as_uint(s_t)) {
    ++bad;
    atomicCAS(first_bad, 0u, tb << 16);
  }
  if (blockIdx.x == 0 && threadIdx.x < 127 &&
      __float_as_uint(puro::ue4m3_value(threadIdx.x)) != __float_as_uint(dec_e4m3(threadIdx.x))) {
    ++bad;
    atomicCAS(first_bad, 0u, 0xFF000000u | threadIdx.x);
  }
  for (uint32_t gb = threadIdx.x; gb <= tb; gb += blockDim.x) {
    const float amax_g = __uint_as_float(gb << 16);
    ++n;
    const uint32_t e_ref = e4m3_of(__fdiv_rn(__fdiv_rn(amax_g, 6.0f), s_t));
    const float S_ref = __fmul_rn(dec_e4m3(e_ref), s_t);
    float S;
    const uint32_t e = puro::nv_factor(amax_g, t, S);
    bool good = e == e_ref && __float_as_uint(S) == __float_as_uint(S_ref);
    if (t.all_fast) {
      ++n2;
      float S2;
      const uint32_t e2 = puro::nv_factor<true>(amax_g, t, S2);
      good = good && e2 == e_ref && __float_as_uint(S2) == __float_as_uint(S_ref);
    }
    if (!good) {
      ++bad;
      atomicCAS(first_bad, 0u, (tb << 16) | gb);
    }
  }
  flush(counts, bad, n, n2);
}

// one value x (bits xb): its code by IEEE division, and by the kernels' helpers for eight
// values of a row (both halves of a word) and of a column (one half of each word)
__device__ __forceinline__ bool codes_agree(uint32_t xb, float S, const puro::NvDivider &d) {
  const float x = __uint_as_float(xb << 16);
  const float q = S == 0.0f ? x * 0.0f : __fdiv_rn(x, S);
  const uint32_t want = puro::e2m1x2(q, q) * 0x01010101u;
  const uint32_t w = xb | (xb << 16);
  const uint4 w4 = make_uint4(w, w, w, w);
  uint32_t row, lo, hi;
  if (d.fast) {
    const uint64_t n = pack2(puro::neg_bf16_lo(w), puro::neg_bf16_hi(w));
    const uint64_t nl = pack2(puro::neg_bf16_lo(w), puro::neg_bf16_lo(w));
    const uint64_t nh = pack2(puro::neg_bf16_hi(w), puro::neg_bf16_hi(w));
    row = puro::nv_codes8_fast(n, n, n, n, d);
    lo = puro::nv_codes8_fast(nl, nl, nl, nl, d);
    hi = puro::nv_codes8_fast(nh, nh, nh, nh, d);
  } else {
    row = puro::nv_codes8_exact(w4, w4, true, false, S);
    lo = puro::nv_codes8_exact(w4, w4, false, false, S);
    hi = puro::nv_codes8_exact(w4, w4, false, true, S);
  }
  return row == want && lo == want && hi == want;
}

__global__ void k_codes_check(unsigned long long *counts, unsigned int *first_bad) {
  const uint32_t tb = blockIdx.x + 1;
  const uint32_t e = blockIdx.y;  // factor byte 0 .. 0x7E
  const float s_t = __fdiv_rn(__uint_as_float(tb << 16), 2688.0f);
  const float S = __fmul_rn(dec_e4m3(e), s_t);
  const puro::NvDivider d = puro::nv_divider(S);
  unsigned long long bad = 0, n = 0;
  uint32_t lo = 0, hi = 0;
  if (S == 0.0f) {
    if (tb != 1) return;  // the same divider for every tensor: check it once
    hi = 0x7F7F;
  } else {
    lo = __float_as_uint(__fmul_rn(S, 0x1p-5f)) >> 16;
    const float top = __fmul_rn(S, 16.0f);
    hi = top > 3.0e38f ? 0x7F7Fu : min(0x7F7Fu, (__float_as_uint(top) >> 16) + 1);
  }
  for (uint32_t xb = lo + threadIdx.x; xb <= hi; xb += blockDim.x)
    for (uint32_t sign = 0; sign <= 0x8000u; sign += 0x8000u) {
      ++n;
      if (!codes_agree(xb | sign, S, d)) {
        ++bad;
        atomicCAS(first_bad, 0u, (tb << 16) | xb | sign);
      }
    }
  if (threadIdx.x < 4 && lo > 1) {  // zero and the smallest subnormal, both signs
    const uint32_t xb = (threadIdx.x & 1) | ((threadIdx.x & 2) ? 0x8000u : 0u);
    ++n;
    if (!codes_agree(xb, S, d)) {
      ++bad;
      atomicCAS(first_bad, 0u, (tb << 16) | xb);
    }
  }
  flush(counts, bad, n);
}

int run(void (*launch)(unsigned long long *, unsigned int *), unsigned long long *host_counts,
        unsigned int *host_first_bad) {
  unsigned long long *counts = nullptr;
  unsigned int *first = nullptr;
  if (cudaMalloc(&counts, 3 * sizeof(unsigned long long)) != cudaSuccess) return 1;
  if (cudaMalloc(&first, sizeof(unsigned int)) != cudaSuccess) return 2;
  cudaMemset(counts, 0, 3 * sizeof(unsigned long long));
  cudaMemset(first, 0, sizeof(unsigned int));
  launch(counts, first);
  if (cudaGetLastError() != cudaSuccess) return 3;
  if (cudaMemcpy(host_counts, counts, 3 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return 4;
  cudaMemcpy(host_first_bad, first, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  cudaFree(counts);
  cudaFree(first);
  return 0;
}

}  // namespace

extern "C" int run_nvfp4_factor_check(unsigned long long *host_counts, unsigned int *host_first_bad) {
  return run([](unsigned long long *c, unsigned int *f) { k_factor_check<<<0x7F7F, 256>>>(c, f); }, host_counts,
             host_first_bad);
}

extern "C" int run_nvfp4_codes_check(unsigned long long *host_counts, unsigned int *host_first_bad) {
  return run([](unsigned long long *c, unsigned int *f) { k_codes_check<<<dim3(0x7F7F, 0x7F), 256>>>(c, f); },
             host_counts, host_first_bad);
}
