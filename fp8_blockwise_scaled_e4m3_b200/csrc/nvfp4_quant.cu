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
// (the arithmetic, and how it stays correctly rounded, is in nvfp4_math.cuh). Two codes per
// byte (element 2i in the low nibble). Factors are stored by 256-element K block: F[b][r][j]
// (16 bytes per row and block) is the factor of X[r, 256 b + 16 j ..], so the GEMM reads a K
// block's factors of consecutive rows as one contiguous run. The tensor amax is an output of
// its own kernel, read by the quantising kernel from device memory, so the two launches need no
// host round trip. Inputs must be finite.
//
//   k_nv_amax        max |x| over X [R, C]: a warp per row (or row segment, when rows are too few
//                    to fill the GPU), four 16-byte loads in flight per lane, a block maximum,
//                    then one atomicMax per block on the FP32 bit pattern (non-negative floats
//                    order like their bit patterns); the word starts at zero
//   k_nv_quant_rows  one thread per 16-element group along the columns: 32-byte loads, one
//                    8-byte store of codes and one factor byte, consecutive threads on
//                    consecutive groups of a row (16 consecutive factor bytes per K block)
//   k_nv_quant_cols  groups of 16 consecutive rows, written transposed: a thread takes two
//                    adjacent columns over 64 rows (4-byte loads, a warp reads 128 contiguous
//                    bytes of each row) and writes 32 bytes of codes and 4 factor bytes (one
//                    4-byte store into its K block's 16) per column
//   k_nv_quant_dual  both of the above from one read of X: persistent CTAs take 128 x 128 tiles
//                    through a two-stage TMA ring (two 128-byte-swizzled boxes of 64 columns per
//                    tile); a thread quantises 64 elements of one row, then two columns over 32
//                    rows, both from shared memory without bank conflicts; the transposed codes
//                    leave through a staging buffer as whole 64-byte rows

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>

#include "../../include/puro_fp8.h"
#include "host_cache.h"
#include "quant.h"
#include "nvfp4_math.cuh"
#include "ptx.cuh"
#include "quant_math.cuh"

namespace puro {
namespace {

constexpr int kThreads = 256;

// A warp takes `segs` consecutive work items, each one segment of one row (a row is split into
// `segs` segments of `seg_chunks` 16-byte chunks when there are too few rows to occupy the GPU);
// a lane keeps four 16-byte loads in flight. One atomicMax per block.
__global__ void __launch_bounds__(kThreads) k_nv_amax(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t ldx,
                                                      int segs, int seg_chunks, uint32_t *amax_bits) {
  __shared__ uint32_t part[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cpr = static_cast<int>(C / 8);  // 16-byte chunks of 8 BF16 per row
  const int64_t items = R * segs;
  uint32_t m2 = 0;  // per-half magnitude maximum (sign bits meaningless until masked)
  for (int64_t it = blockIdx.x * static_cast<int64_t>(kThreads / 32) + warp; it < items;
       it += static_cast<int64_t>(gridDim.x) * (kThreads / 32)) {
    const int64_t r = it / segs;
    const int seg = static_cast<int>(it - r * segs);
    const uint4 *row = reinterpret_cast<const uint4 *>(X + r * ldx);
    const int end = min(cpr, (seg + 1) * seg_chunks);
    int c = seg * seg_chunks + lane;
    for (; c + 96 < end; c += 128) {
      const uint4 v0 = __ldg(row + c), v1 = __ldg(row + c + 32), v2 = __ldg(row + c + 64), v3 = __ldg(row + c + 96);
      m2 = bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w)));
      m2 = bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
      m2 = bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v2.x, v2.y), bf16x2_absmax(v2.z, v2.w)));
      m2 = bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v3.x, v3.y), bf16x2_absmax(v3.z, v3.w)));
    }
    for (; c < end; c += 32) {
      const uint4 v = __ldg(row + c);
      m2 = bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w)));
    }
  }
  m2 &= 0x7FFF7FFFu;
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) part[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < kThreads / 32 ? part[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m != 0) atomicMax(amax_bits, m << 16);
  }
}

__global__ void __launch_bounds__(kThreads) k_nv_quant_rows(const uint16_t *__restrict__ X, int64_t R, int64_t C,
                                                            int64_t ldx, uint8_t *__restrict__ Xq, int64_t ldq,
                                                            uint8_t *__restrict__ F, const float *amax_t) {
  const NvTensor t = nv_tensor(*amax_t);
  const int64_t groups_per_row = C / 16;
  const int64_t total = R * groups_per_row;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = g / groups_per_row, j = g - r * groups_per_row;
    const uint4 *src = reinterpret_cast<const uint4 *>(X + r * ldx + 16 * j);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    uint2 out;
    const uint32_t e = nv_row_group(v0, v1, t, out.x, out.y);
    *reinterpret_cast<uint2 *>(Xq + r * ldq + 8 * j) = out;
    F[((j >> 4) * R + r) * 16 + (j & 15)] = static_cast<uint8_t>(e);
  }
}

// X [R, C] -> XqT [C, R/2] (row stride ldq bytes), FT [R/256 (rounded up)][C][16]; R % 64 == 0,
// C % 2 == 0.
__global__ void __launch_bounds__(kThreads) k_nv_quant_cols(const uint16_t *__restrict__ X, int64_t R, int64_t C,
                                                            int64_t ldx, uint8_t *__restrict__ XqT, int64_t ldq,
                                                            uint8_t *__restrict__ FT, const float *amax_t) {
  const NvTensor t = nv_tensor(*amax_t);
  const int64_t pairs = C / 2, slabs = R / 64;
  const int64_t total = pairs * slabs;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t slab = u / pairs, c0 = 2 * (u - slab * pairs), r0 = 64 * slab;
    const uint32_t *src = reinterpret_cast<const uint32_t *>(X + r0 * ldx + c0);
    const int64_t step = ldx / 2;  // 4-byte words per row
    uint32_t w[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) w[i] = __ldg(src + i * step);
    uint32_t m2[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) m2[g] = nv_absmax16(w + 16 * g);
#pragma unroll
    for (int col = 0; col < 2; ++col) {
      uint32_t fac = 0;
      uint32_t out[8];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t e = col ? nv_col_group<true>(w + 16 * g, m2[g], t, out[2 * g], out[2 * g + 1])
                               : nv_col_group<false>(w + 16 * g, m2[g], t, out[2 * g], out[2 * g + 1]);
        fac |= e << (8 * g);
      }
      uint8_t *dst = XqT + (c0 + col) * ldq + r0 / 2;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
      *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(out[4], out[5], out[6], out[7]);
      // groups 4 slab .. 4 slab + 3 of column c0 + col: K block slab / 4, bytes 4 (slab % 4) ..
      *reinterpret_cast<uint32_t *>(FT + ((slab >> 2) * C + (c0 + col)) * 16 + 4 * (slab & 3)) = fac;
    }
  }
}

// ---------------------------------------------------------------- both layouts, one read

#ifdef PURO_TEST_HOOKS
// Test builds only, never libpuro_fp8.so: while set, each CTA of the dual kernel skips the load
// of its first tile, so the bounded wait for it runs out. The failure-detection test uses this
// to check that the give-up reaches the status word and that the kernel drains and exits with
// the context intact.
__device__ int g_test_nv_skip_load;
#define PURO_NV_SKIP_LOAD(i) (g_test_nv_skip_load != 0 && (i) == 0)
#else
#define PURO_NV_SKIP_LOAD(i) false
#endif

constexpr int kDualTile = 128;                  // rows and columns of a tile
constexpr int kDualBox = kDualTile * 128;       // one TMA box: 128 rows x 64 BF16 (128 bytes)
constexpr int kDualStage = 2 * kDualBox;        // one tile, 32 KB
constexpr int kDualStages = 2;
constexpr int kDualCtas = 3;                    // CTAs per SM
constexpr int kDualStg = 8192 + 1024;           // staging of a tile's transposed codes and factors
constexpr int kDualSmem = kDualStages * kDualStage + kDualStg + 1024 + 64;  // + alignment, barriers, flag

// The four groups of 64 elements of a row held in v[0..7]: their codes in o, their factors as
// the bytes of the result.
template <bool ALL_FAST>
__device__ __forceinline__ uint32_t dual_row_codes(const uint4 (&v)[8], const NvTensor &t, uint32_t (&o)[8]) {
  uint32_t fac = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) fac |= nv_row_group<ALL_FAST>(v[2 * j], v[2 * j + 1], t, o[2 * j], o[2 * j + 1]) << (8 * j);
  return fac;
}

// The two 16-row groups of column `col` of a column pair held in w[0..31] (m0, m1: their
// per-half maxima): codes in o, factors e0, e1.
template <bool ALL_FAST, bool HI>
__device__ __forceinline__ void dual_col_codes(const uint32_t (&w)[32], uint32_t m0, uint32_t m1, const NvTensor &t,
                                               uint32_t (&o)[4], uint32_t &e0, uint32_t &e1) {
  e0 = nv_col_group<HI, ALL_FAST>(w, m0, t, o[0], o[1]);
  e1 = nv_col_group<HI, ALL_FAST>(w + 16, m1, t, o[2], o[3]);
}

struct NvDualArgs {
  int64_t R, C, ldq, ldqt;
  uint8_t *Xq, *F, *XqT, *FT;
  const float *amax;
  int tiles, tiles_c;
  unsigned long long timeout_ns;
  int *status;
};

// Tile t of CTA b is global tile b + t * gridDim.x, in stage t % kDualStages. Thread 0 loads
// tiles ahead through the ring; every thread waits (bounded) for the tile's barrier, then
//  - rows: thread (row = tid % 128, half = tid / 128) quantises the 64 elements of its row in
//    box `half` (four groups): eight 16-byte shared loads of chunk k at k ^ (row % 8), so the
//    eight rows of a quarter warp hit eight different bank groups; 32 bytes of codes and 4
//    factor bytes (one K block's bytes 4 m .. 4 m + 3) per thread;
//  - columns: thread (pair p = tid % 64, quarter = tid / 64) reads the 4-byte word of columns
//    2p, 2p + 1 from the 32 rows of its quarter (a warp reads the 32 words of one row), takes
//    both columns' group maxima with packed BF16 maxima, and forms 16 bytes of codes and 2
//    factor bytes per column, written into a staging buffer (8 KB of codes, 1 KB of factors);
//    after a CTA sync they leave it as whole 64-byte rows of XqT and 8-byte runs of FT, instead
//    of one partial sector per thread and column;
// then the CTA syncs (the stage and the staging buffer are free) and thread 0 refills the stage.
__global__ void __launch_bounds__(kThreads, kDualCtas)
    k_nv_quant_dual(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ NvDualArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t *stg = smem + kDualStages * kDualStage;
  const uint32_t bar0 = sbase + kDualStages * kDualStage + kDualStg;
  volatile int *fail = reinterpret_cast<volatile int *>(smem + kDualStages * kDualStage + kDualStg + 8 * kDualStages);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kDualStages; ++s) mbar_init(bar0 + 8 * s, 1);
    *fail = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmX);
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int tile = blockIdx.x + i * gridDim.x;
    if (tile >= a.tiles || PURO_NV_SKIP_LOAD(i)) return;
    const int tr = tile / a.tiles_c, tc = tile - tr * a.tiles_c;
    const uint32_t bar = bar0 + 8 * (i % kDualStages), dst = sbase + (i % kDualStages) * kDualStage;
    mbar_arrive_expect_tx(bar, kDualStage);
    tma_load_2d(dst, &tmX, bar, tc * kDualTile, tr * kDualTile);
    tma_load_2d(dst + kDualBox, &tmX, bar, tc * kDualTile + 64, tr * kDualTile);
  };
  if (tid == 0)
    for (int i = 0; i < kDualStages; ++i) issue(i);

  const NvTensor t = nv_tensor(*a.amax);
  const int row = tid & 127, half = tid >> 7;
  const int p = tid & 63, quarter = tid >> 6;
  int i = 0;
  for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++i) {
    const int s = i % kDualStages;
    const bool waited = mbar_wait(bar0 + 8 * s, (i / kDualStages) & 1, a.timeout_ns, fail);
    if (__syncthreads_or(!waited)) {
      if (tid == 0) {
        *fail = 1;
        atomicOr(a.status, 1);
      }
      break;
    }
    const int tr = tile / a.tiles_c, tc = tile - tr * a.tiles_c;
    const int64_t r0 = static_cast<int64_t>(tr) * kDualTile, c0 = static_cast<int64_t>(tc) * kDualTile;
    const uint8_t *stage = smem + s * kDualStage;

    // ---- along the rows
    {
      const int64_t gr = r0 + row, cb = c0 + 64 * half;
      if (gr < a.R && cb < a.C) {
        const uint8_t *rp = stage + half * kDualBox + row * 128;
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = *reinterpret_cast<const uint4 *>(rp + ((k ^ (row & 7)) << 4));
        uint32_t o[8];
        // one branch per tile phase, uniform over the grid: the tensor decides the path
        const uint32_t fac = t.all_fast ? dual_row_codes<true>(v, t, o) : dual_row_codes<false>(v, t, o);
        uint8_t *dq = a.Xq + gr * a.ldq + cb / 2;
        uint8_t *df = a.F + ((cb >> 8) * a.R + gr) * 16 + ((cb >> 4) & 15);
        if (cb + 64 <= a.C) {
          if ((reinterpret_cast<uintptr_t>(dq) & 15) == 0) {
            *reinterpret_cast<uint4 *>(dq) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(dq + 16) = make_uint4(o[4], o[5], o[6], o[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) *reinterpret_cast<uint2 *>(dq + 8 * j) = make_uint2(o[2 * j], o[2 * j + 1]);
          }
          *reinterpret_cast<uint32_t *>(df) = fac;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (cb + 16 * j < a.C) {
              *reinterpret_cast<uint2 *>(dq + 8 * j) = make_uint2(o[2 * j], o[2 * j + 1]);
              df[j] = static_cast<uint8_t>(fac >> (8 * j));
            }
        }
      }
    }

    // ---- down the columns, staged
    {
      const int64_t c = c0 + 2 * p, rq = r0 + 32 * quarter;
      if (c < a.C && rq < a.R) {
        const int k = (p & 31) >> 2;
        const uint8_t *bp = stage + (p >> 5) * kDualBox + quarter * 32 * 128 + ((p & 3) << 2);
        uint32_t w[32];
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) w[ii] = *reinterpret_cast<const uint32_t *>(bp + ii * 128 + ((k ^ (ii & 7)) << 4));
        const uint32_t m0 = nv_absmax16(w), m1 = nv_absmax16(w + 16);
#pragma unroll
        for (int col = 0; col < 2; ++col) {
          uint32_t o[4], e0, e1;
          if (t.all_fast) {
            if (col) dual_col_codes<true, true>(w, m0, m1, t, o, e0, e1);
            else dual_col_codes<true, false>(w, m0, m1, t, o, e0, e1);
          } else {
            if (col) dual_col_codes<false, true>(w, m0, m1, t, o, e0, e1);
            else dual_col_codes<false, false>(w, m0, m1, t, o, e0, e1);
          }
          // codes of column 2p + col, rows 32 quarter .. + 31: 16-byte chunk 4 col + quarter of
          // staging pair-row p (columns 2p, 2p + 1), XOR-swizzled by p so that the eight
          // threads of a quarter warp write eight different bank groups
          *reinterpret_cast<uint4 *>(stg + p * 128 + (((4 * col + quarter) ^ (p & 7)) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint16_t *>(stg + 8192 + (2 * p + col) * 8 + 2 * quarter) =
              static_cast<uint16_t>(e0 | (e1 << 8));
        }
      }
    }
    __syncthreads();
    // copy-out: each column's 64 bytes of codes as four 16-byte stores (a warp writes 8 full
    // 64-byte row segments of XqT), its 8 factor bytes as one 8-byte store
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int u = tid + kThreads * h, r = u >> 2, j = u & 3;
      if (c0 + r < a.C && r0 + 32 * j < a.R)
        *reinterpret_cast<uint4 *>(a.XqT + (c0 + r) * a.ldqt + r0 / 2 + 16 * j) =
            *reinterpret_cast<const uint4 *>(stg + (r >> 1) * 128 + (((4 * (r & 1) + j) ^ ((r >> 1) & 7)) << 4));
    }
    if (tid < kDualTile && c0 + tid < a.C) {
      // groups r0/16 .. r0/16 + 7 of column c0 + tid: K block r0 / 256, bytes 8 (tr % 2) ..
      uint8_t *df = a.FT + ((r0 >> 8) * a.C + c0 + tid) * 16 + ((r0 >> 4) & 15);
      const uint2 f = *reinterpret_cast<const uint2 *>(stg + 8192 + tid * 8);
      if (r0 + kDualTile <= a.R)
        *reinterpret_cast<uint2 *>(df) = f;
      else  // 64 rows left: their four groups only
        *reinterpret_cast<uint32_t *>(df) = f.x;
    }
    __syncthreads();  // the stage is consumed
    if (tid == 0) issue(i + kDualStages);
  }
  if (tid == 0 && *fail) {
    // let the loads still in flight land before the CTA exits (bounded)
    for (int k = 0; k < kDualStages; ++k) {
      const int ii = i + k;
      if (blockIdx.x + ii * gridDim.x < a.tiles)
        mbar_wait(bar0 + 8 * (ii % kDualStages), (ii / kDualStages) & 1, a.timeout_ns, nullptr);
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
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  // enough warps to fill every SM (64 warps each); a segment keeps at least one batch of four
  // loads per lane
  const int64_t cpr = C / 8, want = static_cast<int64_t>(sms) * 64;
  const int64_t max_segs = cpr / 128 > 1 ? cpr / 128 : 1;
  int64_t segs = (want + R - 1) / R;
  segs = segs < 1 ? 1 : (segs > max_segs ? max_segs : segs);
  const int64_t seg_chunks = (cpr + segs - 1) / segs;
  const int64_t blocks = (R * segs + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const int grid = static_cast<int>(blocks < cap ? blocks : cap);
  k_nv_amax<<<grid, kThreads, 0, stream>>>(X, R, C, ldx, static_cast<int>(segs), static_cast<int>(seg_chunks),
                                           reinterpret_cast<uint32_t *>(amax));
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

int launch_nvfp4_quant_dual(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq, int64_t ldq,
                            uint8_t *F, uint8_t *XqT, int64_t ldqt, uint8_t *FT, float *amax,
                            cudaStream_t stream) {
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  static PerDevice<bool> smem_opt_in;  // dynamic shared memory opted in once per device
  bool ok = false;
  if (!smem_opt_in.get(ok, [](int, bool &v) {
        v = cudaFuncSetAttribute(k_nv_quant_dual, cudaFuncAttributeMaxDynamicSharedMemorySize, kDualSmem) ==
            cudaSuccess;
        return v;
      }))
    return PURO_ERR_CUDA;
  NvDualArgs args{};
  args.R = R;
  args.C = C;
  args.ldq = ldq;
  args.ldqt = ldqt;
  args.Xq = Xq;
  args.F = F;
  args.XqT = XqT;
  args.FT = FT;
  args.amax = amax;
  args.tiles_c = static_cast<int>((C + kDualTile - 1) / kDualTile);
  args.tiles = static_cast<int>(((R + kDualTile - 1) / kDualTile) * args.tiles_c);
  args.timeout_ns = nv_wait_timeout_ns();
  args.status = nv_status_word();
  if (args.status == nullptr) return PURO_ERR_CUDA;
  CUtensorMap tmX;
  if (!nv_bf16_map(&tmX, X, R, C, ldx, kDualTile)) return PURO_ERR_CUDA;
  const int rc = launch_amax(X, R, C, ldx, amax, stream);
  if (rc != PURO_OK) return rc;
  const int grid = args.tiles < kDualCtas * sms ? args.tiles : kDualCtas * sms;
  k_nv_quant_dual<<<grid, kThreads, kDualSmem, stream>>>(tmX, args);
  return cudaGetLastError() == cudaSuccess ? PURO_OK : PURO_ERR_LAUNCH;
}

}  // namespace puro

#ifdef PURO_TEST_HOOKS
extern "C" __attribute__((visibility("default"))) int puro_test_set_nv_skip_load(int on) {
  return cudaMemcpyToSymbol(puro::g_test_nv_skip_load, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
