// Blockwise BF16 -> E4M3 quantisers (memory-bound), sm_100a.
//
// "Paper walkthrough: Puro-2B ...", section "Lever 2: use blockwise FP8 from step zero":
// activations and their gradients get one scale per 128 elements along the reduction
// dimension, weights one scale per 128x128 block. Per block, in FP32:
//   amax = max|x|;  s = amax / 448 (IEEE division);  q = E4M3_rn_satfinite(x / s)
// and an all-zero block stores s = 0 with signed-zero codes (x / 1 keeps the sign).
//
// One persistent kernel serves every quantiser; it walks 128 x 128 BF16 tiles of the
// input X [R, C] (row stride ldx):
//   Q_ROWS    1x128 groups along the columns:   Xq [R, C] (row stride ldq), S [C/128][R]
//   Q_COLS    1x128 groups along the rows, transposed: XqT [C, R], ST [R/128][C]
//   Q_DUAL    both of the above from one read of X
//   Q_WEIGHT  one group per 128x128 tile:        Wq [R, C], S [ceil(R/128)][C/128],
//             and optionally the same codes transposed, WqT [C, R]
// Tiles arrive by TMA (two 64-column boxes with the 128-byte swizzle) into a 2-stage
// mbarrier ring of shared memory per CTA (two CTAs per SM), so the next tiles are in
// flight while the current one is computed and nothing in flight occupies registers.
// Row-wise codes leave with coalesced 8-byte stores; transposed codes are assembled in a
// swizzled shared tile and written by one TMA tensor store. TMA zero-fills reads past the
// edge (no effect on amax) and clips writes past it. Every wait is bounded.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "../../include/puro_fp8.h"
#include "host_cache.h"
#include "ptx.cuh"
#include "quant.h"
#include "quant_math.cuh"

namespace puro {
namespace {

enum QMode { Q_ROWS = 1, Q_COLS = 2, Q_DUAL = 3, Q_WEIGHT = 4 };

constexpr int kTile = 128;
// Two CTAs per SM, each with its own 2-stage ring: the phases of one CTA's tile are
// separated by CTA barriers, and the other CTA's work fills the SM while they drain.
// Threads per CTA: the register budget (64K per SM, two CTAs) sets the count per mode.
template <int MODE>
struct Threads {
  static constexpr int value = MODE == 1 ? 512 : 256;
};
constexpr int kStages = 2;
constexpr int kCtasPerSm = 2;
constexpr int kBoxBytes = kTile * 128;         // 128 rows x 64 BF16 (128 bytes), swizzled
constexpr int kStageBytes = 2 * kBoxBytes;     // one 128 x 128 BF16 tile
constexpr int kOffCodes = kStages * kStageBytes;
constexpr int kOffPart = kOffCodes + kTile * kTile;  // 128 x 128 code tile, swizzled
constexpr int kOffWarpMax = kOffPart + 16 * kTile * 4;   // up to 16 token groups
constexpr int kOffColDiv = kOffWarpMax + 32 * 4;     // per tile column: divisor s, 1/s
constexpr int kOffBar = kOffColDiv + kTile * 8;
constexpr int kOffMisc = kOffBar + 8 * kStages;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

struct QArgs {
  int64_t R, C;
  uint8_t *q;        // row-wise codes (Q_ROWS, Q_DUAL) or Wq (Q_WEIGHT)
  int64_t ldq;
  float *s;          // S of the row-wise groups, or of the weight blocks
  float *st;         // ST of the transposed groups (Q_COLS, Q_DUAL)
  int write_t;       // Q_WEIGHT: also write WqT through the transposed store
  uint8_t *sb;       // P2: UE8M0 scale bytes in place of s
  uint8_t *stb;      // P2: UE8M0 scale bytes in place of st
  int tiles_r, tiles_c;
  int tile_begin;    // first tile of this problem in the launch's joint tile sequence
  unsigned long long timeout_ns;
  int *status;
};

// Kernel parameters: G problems of the same mode (G = 1 for the single-tensor entry
// points), their tensor maps and arguments passed by value as a __grid_constant__ (the
// TMA unit reads the maps from the parameter space). Problem p owns tiles
// [args[p].tile_begin, args[p].tile_begin + tiles_r * tiles_c) of the joint sequence.
template <int G>
struct alignas(64) QParams {
  CUtensorMap tmX[G];
  CUtensorMap tmT[G];
  QArgs args[G];
  int count;
  int tiles;
};
constexpr int QGROUP_MAX = 64;  // weights per grouped launch (parameter space: 32 KB)
static_assert(sizeof(QParams<QGROUP_MAX>) <= 32000, "kernel parameter space");

// The problem that owns `tile`, searched forward from p (a CTA's tiles only increase).
template <int G>
__device__ __forceinline__ int problem_of(const QParams<G> &prm, int p, int tile) {
  if constexpr (G == 1) {
    return 0;
  } else {
    while (p + 1 < prm.count && tile >= prm.args[p + 1].tile_begin) ++p;
    return p;
  }
}

__device__ int g_quant_status;  // non-zero: a bounded wait gave up since the last read

#ifdef PURO_TEST_HOOKS
// Test builds only, never libpuro_fp8.so: while set, each CTA skips the load of its first
// tile, so the bounded wait for that tile runs out. The failure-detection test uses this to
// check that a give-up inside the quantiser reaches the status word and that the kernel
// drains and exits with the context intact.
__device__ int g_test_quant_skip_load;
#define PURO_QUANT_SKIP_LOAD(i) (g_test_quant_skip_load != 0 && (i) == 0)
#else
#define PURO_QUANT_SKIP_LOAD(i) false
#endif


// Packed magnitude maximum of the 16 BF16 values in v0 and v1 (per half, see
// bf16x2_absmax).
__device__ __forceinline__ uint32_t absmax16(const uint4 &v0, const uint4 &v1) {
  return bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w)),
                       bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
}

__device__ __forceinline__ uint2 codes8(const uint4 &v, const BlockDivider &div) {
  return make_uint2(block_codes4(v.x, v.y, div), block_codes4(v.z, v.w, div));
}
__device__ __forceinline__ uint2 codes8_fast(const uint4 &v, uint64_t nr2, uint64_t s2) {
  return make_uint2(block_codes4_fast(v.x, v.y, nr2, s2), block_codes4_fast(v.z, v.w, nr2, s2));
}


// The tile in a stage: box b = columns 64b .. 64b+63; row r of a box is 128 bytes with
// its 16-byte chunk k stored at chunk position k ^ (r % 8).
// Row phase: 8 lanes per tile row; lane j of the group holds columns 8j .. 8j+7 (box 0)
// and 64+8j .. 64+8j+7 (box 1), so each load of the group covers one whole swizzled row.
__device__ __forceinline__ uint4 row_chunk(const uint8_t *stage, int r, int box, int j) {
  return *reinterpret_cast<const uint4 *>(stage + box * kBoxBytes + r * 128 +
                                          ((j ^ (r & 7)) << 4));
}
// Column phase: thread (cp, g) holds columns 2cp, 2cp+1 of tile rows TG*g .. TG*g+TG-1
// as BF16 pairs (TG = 8192 / NT); a warp reads one 128-byte row of one box per load,
// conflict free.
template <int TG>
__device__ __forceinline__ void read_column_pairs(const uint8_t *stage, uint32_t (&w)[TG]) {
  const int cp = threadIdx.x & 63;
  const int g = threadIdx.x >> 6;
  const uint8_t *box = stage + (cp >> 5) * kBoxBytes;
  const int chunk = (cp & 31) >> 2;
  const int byte = (cp & 3) * 4;
#pragma unroll
  for (int i = 0; i < TG; ++i) {
    const int t = TG * g + i;
    w[i] = *reinterpret_cast<const uint32_t *>(box + t * 128 + ((chunk ^ (t & 7)) << 4) + byte);
  }
}

// Codes of the held column pair into the code tile: code-tile row = tile column (128
// bytes = the 128 tile rows), 16-byte chunk k at position k ^ (row % 8). TG = 16 gives
// one chunk per column, TG = 32 two.
template <int TG, bool FAST>
__device__ __forceinline__ void column_codes_to_smem(const uint32_t (&w)[TG],
                                                     const BlockDivider &div0,
                                                     const BlockDivider &div1, uint8_t *codes) {
  static_assert(TG == 16 || TG == 32, "16 or 32 tile rows per thread");
  const int cp = threadIdx.x & 63;
  const int g = threadIdx.x >> 6;
  uint32_t q0[TG / 4], q1[TG / 4];
#pragma unroll
  for (int i = 0; i < TG / 4; ++i) {
    // column 2cp is the low half of each word, column 2cp+1 the high half
    const uint32_t *wi = &w[4 * i];
    if constexpr (FAST) {
      q0[i] = half_codes4_fast<false>(wi[0], wi[1], wi[2], wi[3], pack2(-div0.r, -div0.r), pack2(div0.s, div0.s));
      q1[i] = half_codes4_fast<true>(wi[0], wi[1], wi[2], wi[3], pack2(-div1.r, -div1.r), pack2(div1.s, div1.s));
    } else {
      q0[i] = block_codes4(__byte_perm(wi[0], wi[1], 0x5410), __byte_perm(wi[2], wi[3], 0x5410), div0);
      q1[i] = block_codes4(__byte_perm(wi[0], wi[1], 0x7632), __byte_perm(wi[2], wi[3], 0x7632), div1);
    }
  }
  const int r0 = 2 * cp, r1 = 2 * cp + 1;
  uint8_t *row0 = codes + r0 * 128;
  uint8_t *row1 = codes + r1 * 128;
#pragma unroll
  for (int k = 0; k < TG / 16; ++k) {
    const int chunk = (TG / 16) * g + k;
    *reinterpret_cast<uint4 *>(row0 + ((chunk ^ (r0 & 7)) << 4)) =
        make_uint4(q0[4 * k], q0[4 * k + 1], q0[4 * k + 2], q0[4 * k + 3]);
    *reinterpret_cast<uint4 *>(row1 + ((chunk ^ (r1 & 7)) << 4)) =
        make_uint4(q1[4 * k], q1[4 * k + 1], q1[4 * k + 2], q1[4 * k + 3]);
  }
}

// P2: power-of-two scales (UE8M0 bytes) instead of the method's FP32 amax / 448; the codes
// then come out of the same fast path exactly as x * 2^-e (see pow2_scale).
template <int MODE, bool P2, int G>
__global__ void __launch_bounds__(Threads<MODE>::value, kCtasPerSm)
    k_quant_tiles(const __grid_constant__ QParams<G> prm) {
  constexpr bool kRows = MODE == Q_ROWS || MODE == Q_DUAL;
  constexpr bool kCols = MODE == Q_COLS || MODE == Q_DUAL;
  constexpr bool kWeight = MODE == Q_WEIGHT;
  constexpr int NT = Threads<MODE>::value;
  constexpr int NG = NT / 64;           // token groups of the column phase
  constexpr int TG = kTile / NG;        // tile rows per thread in the column phase
  constexpr int RSTEP = NT / 8;         // tile rows per pass of the row phase
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t *codes = smem + kOffCodes;
  float (*part)[kTile] = reinterpret_cast<float (*)[kTile]>(smem + kOffPart);
  float *warp_max = reinterpret_cast<float *>(smem + kOffWarpMax);
  float2 *col_div = reinterpret_cast<float2 *>(smem + kOffColDiv);
  const uint32_t bar0 = sbase + kOffBar;
  volatile int *fail = reinterpret_cast<volatile int *>(smem + kOffMisc);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tiles = prm.tiles;
  const unsigned long long timeout_ns = prm.args[0].timeout_ns;
  int *const status = prm.args[0].status;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
    *fail = 0;
    fence_barrier_init();
    const int p0 = problem_of(prm, 0, blockIdx.x < tiles ? blockIdx.x : 0);
    prefetch_tensormap(&prm.tmX[p0]);
    if (kCols || (kWeight && prm.args[p0].write_t)) prefetch_tensormap(&prm.tmT[p0]);
  }
  __syncthreads();

  // Tile i of this CTA is global tile blockIdx.x + i * gridDim.x; stage i % kStages.
  int p_issue = 0;  // thread 0: the problem of the last tile it issued
  auto issue = [&](int i) {
    const int tile = blockIdx.x + i * gridDim.x;
    if (tile >= tiles || PURO_QUANT_SKIP_LOAD(i)) return;
    const int p = problem_of(prm, p_issue, tile);
    if (p != p_issue) {
      prefetch_tensormap(&prm.tmX[p]);
      if (kCols || (kWeight && prm.args[p].write_t)) prefetch_tensormap(&prm.tmT[p]);
      p_issue = p;
    }
    const QArgs &a = prm.args[p];
    const int lt = tile - a.tile_begin;
    const int tr = lt / a.tiles_c, tc = lt % a.tiles_c;
    const int s = i % kStages;
    const uint32_t bar = bar0 + 8 * s;
    const uint32_t dst = sbase + s * kStageBytes;
    mbar_arrive_expect_tx(bar, kStageBytes);
    tma_load_2d(dst, &prm.tmX[p], bar, tc * kTile, tr * kTile);
    tma_load_2d(dst + kBoxBytes, &prm.tmX[p], bar, tc * kTile + 64, tr * kTile);
  };
  if (tid == 0)
    for (int i = 0; i < kStages; ++i) issue(i);

  const int rg = tid >> 3, j8 = tid & 7;   // row group and its lane in the row phase
  const int cp = tid & 63, g = tid >> 6;
  int i = 0;
  int prob = 0;           // the problem of the current tile
  bool any_t = false;     // thread 0: a transposed store was issued
  for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
    const int s = i % kStages;
    prob = problem_of(prm, prob, tile);
    const QArgs &args = prm.args[prob];
    const bool write_t = kCols || (kWeight && args.write_t);
    const int lt = tile - args.tile_begin;
    const int tr = lt / args.tiles_c, tc = lt % args.tiles_c;
    const int64_t r0 = static_cast<int64_t>(tr) * kTile;
    const int64_t c0 = static_cast<int64_t>(tc) * kTile;
    const uint8_t *stage = smem + s * kStageBytes;
    const bool waited = mbar_wait(bar0 + 8 * s, (i / kStages) & 1, timeout_ns, fail);
    if (__syncthreads_or(!waited)) {
      if (tid == 0) {
        *fail = 1;
        atomicOr(status, 1);
      }
      break;
    }
    if (tid == 0 && write_t) bulk_wait_group_read<0>();  // the code tile is free again

    // ---------------------------------------------------------------- weight block
    BlockDivider wdiv = zero_block_divider();
    if (kWeight) {
      uint32_t m2 = 0u;
#pragma unroll
      for (int p = 0; p < kTile / RSTEP; ++p)
        m2 = bf16x2_absmax(m2, absmax16(row_chunk(stage, rg + RSTEP * p, 0, j8),
                                        row_chunk(stage, rg + RSTEP * p, 1, j8)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m2 = bf16x2_absmax(m2, __shfl_xor_sync(0xffffffffu, m2, o));
      const float m = bf16x2_absmax_to_f32(m2);
      if (lane == 0) warp_max[warp] = m;
      __syncthreads();
      float amax = warp_max[0];
#pragma unroll
      for (int k = 1; k < NT / 32; ++k) amax = fmaxf(amax, warp_max[k]);
      if constexpr (P2) {
        const uint32_t byte = pow2_scale(amax, wdiv);
        if (tid == 0) args.sb[static_cast<int64_t>(tr) * args.tiles_c + tc] = static_cast<uint8_t>(byte);
      } else {
        float sblk;
        block_scale(amax, sblk, wdiv);
        if (tid == 0) args.s[static_cast<int64_t>(tr) * args.tiles_c + tc] = sblk;
      }
    }

    // ---------------------------------------------------------------- row-wise codes
    if (kRows || kWeight) {
      // A thread holds 16 columns of NP rows. All NP rows are loaded and their scales
      // formed before any code, and the codes take the fast path without a branch when
      // every block the warp holds allows it (the slow path only serves tiny, infinite
      // or NaN maxima).
      constexpr int NP = kTile / RSTEP;
      static_assert(NP <= 8, "one lane of the row's 8 forms each of a thread's row scales");
      uint4 v0[NP], v1[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        v0[p] = row_chunk(stage, rg + RSTEP * p, 0, j8);
        v1[p] = row_chunk(stage, rg + RSTEP * p, 1, j8);
      }
      // One lane per row forms the row's scale and divider (lane j8 of the row group takes
      // row p = j8) and shares the divider by shuffle; it also writes the row's scale.
      float srow_mine = 0.0f;   // lane j8 < NP: the scale of its row p = j8
      uint32_t brow_mine = 0u;  // P2: its scale byte
      uint32_t m[NP];
      BlockDivider div[NP];
      bool ok = true;
      if (kRows) {
#pragma unroll
        for (int p = 0; p < NP; ++p) m[p] = absmax16(v0[p], v1[p]);
#pragma unroll
        for (int o = 4; o > 0; o >>= 1)
#pragma unroll
          for (int p = 0; p < NP; ++p) m[p] = bf16x2_absmax(m[p], __shfl_xor_sync(0xffffffffu, m[p], o));
        uint32_t mm = 0u;  // lanes j8 >= NP take amax 0, which stays on the fast path
#pragma unroll
        for (int p = 0; p < NP; ++p)
          if (j8 == p) mm = m[p];
        BlockDivider dm;
        if constexpr (P2)
          brow_mine = pow2_scale(bf16x2_absmax_to_f32(mm), dm);
        else
          block_scale_fast(bf16x2_absmax_to_f32(mm), srow_mine, dm, ok);
        const int src = lane & ~7;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          div[p].s = __shfl_sync(0xffffffffu, dm.s, src + p);
          div[p].r = __shfl_sync(0xffffffffu, dm.r, src + p);
          div[p].fast = true;
        }
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) div[p] = wdiv;
        ok = wdiv.fast;
      }
      uint2 q0[NP], q1[NP];
      if (__all_sync(0xffffffffu, ok)) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const uint64_t nr2 = pack2(-div[p].r, -div[p].r), s2 = pack2(div[p].s, div[p].s);
          q0[p] = codes8_fast(v0[p], nr2, s2);
          q1[p] = codes8_fast(v1[p], nr2, s2);
        }
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          if constexpr (kRows && !P2) {  // the general scale and divider, on every lane
            float sp;
            block_scale(bf16x2_absmax_to_f32(m[p]), sp, div[p]);
            if (j8 == p) srow_mine = sp;
          }
          q0[p] = codes8(v0[p], div[p]);
          q1[p] = codes8(v1[p], div[p]);
        }
      }
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int64_t row = r0 + rg + RSTEP * p;
        if (row < args.R) {  // C is a multiple of 128 in these modes
          uint8_t *qrow = args.q + row * args.ldq + c0 + 8 * j8;
          *reinterpret_cast<uint2 *>(qrow) = q0[p];
          *reinterpret_cast<uint2 *>(qrow + 64) = q1[p];
          if (kRows && j8 == p) {
            if constexpr (P2)
              args.sb[(c0 / kTile) * args.R + row] = static_cast<uint8_t>(brow_mine);
            else
              args.s[(c0 / kTile) * args.R + row] = srow_mine;
          }
        }
      }
    }

    // ---------------------------------------------------------------- transposed codes
    if constexpr (kCols || kWeight) if (write_t) {
      uint32_t w[TG];
      read_column_pairs<TG>(stage, w);
      BlockDivider d0 = wdiv, d1 = wdiv;
      if (kCols) {
        uint32_t m2 = 0u;  // column 2cp in the low half, 2cp + 1 in the high half
#pragma unroll
        for (int k = 0; k < TG; ++k) m2 = bf16x2_absmax(m2, w[k]);
        part[g][2 * cp] = __uint_as_float((m2 & 0x7FFFu) << 16);
        part[g][2 * cp + 1] = __uint_as_float(m2 & 0x7FFF0000u);
      }
      __syncthreads();  // column partials ready; the code tile is free (thread 0 waited)
      bool tile_fast = wdiv.fast;
      if (kCols) {
        // The first 64 threads finish the column maxima and form the 128 column scales
        // and divisors once; every thread then reads the two it needs. A column off the
        // fast path stores r = -1, and sends the whole tile to the general code.
        bool ok = true;
        if (g == 0) {
          float a0 = part[0][2 * cp], a1 = part[0][2 * cp + 1];
#pragma unroll
          for (int k = 1; k < NG; ++k) {
            a0 = fmaxf(a0, part[k][2 * cp]);
            a1 = fmaxf(a1, part[k][2 * cp + 1]);
          }
          float s0, s1;
          bool ok0 = true, ok1 = true;
          uint32_t b0 = 0, b1 = 0;
          if constexpr (P2) {
            b0 = pow2_scale(a0, d0);
            b1 = pow2_scale(a1, d1);
          } else {
            block_scale_fast(a0, s0, d0, ok0);
            block_scale_fast(a1, s1, d1, ok1);
            if (!ok0) block_scale(a0, s0, d0);
            if (!ok1) block_scale(a1, s1, d1);
          }
          ok = ok0 && ok1;
          col_div[2 * cp] = make_float2(d0.s, d0.fast ? d0.r : -1.0f);
          col_div[2 * cp + 1] = make_float2(d1.s, d1.fast ? d1.r : -1.0f);
          const int64_t c = c0 + 2 * cp;
          if constexpr (P2) {
            uint8_t *strow = args.stb + static_cast<int64_t>(tr) * args.C;
            if (c < args.C) strow[c] = static_cast<uint8_t>(b0);
            if (c + 1 < args.C) strow[c + 1] = static_cast<uint8_t>(b1);
          } else {
            float *strow = args.st + static_cast<int64_t>(tr) * args.C;
            if (c < args.C) strow[c] = s0;
            if (c + 1 < args.C) strow[c + 1] = s1;
          }
        }
        tile_fast = __syncthreads_and(ok);
        const float2 e0 = col_div[2 * cp], e1 = col_div[2 * cp + 1];
        d0 = BlockDivider{e0.x, e0.y, e0.y >= 0.0f};
        d1 = BlockDivider{e1.x, e1.y, e1.y >= 0.0f};
      }
      if (tile_fast)
        column_codes_to_smem<TG, true>(w, d0, d1, codes);
      else
        column_codes_to_smem<TG, false>(w, d0, d1, codes);
      fence_proxy_async_smem();
    }
    __syncthreads();  // the stage and (if any) the code tile are complete
    if (tid == 0) {
      if (write_t) {
        tma_store_2d(&prm.tmT[prob], sbase + kOffCodes, static_cast<int32_t>(r0), static_cast<int32_t>(c0));
        bulk_commit_group();
        any_t = true;
      }
      issue(i + kStages);  // refill the stage just consumed
    }
  }

  if (tid == 0) {
    if (any_t) bulk_wait_group_all();
    if (*fail) {
      // Let every load still in flight land before the CTA exits (bounded).
      for (int k = 0; k < kStages; ++k) {
        const int ii = i + k;
        if (blockIdx.x + ii * gridDim.x < tiles)
          mbar_wait(bar0 + 8 * (ii % kStages), (ii / kStages) & 1, timeout_ns, nullptr);
      }
    }
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [rows, cols] with row stride `ld` elements of `elem` bytes, box [box_rows, box_cols],
// 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem,
              uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long ns = [] {
    const char *e = std::getenv("PURO_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return ns;
}

// Fills the tensor maps and the sizes of one problem; the caller's args carry the outputs.
template <int MODE>
bool set_problem(CUtensorMap &tmX, CUtensorMap &tmT, QArgs &args, const uint16_t *X, int64_t R, int64_t C,
                 int64_t ldx, uint8_t *qt) {
  if (!make_map(&tmX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, R, C, ldx, kTile, 64)) return false;
  if (qt != nullptr) {
    // the transposed codes [C, R]: one box of 128 rows (tile columns) x 128 bytes
    if (!make_map(&tmT, qt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, C, R, R, kTile, kTile)) return false;
  } else {
    tmT = tmX;  // unused
  }
  args.R = R;
  args.C = C;
  args.tiles_r = static_cast<int>((R + kTile - 1) / kTile);
  args.tiles_c = static_cast<int>((C + kTile - 1) / kTile);
  args.timeout_ns = wait_timeout_ns();
  return true;
}

// Launches k_quant_tiles<MODE, P2, G> over prm (its problems, count and tiles filled in).
template <int MODE, bool P2, int G>
int launch_params(QParams<G> &prm, cudaStream_t stream) {
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  static PerDevice<int *> status_addr;  // g_quant_status on this device, looked up once
  int *st = nullptr;
  if (!status_addr.get(st, [](int, int *&v) {
        return cudaGetSymbolAddress(reinterpret_cast<void **>(&v), g_quant_status) == cudaSuccess;
      }))
    return PURO_ERR_CUDA;
  for (int p = 0; p < prm.count; ++p) prm.args[p].status = st;
  const int grid = prm.tiles < kCtasPerSm * sms ? prm.tiles : kCtasPerSm * sms;
  auto kern = k_quant_tiles<MODE, P2, G>;
  static PerDevice<bool> smem_opt_in;  // dynamic shared memory opted in once per device
  bool done = false;
  if (!smem_opt_in.get(done, [&](int, bool &v) {
        v = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) ==
            cudaSuccess;
        return v;
      }))
    return PURO_ERR_CUDA;
  kern<<<grid, Threads<MODE>::value, kSmemBytes, stream>>>(prm);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    std::fprintf(stderr, "puro_fp8: quantiser launch: %s\n", cudaGetErrorString(e));
    return PURO_ERR_LAUNCH;
  }
  return PURO_OK;
}

template <int MODE, bool P2>
int launch_tiles(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *qt, QArgs args,
                 cudaStream_t stream) {
  QParams<1> prm;
  prm.args[0] = args;
  if (!set_problem<MODE>(prm.tmX[0], prm.tmT[0], prm.args[0], X, R, C, ldx, qt)) return PURO_ERR_CUDA;
  prm.args[0].tile_begin = 0;
  prm.count = 1;
  prm.tiles = prm.args[0].tiles_r * prm.args[0].tiles_c;
  return launch_params<MODE, P2, 1>(prm, stream);
}

}  // namespace

// ------------------------------------------------------------------ launchers
int launch_quant_rows(const uint16_t *X, int64_t R, int64_t C, int64_t ldx, uint8_t *Xq,
                      int64_t ldq, float *S, cudaStream_t stream, uint8_t *Sb) {
  QArgs a{};
  a.q = Xq;
  a.ldq = ldq;
  a.s = S;
  a.sb = Sb;
  return Sb != nullptr ? launch_tiles<Q_ROWS, true>(X, R, C, ldx, nullptr, a, stream)
                       : launch_tiles<Q_ROWS, false>(X, R, C, ldx, nullptr, a, stream);
}

int launch_quant_cols(const uint16_t *X, int64_t T, int64_t C, int64_t ldx, uint8_t *XqT,
                      float *ST, uint8_t *Xq, float *S, cudaStream_t stream, uint8_t *STb, uint8_t *Sb) {
  QArgs a{};
  a.st = ST;
  a.stb = STb;
  const bool p2 = STb != nullptr;
  if (Xq != nullptr) {
    a.q = Xq;
    a.ldq = C;
    a.s = S;
    a.sb = Sb;
    return p2 ? launch_tiles<Q_DUAL, true>(X, T, C, ldx, XqT, a, stream)
              : launch_tiles<Q_DUAL, false>(X, T, C, ldx, XqT, a, stream);
  }
  return p2 ? launch_tiles<Q_COLS, true>(X, T, C, ldx, XqT, a, stream)
            : launch_tiles<Q_COLS, false>(X, T, C, ldx, XqT, a, stream);
}

int launch_quant_weight(const uint16_t *W, int64_t R, int64_t C, int64_t ldw, uint8_t *Wq,
                        uint8_t *WqT, float *S, cudaStream_t stream, uint8_t *Sb) {
  QArgs a{};
  a.q = Wq;
  a.ldq = C;
  a.s = S;
  a.sb = Sb;
  a.write_t = WqT != nullptr;
  return Sb != nullptr ? launch_tiles<Q_WEIGHT, true>(W, R, C, ldw, WqT, a, stream)
                       : launch_tiles<Q_WEIGHT, false>(W, R, C, ldw, WqT, a, stream);
}

int launch_quant_weight_grouped(const WeightProblem *probs, int count, cudaStream_t stream) {
  // Up to QGROUP_MAX weights per launch; the parameter block lives on the host stack only
  // until the launch has copied it.
  static thread_local QParams<QGROUP_MAX> prm;
  for (int first = 0; first < count; first += QGROUP_MAX) {
    const int n = count - first < QGROUP_MAX ? count - first : QGROUP_MAX;
    int tiles = 0;
    for (int k = 0; k < n; ++k) {
      const WeightProblem &w = probs[first + k];
      QArgs a{};
      a.q = w.Wq;
      a.ldq = w.C;
      a.s = w.S;
      a.write_t = w.WqT != nullptr;
      if (!set_problem<Q_WEIGHT>(prm.tmX[k], prm.tmT[k], a, w.W, w.R, w.C, w.ldw, w.WqT)) return PURO_ERR_CUDA;
      a.tile_begin = tiles;
      tiles += a.tiles_r * a.tiles_c;
      prm.args[k] = a;
    }
    prm.count = n;
    prm.tiles = tiles;
    if (int e = launch_params<Q_WEIGHT, false, QGROUP_MAX>(prm, stream)) return e;
  }
  return PURO_OK;
}

int read_and_clear_quant_status(cudaStream_t stream, int *status_out) {
  int host = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_quant_status, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_quant_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                              stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return PURO_ERR_CUDA;
  *status_out = host;
  return PURO_OK;
}

}  // namespace puro

#ifdef PURO_TEST_HOOKS
extern "C" __attribute__((visibility("default"))) int puro_test_set_quant_skip_load(int on) {
  return cudaMemcpyToSymbol(puro::g_test_quant_skip_load, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
