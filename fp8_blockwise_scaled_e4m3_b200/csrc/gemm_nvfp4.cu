// NVFP4 GEMM for sm_100a: C[M, N] = A . B^T with both operands in E2M1 (two codes per byte,
// quantised along K in groups of 16 with a UE4M3 factor each, and an FP32 tensor scale each),
// on the block-scaled tensor-core MMA (tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X),
// which applies the factors inside the MMA and accumulates all of K in FP32 in TMEM.
//
// The pages name FP4 only as a capability of the hardware they chose (the jj-blog page, the
// paragraph after its Table 2); the format is NVIDIA's published NVFP4 (see nvfp4_quant.cu):
//   C[m, n] = s_tA * s_tB * sum_k dec(qA[m, k]) * fA[m, k/16] * dec(qB[n, k]) * fB[n, k/16]
// with s_t = amax_t / 2688, rounded to BF16 once at the end. Every pass of a linear layer is
// this product with both operands quantised along its reduction dimension (fprop: X and W
// row-wise; dgrad: dY row-wise and W along N_out; wgrad: dY and X along the tokens).
//
// Structure as the block-scaled FP8 kernel (gemm_mx.cu): persistent, one CTA (M <= 128) or
// one CTA pair (cta_group::2, 256-row tiles) per SM (pair), 512 threads:
//   warp 0       TMA producer: A and B K blocks of 128 bytes (256 codes) per ring stage, and
//                the stage's factors (this CTA's 128 A rows and the tile's 256 B rows, 16
//                bytes each) into shared memory, counted on the stage's factor barrier
//   warp 1       MMA issuer: per K block four MMAs of K = 64 (32 bytes), each with its own
//                factor cells, one commit to the stage's empty barrier
//   warps 4..11  epilogue: the tile's FP32 accumulator times s_tA * s_tB, BF16, TMA stores
//   warps 12..15 scale writers, one per TMEM lane quadrant: for every K block they read the
//                16 factor bytes of each row they serve from the stage's shared memory (a
//                warp's 32 rows are 512 contiguous bytes) and store them as TMEM cells in the
//                layout the MMA reads (below), counted on the stage's full barrier. (Loading
//                the factors from global memory in these warps, even coalesced, held the
//                kernel near 1.5 PFLOP/s; without those loads it ran near 4.5.)
// Factor layout in TMEM (probed on B200 with single MMAs): for each MMA, the factors of A row
// m are read from lane m, column m / 32, and those of B row n from lane 32 q + n % 32, column
// n / 32 of the lane quadrant q of the row being computed; byte j of a 32-bit cell is the
// factor of the MMA's 16-element group j. Each quadrant therefore holds its 32 A rows'
// cells (written into all four A columns) and all 256 B rows' cells (8 columns) for every
// one of a K block's four MMAs.
// TMEM: accumulator columns 0..255; ring slot s: 48 columns from 256 + 48 s, MMA k's A
// cells at + 12 k (4 columns) and its B cells at + 12 k + 4 (8 columns).
// K % 128 == 0: when K % 256 == 128 the last K block is half a block; TMA fills its missing
// bytes with zeros and the writers give the missing groups the factor 0.
// Every mbarrier wait is bounded; a wait that gives up sets the abort flag and the device
// status word, and the CTA drains and exits.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "../../include/puro_fp8.h"
#include "host_cache.h"
#include "ptx.cuh"
#include "quant.h"

namespace puro {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in bytes: 256 codes per K block
constexpr int THREADS = 512;
constexpr int EPI_FIRST = 4, EPI_WARPS = 8, SFW_FIRST = 12;
constexpr int A_BYTES = BM * BK;
constexpr int STG_BOX_BYTES = 32 * 128;            // 32 rows x 64 BF16, 128B-swizzled
constexpr int STG_WARP_BYTES = 2 * STG_BOX_BYTES;  // 128 columns per epilogue warp

constexpr int SFA_BYTES = BM * 16;  // one K block's factors of 128 A rows
constexpr int SFB_BYTES = BN * 16;  // ... and of 256 B rows

template <bool PAIR>
struct NvCfg {
  static constexpr int STAGES = PAIR ? 4 : 2;  // single CTAs (M <= 128) stage all 256 B rows
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA stages
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int TILE_ROWS = PAIR ? 2 * BM : BM;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_STG = OFF_SFB + STAGES * SFB_BYTES;
  static constexpr int OFF_BAR = OFF_STG + EPI_WARPS * STG_WARP_BYTES;
  // full/empty per stage, tfull, tempty, drain, a factor barrier per stage
  static constexpr int N_BARS = 3 * STAGES + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(OFF_STG % 1024 == 0, "swizzled staging must be 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};
constexpr uint32_t ACC_COL = 0, SF_COL = 256, SF_SLOT_COLS = 48, SF_MMA_COLS = 12;
static_assert(SF_COL + NvCfg<true>::STAGES * SF_SLOT_COLS <= 512, "TMEM columns");
// Register split: warpgroup 0 (producer, issuer), warpgroups 1-2 (epilogue: 128 accumulator
// registers), warpgroup 3 (scale writers)
constexpr int LAUNCH_REGS = 128;  // 65536 / 512
constexpr int REGS_WG0 = 56, REGS_EPI = 168, REGS_SFW = 120;
static_assert(128 * REGS_WG0 + 256 * REGS_EPI + 128 * REGS_SFW == THREADS * LAUNCH_REGS, "register split");
static_assert(REGS_WG0 <= LAUNCH_REGS && REGS_SFW <= LAUNCH_REGS && REGS_EPI >= LAUNCH_REGS, "dec / inc directions");

// Block-scaled instruction descriptor: E2M1 A and B (format 1), K-major, FP32 accumulate,
// UE4M3 factors (scale format 0), K = 64, M x N, factor ids 0.
__host__ __device__ constexpr uint32_t idesc_nv(int m, int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void mma_nv(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_nv_pair(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, const uint32_t (&v)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct NvArgs {
  const uint8_t *As;  // UE4M3 [K blocks][M][16]
  const uint8_t *Bs;  // UE4M3 [K blocks][N][16]
  const float *a_amax, *b_amax;
  int M, N, K;
  int num_m, num_n, kblocks, m_fastest;
  unsigned long long timeout_ns;
  int *status;
};

__device__ int g_nv_status;  // non-zero: a bounded wait gave up since the last read

__device__ __forceinline__ void nv_tile_coords(int tile, const NvArgs &a, int &mt, int &nt) {
  if (a.m_fastest) {
    mt = tile % a.num_m;
    nt = tile / a.num_m;
  } else {
    nt = tile % a.num_n;
    mt = tile / a.num_n;
  }
}

__device__ __forceinline__ uint32_t bf16x2_bits_nv(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_nvfp4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmSA,
                 const __grid_constant__ CUtensorMap tmSB, const NvArgs args) {
  using C = NvCfg<PAIR>;
  constexpr int STAGES = C::STAGES, B_BYTES = C::B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t tempty_bar = tfull_bar + 8u;
  const uint32_t drain_bar = tfull_bar + 16u;
  auto sf_full_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 3 + s); };  // this CTA's factor bytes
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // PAIR: rank 0 of the cluster is the leader: it issues the MMAs for both CTAs and holds the
  // barriers both CTAs report to. Tiles are walked per cluster; rank r owns rows 128 r .. of
  // a 256-row tile.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int first_tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  auto row_base = [&](int mt) { return mt * C::TILE_ROWS + static_cast<int>(rank) * BM; };
  auto arrive_leader = [&](uint32_t bar) {
    if constexpr (PAIR)
      mbar_arrive_cluster(map_to_rank(bar, 0));
    else
      mbar_arrive(bar);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // the producer's arrival (with the stage's TMA bytes) and the scale writers' (of both
      // CTAs of a pair)
      mbar_init(full_bar(s), 1 + (PAIR ? 8 : 4));
      mbar_init(empty_bar(s), 1);  // the MMA commit
      mbar_init(sf_full_bar(s), 1);  // this CTA's producer, with the factor bytes
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, PAIR ? 2 * EPI_WARPS : EPI_WARPS);
    mbar_init(drain_bar, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmC);
    prefetch_tensormap(&tmSA);
    prefetch_tensormap(&tmSB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync();  // both CTAs' barriers exist before either reports to the other
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  const int tiles = args.num_m * args.num_n;
  const int kblocks = args.kblocks;
  const uint64_t tmo = args.timeout_ns;

  if (warp < EPI_FIRST) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_WG0));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
        int mt, nt;
        nv_tile_coords(tile, args, mt, nt);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(s), ph ^ 1u, tmo, abort)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            // Both CTAs' loads count on the leader's barrier, armed by the leader with the
            // pair's bytes; a peer load for a stage's next use starts only after the MMA that
            // read the stage completed (its empty barrier), so never in the previous phase.
            const uint32_t fb = map_to_rank(full_bar(s), 0);
            if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * (A_BYTES + B_BYTES));
            tma_load_2d_pair(sbase + C::OFF_A + s * A_BYTES, &tmA, fb, kb * BK, row_base(mt));
            tma_load_2d_pair(sbase + C::OFF_B + s * B_BYTES, &tmB, fb, kb * BK,
                             nt * BN + static_cast<int>(rank) * C::B_ROWS);
          } else {
            mbar_arrive_expect_tx(full_bar(s), A_BYTES + B_BYTES);
            tma_load_2d(sbase + C::OFF_A + s * A_BYTES, &tmA, full_bar(s), kb * BK, mt * BM);
            tma_load_2d(sbase + C::OFF_B + s * B_BYTES, &tmB, full_bar(s), kb * BK, nt * BN);
          }
          // this CTA's factors of the K block: its A rows and the tile's B rows (rows past the
          // matrix read as zeros), for its own scale writers
          mbar_arrive_expect_tx(sf_full_bar(s), SFA_BYTES + SFB_BYTES);
          tma_load_3d(sbase + C::OFF_SFA + s * SFA_BYTES, &tmSA, sf_full_bar(s), 0, row_base(mt), kb);
          tma_load_3d(sbase + C::OFF_SFB + s * SFB_BYTES, &tmSB, sf_full_bar(s), 0, nt * BN, kb);
          issued |= 1u << s;
          issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
          if (++s == STAGES) s = 0, ph ^= 1u;
        }
      }
      if (!ok) {
        *abort = 1;
        atomicOr(args.status, 1);
        // Every issued load lands before the CTA can exit (a peer's loads count on the
        // leader's barriers; the peer stays alive through the final cluster barrier).
        for (int i = 0; i < STAGES; ++i)
          if ((issued >> i) & 1u) {
            if (leader) mbar_wait(full_bar(i), (issued_parity >> i) & 1u, tmo, nullptr);
            mbar_wait(sf_full_bar(i), (issued_parity >> i) & 1u, tmo, nullptr);
          }
      }
    } else if (warp == 1 && lane == 0 && leader) {
      // ---------------------------------------------------------------- MMA issuer
      int s = 0;
      uint32_t ph = 0, it = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step, ++it) {
        if (!mbar_wait(tempty_bar, (it & 1u) ^ 1u, tmo, abort)) {  // the accumulator is free
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full_bar(s), ph, tmo, abort)) {  // operands and factors
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = sbase + C::OFF_A + s * A_BYTES, b_addr = sbase + C::OFF_B + s * B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            const uint32_t sfa = tmem + SF_COL + SF_SLOT_COLS * s + SF_MMA_COLS * k, sfb = sfa + 4;
            if constexpr (PAIR)
              mma_nv_pair(tmem + ACC_COL, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k),
                          idesc_nv(2 * BM, BN), sfa, sfb, acc);
            else
              mma_nv(tmem + ACC_COL, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k),
                     idesc_nv(BM, BN), sfa, sfb, acc);
          }
          if constexpr (PAIR)
            mma_commit_pair_mc(empty_bar(s), 0x3);  // both CTAs' stage s and its factors are free
          else
            mma_commit(empty_bar(s));
          if (++s == STAGES) s = 0, ph ^= 1u;
        }
        if (ok) {
          if constexpr (PAIR)
            mma_commit_pair_mc(tfull_bar, 0x3);  // both CTAs' accumulators are complete
          else
            mma_commit(tfull_bar);
        }
      }
      if (!ok) {
        *abort = 1;
        atomicOr(args.status, 1);
        // arrives once every MMA issued here has finished
        if constexpr (PAIR)
          mma_commit_pair(drain_bar);
        else
          mma_commit(drain_bar);
        mbar_wait(drain_bar, 0, tmo, nullptr);
      }
    }
  } else if (warp >= SFW_FIRST) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_SFW));
    // ------------------------------------------------------------------ scale writers
    // Each K block's factors wait in the stage's shared memory (the producer's TMA); a writer
    // reads its rows' 16 bytes per K block and stores them as TMEM cells. The factor barrier
    // of a stage's next use completes only after the producer saw the stage's empty barrier,
    // i.e. after the MMA that read the previous cells, so the cells are free to overwrite.
    // A CTA pair reads each CTA's factors from that CTA's own TMEM: its 128 rows of A and all
    // 256 rows of B.
    const int quad = warp & 3;
    const uint32_t lane_field = static_cast<uint32_t>(quad * 32) << 16;
    const int kfac = args.K / 16;
    int s = 0;
    uint32_t ph = 0, seq = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
      for (int kb = 0; kb < kblocks; ++kb, ++seq) {
        // warp-uniform outcome: the stores below need the whole warp
        if (!__all_sync(0xffffffffu, mbar_wait(sf_full_bar(s), ph, tmo, abort))) {
          ok = false;
          break;
        }
        const uint8_t *fa = smem + C::OFF_SFA + s * SFA_BYTES;
        const uint8_t *fb = smem + C::OFF_SFB + s * SFB_BYTES;
        const uint4 va = *reinterpret_cast<const uint4 *>(fa + 16 * (32 * quad + lane));
        uint4 vb[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) vb[g] = *reinterpret_cast<const uint4 *>(fb + 16 * (32 * g + lane));
        // a half K block (K % 256 == 128) has factors for its first 128 codes only
        const bool full = 16 * kb + 8 < kfac;
        auto word = [&](const uint4 &v, int k) -> uint32_t {
          return k == 0 ? v.x : k == 1 ? v.y : !full ? 0u : k == 2 ? v.z : v.w;
        };
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < BK / 32; ++k) {
          const uint32_t a = word(va, k);
          const uint32_t ca[4] = {a, a, a, a};
          uint32_t cb[8];
#pragma unroll
          for (int g = 0; g < 8; ++g) cb[g] = word(vb[g], k);
          const uint32_t col = SF_COL + SF_SLOT_COLS * s + SF_MMA_COLS * k;
          tmem_st_x4(tmem + lane_field + col, ca);
          tmem_st_x8(tmem + lane_field + col + 4, cb);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) arrive_leader(full_bar(s));
        if (++s == STAGES) s = 0, ph ^= 1u;
      }
    }
    (void)seq;
    if (!ok && lane == 0) {
      *abort = 1;
      atomicOr(args.status, 1);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_EPI));
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3, half = (warp - EPI_FIRST) >> 2;
    const uint32_t taddr = tmem + ACC_COL + (static_cast<uint32_t>(quad * 32) << 16) + half * 128;
    const uint32_t stg = sbase + C::OFF_STG + (warp - EPI_FIRST) * STG_WARP_BYTES;
    // s_tA * s_tB, each s_t = amax_t / 2688 (correctly rounded)
    const float gs = __fmul_rn(__fdiv_rn(*args.a_amax, 2688.0f), __fdiv_rn(*args.b_amax, 2688.0f));
    uint32_t it = 0;
    bool ok = true;
    for (int tile = first_tile; tile < tiles; tile += tile_step, ++it) {
      int mt, nt;
      nv_tile_coords(tile, args, mt, nt);
      if (!mbar_wait(tfull_bar, it & 1u, tmo, abort)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t r0[64], r1[64];
      tmem_ld_64cols(taddr, r0);
      tmem_ld_64cols(taddr + 64, r1);
      tmem_wait_ld_dep(r0);
      tmem_wait_ld_dep(r1);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) arrive_leader(tempty_bar);  // the MMA may start the next tile
      if (lane == 0) bulk_wait_group_read<0>();  // the previous tile's stores left the staging
      __syncwarp();
      auto v = [&](const uint32_t *r, int i) { return __fmul_rn(__uint_as_float(r[i]), gs); };
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t *r = j < 8 ? r0 : r1;
        const int jj = j & 7;
        const uint32_t addr = stg + (j >> 3) * STG_BOX_BYTES + lane * 128 + ((jj ^ (lane & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                     "r"(bf16x2_bits_nv(v(r, 8 * jj), v(r, 8 * jj + 1))),
                     "r"(bf16x2_bits_nv(v(r, 8 * jj + 2), v(r, 8 * jj + 3))),
                     "r"(bf16x2_bits_nv(v(r, 8 * jj + 4), v(r, 8 * jj + 5))),
                     "r"(bf16x2_bits_nv(v(r, 8 * jj + 6), v(r, 8 * jj + 7)))
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int row0 = row_base(mt) + quad * 32, col0 = nt * BN + half * 128;
        if (row0 < args.M) {
          if (col0 < args.N) tma_store_2d(&tmC, stg, col0, row0);
          if (col0 + 64 < args.N) tma_store_2d(&tmC, stg + STG_BOX_BYTES, col0 + 64, row0);
        }
        bulk_commit_group();
      }
    }
    if (lane == 0) bulk_wait_group_all();
    if (!ok && lane == 0) {
      *abort = 1;
      atomicOr(args.status, 1);
    }
  }

  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync();  // neither CTA leaves while the other may still use its shared memory or TMEM
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn nv_encode_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Row-major [rows, cols] matrix of `elem`-byte elements, box [box_rows, box_cols], 128B
// swizzle; reads past the edge return zeros.
bool nv_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem, uint64_t rows, uint64_t cols,
            uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn fn = nv_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Factors stored by K block, [kblocks][rows][16] bytes, as a 3-D tensor (16 bytes, rows,
// K blocks); a box is 16 bytes x box_rows rows of one K block, rows past the matrix read as
// zeros.
bool nv_factor_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t kblocks, uint32_t box_rows) {
  EncodeTiledFn fn = nv_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {16, rows, kblocks};
  const cuuint64_t strides[2] = {16, rows * 16};
  const cuuint32_t box[3] = {16, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned long long nv_timeout_ns() {
  static unsigned long long ns = [] {
    const char *e = std::getenv("PURO_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return ns;
}

template <bool PAIR>
int launch_nv(const uint8_t *Aq, const uint8_t *As, const float *a_amax, const uint8_t *Bq, const uint8_t *Bs,
              const float *b_amax, uint16_t *C, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  using CF = NvCfg<PAIR>;
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  static PerDevice<int *> status_addr;
  NvArgs args{};
  if (!status_addr.get(args.status, [](int, int *&v) {
        return cudaGetSymbolAddress(reinterpret_cast<void **>(&v), g_nv_status) == cudaSuccess;
      }))
    return PURO_ERR_CUDA;
  CUtensorMap ta, tb, tc, tsa, tsb;
  // operands as bytes: [rows, K/2], two codes per byte
  if (!nv_map(&ta, Aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K / 2, BM, BK) ||
      !nv_map(&tb, Bq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, CF::B_ROWS, BK) ||
      !nv_map(&tc, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, 32, 64) ||
      !nv_factor_map(&tsa, As, M, (K + 255) / 256, BM) || !nv_factor_map(&tsb, Bs, N, (K + 255) / 256, BN))
    return PURO_ERR_CUDA;
  args.As = As;
  args.Bs = Bs;
  args.a_amax = a_amax;
  args.b_amax = b_amax;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.kblocks = static_cast<int>((K / 2 + BK - 1) / BK);
  args.num_m = static_cast<int>((M + CF::TILE_ROWS - 1) / CF::TILE_ROWS);
  args.num_n = static_cast<int>((N + BN - 1) / BN);
  args.m_fastest = M <= N ? 1 : 0;
  args.timeout_ns = nv_timeout_ns();
  const int64_t tiles = static_cast<int64_t>(args.num_m) * args.num_n;
  auto kern = k_gemm_nvfp4<PAIR>;
  auto cluster_cfg = [&](int grid, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg{};
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = CF::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
  };
  // Once per device: the register split assumes exactly LAUNCH_REGS per thread at launch
  // (otherwise a setmaxnreg.inc could wait forever); shared memory opt-in; for a CTA pair,
  // the clusters that can be resident at once (the persistent grid's size).
  static PerDevice<int> prepared;
  int prep = PURO_ERR_CUDA;
  if (!prepared.get(prep, [&](int, int &v) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
        if (fa.numRegs != LAUNCH_REGS) {
          std::fprintf(stderr, "puro_fp8: NVFP4 GEMM kernel built with %d registers (expected %d); not launched\n",
                       fa.numRegs, LAUNCH_REGS);
          v = PURO_ERR_LAUNCH;
          return true;
        }
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CF::SMEM_BYTES) != cudaSuccess)
          return false;
        v = PURO_OK;
        if constexpr (PAIR) {
          cudaLaunchAttribute attr[1];
          cudaLaunchConfig_t cfg = cluster_cfg(2 * (sms / 2), attr);
          int clusters = 0;
          if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
            std::fprintf(stderr, "puro_fp8: no CTA pair of the NVFP4 GEMM kernel fits on this device\n");
            v = PURO_ERR_LAUNCH;
            return true;
          }
          v = clusters;  // > 0
        }
        return true;
      }))
    return PURO_ERR_CUDA;
  if (prep < 0) return prep;
  cudaError_t e;
  int grid;
  if constexpr (PAIR) {
    grid = static_cast<int>(2 * (tiles < prep ? tiles : prep));
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = cluster_cfg(grid, attr);
    e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, tsa, tsb, args);
    if (e == cudaSuccess) e = cudaGetLastError();
  } else {
    grid = static_cast<int>(tiles < sms ? tiles : sms);
    kern<<<grid, THREADS, CF::SMEM_BYTES, stream>>>(ta, tb, tc, tsa, tsb, args);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    std::fprintf(stderr, "puro_fp8: NVFP4 GEMM launch (grid %d): %s\n", grid, cudaGetErrorString(e));
    return PURO_ERR_LAUNCH;
  }
  return PURO_OK;
}

}  // namespace

// CTA pairs unless the output has at most 128 rows.
int launch_gemm_nvfp4(const uint8_t *Aq, const uint8_t *As, const float *a_amax, const uint8_t *Bq,
                      const uint8_t *Bs, const float *b_amax, uint16_t *C, int64_t M, int64_t N, int64_t K,
                      cudaStream_t stream) {
  return M > BM ? launch_nv<true>(Aq, As, a_amax, Bq, Bs, b_amax, C, M, N, K, stream)
                : launch_nv<false>(Aq, As, a_amax, Bq, Bs, b_amax, C, M, N, K, stream);
}

int *nv_status_word() {
  static PerDevice<int *> status_addr;
  int *st = nullptr;
  if (!status_addr.get(st, [](int, int *&v) {
        return cudaGetSymbolAddress(reinterpret_cast<void **>(&v), g_nv_status) == cudaSuccess;
      }))
    return nullptr;
  return st;
}

unsigned long long nv_wait_timeout_ns() { return nv_timeout_ns(); }

bool nv_bf16_map(CUtensorMap *map, const uint16_t *X, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows) {
  EncodeTiledFn fn = nv_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(X), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int read_and_clear_nv_status(cudaStream_t stream, int *status_out) {
  int host = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_nv_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_nv_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return PURO_ERR_CUDA;
  *status_out = host;
  return PURO_OK;
}

}  // namespace puro
