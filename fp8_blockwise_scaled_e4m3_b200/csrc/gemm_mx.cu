// Blockwise-FP8 GEMM with power-of-two (UE8M0) scales on the tensor cores' block-scaled MMA
// (tcgen05.mma.kind::mxf8f6f4.block_scale), sm_100a.
//
// The groups are the method's ("Paper walkthrough: Puro-2B ...", section "Lever 2: use
// blockwise FP8 from step zero": 1x128 along K for activations and gradients, 128x128
// weight blocks); the scales are the power-of-two mode's bytes (2^(byte - 127)). A power of
// two is applied exactly by the tensor core, which takes one scale per row of A and per
// column of B for every 32 elements of K and accumulates the whole K in FP32 in TMEM, so
// no promotion runs on the CUDA cores: the tile's accumulator is read once, at its end.
//
// One CTA per SM with 128 x 256 tiles when the output has at most 128 rows, otherwise a
// cluster of two CTAs (cta_group::2 MMAs) with 256 x 256 tiles, each CTA staging its own 128
// rows of A and half of B and holding its 128 rows of the accumulator. 512 threads in four
// warpgroups:
//   warp 0       TMA producer: A and B K blocks (128 wide) into a 3-stage ring (pair: 4)
//   warp 1       MMA issuer (pair: the leader CTA's, for both CTAs) and TMEM owner: per K
//                block 4 block-scaled MMAs (K = 32 each) into the tile's accumulator
//   warps 4..11  epilogue: at a tile's end each reads its 32 rows x 128 columns of the
//                accumulator, hands it back to the MMA issuer, then rounds to BF16 into
//                swizzled shared memory and stores with the TMA unit
//   warps 12..15 scale writers, one per TMEM lane quadrant: for every K block they write
//                its scale factors into a ring slot of TMEM columns (one slot per pipeline
//                stage, reported on the stage's full barrier beside the TMA bytes, so the
//                MMA issuer waits once and commits once per K block), loading them from
//                global memory as many K blocks ahead as the ring has slots. The MMA reads
//                the factor of A row m from lane m, column m / 32, and that of B column n
//                from lane 32q + n % 32, column n / 32, in the lane quadrant q of the row
//                it computes; each quadrant therefore holds its 32 rows' A factors (written
//                into all 4 A columns of its lanes) and all 256 columns' B factors (8
//                columns). A CTA pair's MMA reads each CTA's factors from that CTA's own
//                TMEM in the same layout (its own rows of A, all of B). A 32-bit cell holds
//                the factors of four K sub-blocks; one scale covers all 128 of K here, so
//                its byte is written four times.
// TMEM: accumulator columns 0..255; ring slot i: A factors at 256 + 16i (4 columns), B
// factors at 260 + 16i (8 columns). Every mbarrier wait is bounded; a wait that gives up
// sets the abort flag and the device status word, and the CTA drains and exits.

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

constexpr int BM = 128, BN = 256, BK = 128;  // BM: rows per CTA (a CTA pair: 256-row tiles)
constexpr int THREADS = 512;
constexpr int EPI_FIRST = 4, EPI_WARPS = 8, SFW_FIRST = 12;
constexpr int A_BYTES = BM * BK;
constexpr int STG_BOX_BYTES = 32 * 128;               // 32 rows x 64 BF16, 128B-swizzled
constexpr int STG_WARP_BYTES = 2 * STG_BOX_BYTES;     // 128 columns per epilogue warp
// PAIR: a cluster of two CTAs computes a 256 x 256 tile with cta_group::2 MMAs; each CTA
// stages its own 128 rows of A and half of B, and holds its 128 rows of the accumulator.
template <bool PAIR>
struct MxCfg {
  static constexpr int STAGES = PAIR ? 4 : 3;
  // One scale-factor ring slot per stage: a K block's factors are written into the slot of
  // its operands' stage and counted on the same full barrier, and the MMA's one commit frees
  // both, so the MMA issuer waits on one barrier and commits one per K block.
  static constexpr int SF_SLOTS = STAGES;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // rows of B this CTA stages
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int TILE_ROWS = PAIR ? 2 * BM : BM;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_STG = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_STG + EPI_WARPS * STG_WARP_BYTES;
  // full/empty per stage, tfull, tempty, drain
  static constexpr int N_BARS = 2 * STAGES + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(OFF_STG % 1024 == 0, "swizzled staging must be 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};
constexpr uint32_t ACC_COL = 0, SF_COL = 256, SF_SLOT_COLS = 16;
static_assert(SF_COL + MxCfg<true>::SF_SLOTS * SF_SLOT_COLS <= 512, "TMEM columns");
constexpr int LAUNCH_REGS = 128;   // 65536 / 512
constexpr int REGS_SMALL = 56;     // warpgroups 0 and 3
constexpr int REGS_EPI = 200;      // warpgroups 1 and 2
static_assert(128 * REGS_SMALL * 2 + 256 * REGS_EPI == THREADS * LAUNCH_REGS, "register split");

// Block-scaled instruction descriptor: E4M3 A and B, K-major, FP32 accumulate, UE8M0 scale
// factors, M x N; sf_a / sf_b pick the byte (K sub-block) of the scale-factor cells.
__host__ __device__ constexpr uint32_t idesc_mx(int m, int n, uint32_t sf_a, uint32_t sf_b) {
  return (sf_b << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(m >> 4) << 24) | (sf_a << 29);
}

__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_mx_pair(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
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

struct MxArgs {
  const uint8_t *As;  // UE8M0 [K/128, M]
  const uint8_t *Bs;  // UE8M0, layout-dependent (see the C declaration)
  int M, N, K;
  int num_m, num_n, kblocks, m_fastest;
  unsigned long long timeout_ns;
  int *status;
};

__device__ int g_mx_status;  // non-zero: a bounded wait gave up since the last read

#ifdef PURO_TEST_HOOKS
// Test builds only, never libpuro_fp8.so: while set, the scale writers withhold their
// arrival for the first K block, so the MMA issuer's bounded wait for the scale factors runs
// out. The failure-detection test uses this to check that a give-up inside this kernel
// reaches the status word and that the kernel drains and exits with the context intact.
__device__ int g_test_mx_skip_sf;
#define PURO_MX_SKIP_SF(seq) (g_test_mx_skip_sf != 0 && (seq) == 0)
#else
#define PURO_MX_SKIP_SF(seq) false
#endif

__device__ __forceinline__ void mx_tile_coords(int tile, const MxArgs &a, int &mt, int &nt) {
  if (a.m_fastest) {
    mt = tile % a.num_m;
    nt = tile / a.num_m;
  } else {
    nt = tile % a.num_n;
    mt = tile / a.num_n;
  }
}

__device__ __forceinline__ uint32_t bf16x2_bits_mx(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

template <int LAYOUT, bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_mx(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, const MxArgs args) {
  using C = MxCfg<PAIR>;
  constexpr int STAGES = C::STAGES, B_BYTES = C::B_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  constexpr int SF_SLOTS = C::SF_SLOTS;
  const uint32_t tfull_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t tempty_bar = tfull_bar + 8u;
  const uint32_t drain_bar = tfull_bar + 16u;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // PAIR: rank 0 of the cluster is the leader: it issues the MMAs for both CTAs and holds the
  // barriers both CTAs report to (the operands' arrival, the scale factors, the accumulator's
  // hand-back). Tiles are walked per cluster; rank r owns rows 128 r .. of a 256-row tile.
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
      // the producer's arrival (with the stage's TMA bytes) and the scale-writer warps' (of
      // both CTAs of a pair)
      mbar_init(full_bar(s), 1 + (PAIR ? 8 : 4));
      mbar_init(empty_bar(s), 1);  // the MMA commit
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
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_SMALL));
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
        int mt, nt;
        mx_tile_coords(tile, args, mt, nt);
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
        if (leader)
          for (int i = 0; i < STAGES; ++i)
            if ((issued >> i) & 1u) mbar_wait(full_bar(i), (issued_parity >> i) & 1u, tmo, nullptr);
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
          if (!mbar_wait(full_bar(s), ph, tmo, abort)) {  // operands and scale factors
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = sbase + C::OFF_A + s * A_BYTES, b_addr = sbase + C::OFF_B + s * B_BYTES;
          const uint32_t sfa = tmem + SF_COL + SF_SLOT_COLS * s, sfb = sfa + 4;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            if constexpr (PAIR)
              mma_mx_pair(tmem + ACC_COL, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k),
                          idesc_mx(2 * BM, BN, k, k), sfa, sfb, acc);
            else
              mma_mx(tmem + ACC_COL, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k),
                     idesc_mx(BM, BN, k, k), sfa, sfb, acc);
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
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_SMALL));
    // ------------------------------------------------------------------ scale writers
    // Loads run SF_SLOTS K blocks ahead of the stores, in a register ring of raw loaded
    // values (3 registers per K block), so their latency is hidden behind the MMAs. A CTA
    // pair reads each CTA's factors from that CTA's own TMEM: its 128 rows of A and all 256
    // columns of B.
    const int quad = warp & 3;
    const uint32_t lane_field = static_cast<uint32_t>(quad * 32) << 16;
    const int nb_total = (args.N + 127) / 128;
    // raw values of one K block: this lane's A byte (row 32 quad + lane of this CTA's rows)
    // and two words for B (wgrad: bytes 8 lane .. 8 lane + 7 of the tile's 256 columns;
    // fprop/dgrad: the bytes of the tile's two 128-column blocks)
    auto fetch = [&](int tile, int kb, uint32_t &ra, uint32_t &rb0, uint32_t &rb1) {
      int mt, nt;
      mx_tile_coords(tile, args, mt, nt);
      const int m = row_base(mt) + 32 * quad + lane;
      ra = m < args.M ? __ldg(args.As + static_cast<int64_t>(kb) * args.M + m) : 127u;
      if (LAYOUT == PURO_WGRAD) {
        const int n0 = nt * BN + 8 * lane;  // N % 8 == 0: the 8 bytes exist or none do
        if (n0 < args.N) {
          const uint2 w = __ldg(reinterpret_cast<const uint2 *>(args.Bs + static_cast<int64_t>(kb) * args.N + n0));
          rb0 = w.x;
          rb1 = w.y;
        } else {
          rb0 = rb1 = 0x7F7F7F7Fu;
        }
      } else {
        const int j0 = 2 * nt, j1 = 2 * nt + 1;
        auto at = [&](int j) -> uint32_t {
          if (j >= nb_total) return 127u;
          return LAYOUT == PURO_FPROP ? __ldg(args.Bs + static_cast<int64_t>(j) * kblocks + kb)
                                      : __ldg(args.Bs + static_cast<int64_t>(kb) * nb_total + j);
        };
        rb0 = at(j0);
        rb1 = at(j1);
      }
    };
    // TMEM cells of one K block from its raw values; each byte is repeated in the four
    // bytes of its cell (one cell serves the four K sub-blocks of the 128-wide block)
    auto store = [&](uint32_t slot, uint32_t ra, uint32_t rb0, uint32_t rb1) {
      uint32_t ca[4], cb[8];
      const uint32_t a = (ra & 0xFFu) * 0x01010101u;
#pragma unroll
      for (int g = 0; g < 4; ++g) ca[g] = a;
      if (LAYOUT == PURO_WGRAD) {
        // column n = 32 g + lane: byte lane & 7 of the words held by lane 4 g + lane / 8
        const uint32_t sel = ((lane & 3u) * 8u), hi = lane & 4u;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int src = 4 * g + (lane >> 3);
          const uint32_t w0 = __shfl_sync(0xffffffffu, rb0, src), w1 = __shfl_sync(0xffffffffu, rb1, src);
          cb[g] = (((hi ? w1 : w0) >> sel) & 0xFFu) * 0x01010101u;
        }
      } else {
        const uint32_t c0 = (rb0 & 0xFFu) * 0x01010101u, c1 = (rb1 & 0xFFu) * 0x01010101u;
#pragma unroll
        for (int g = 0; g < 8; ++g) cb[g] = g < 4 ? c0 : c1;
      }
      tmem_st_x4(tmem + lane_field + SF_COL + SF_SLOT_COLS * slot, ca);
      tmem_st_x8(tmem + lane_field + SF_COL + SF_SLOT_COLS * slot + 4, cb);
    };
    auto advance = [&](int &tile, int &kb) {
      if (++kb == kblocks) kb = 0, tile += tile_step;
    };
    uint32_t ra[SF_SLOTS], rb0[SF_SLOTS], rb1[SF_SLOTS];
    int ft = first_tile, fk = 0;  // the next K block to fetch
#pragma unroll
    for (int d = 0; d < SF_SLOTS; ++d) {
      if (ft < tiles) fetch(ft, fk, ra[d], rb0[d], rb1[d]);
      advance(ft, fk);
    }
    uint32_t sph = 0, seq = 0;  // seq: K blocks stored so far
    bool ok = true;
    int ct = first_tile, ck = 0;  // the next K block to store
    while (ok && ct < tiles) {
#pragma unroll
      for (int d = 0; d < SF_SLOTS; ++d) {  // ring slot d holds the K block fetched into set d
        if (ct < tiles) {
          // warp-uniform outcome: the stores and shuffles below need the whole warp
          if (!__all_sync(0xffffffffu, mbar_wait(empty_bar(d), sph ^ 1u, tmo, abort))) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          store(d, ra[d], rb0[d], rb1[d]);
          if (ft < tiles) fetch(ft, fk, ra[d], rb0[d], rb1[d]);
          advance(ft, fk);
          tmem_wait_st();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0 && !PURO_MX_SKIP_SF(seq)) arrive_leader(full_bar(d));
          advance(ct, ck);
          ++seq;
        }
      }
      sph ^= 1u;
    }
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
    uint32_t it = 0;
    bool ok = true;
    for (int tile = first_tile; tile < tiles; tile += tile_step, ++it) {
      int mt, nt;
      mx_tile_coords(tile, args, mt, nt);
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
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t *r = j < 8 ? r0 : r1;
        const int jj = j & 7;
        const uint32_t addr = stg + (j >> 3) * STG_BOX_BYTES + lane * 128 + (((jj) ^ (lane & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                     "r"(bf16x2_bits_mx(__uint_as_float(r[8 * jj]), __uint_as_float(r[8 * jj + 1]))),
                     "r"(bf16x2_bits_mx(__uint_as_float(r[8 * jj + 2]), __uint_as_float(r[8 * jj + 3]))),
                     "r"(bf16x2_bits_mx(__uint_as_float(r[8 * jj + 4]), __uint_as_float(r[8 * jj + 5]))),
                     "r"(bf16x2_bits_mx(__uint_as_float(r[8 * jj + 6]), __uint_as_float(r[8 * jj + 7])))
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

EncodeTiledFn mx_encode_fn() {
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

bool mx_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem, uint64_t rows,
            uint64_t cols, uint32_t box_rows, uint32_t box_cols) {
  EncodeTiledFn fn = mx_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned long long mx_timeout_ns() {
  static unsigned long long ns = [] {
    const char *e = std::getenv("PURO_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return ns;
}

template <int LAYOUT, bool PAIR>
int launch_mx(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs, uint16_t *C,
              int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  using CF = MxCfg<PAIR>;
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  static PerDevice<int *> status_addr;
  MxArgs args{};
  if (!status_addr.get(args.status, [](int, int *&v) {
        return cudaGetSymbolAddress(reinterpret_cast<void **>(&v), g_mx_status) == cudaSuccess;
      }))
    return PURO_ERR_CUDA;
  CUtensorMap ta, tb, tc;
  if (!mx_map(&ta, Aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, K, BM, BK) ||
      !mx_map(&tb, Bq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, CF::B_ROWS, BK) ||
      !mx_map(&tc, C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, 32, 64))
    return PURO_ERR_CUDA;
  args.As = As;
  args.Bs = Bs;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.kblocks = static_cast<int>(K / BK);
  args.num_m = static_cast<int>((M + CF::TILE_ROWS - 1) / CF::TILE_ROWS);
  args.num_n = static_cast<int>((N + BN - 1) / BN);
  args.m_fastest = M <= N ? 1 : 0;
  args.timeout_ns = mx_timeout_ns();
  const int64_t tiles = static_cast<int64_t>(args.num_m) * args.num_n;
  auto kern = k_gemm_mx<LAYOUT, PAIR>;
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
  // (otherwise the epilogue's setmaxnreg.inc could wait forever); shared memory opt-in; for
  // a CTA pair, the clusters that can be resident at once (the persistent grid's size).
  static PerDevice<int> prepared;
  int prep = PURO_ERR_CUDA;
  if (!prepared.get(prep, [&](int, int &v) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
        if (fa.numRegs != LAUNCH_REGS) {
          std::fprintf(stderr, "puro_fp8: MX GEMM kernel built with %d registers (expected %d); not launched\n",
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
            std::fprintf(stderr, "puro_fp8: no CTA pair of the MX GEMM kernel fits on this device\n");
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
    e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, args);
    if (e == cudaSuccess) e = cudaGetLastError();
  } else {
    grid = static_cast<int>(tiles < sms ? tiles : sms);
    kern<<<grid, THREADS, CF::SMEM_BYTES, stream>>>(ta, tb, tc, args);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    std::fprintf(stderr, "puro_fp8: MX GEMM launch (grid %d): %s\n", grid, cudaGetErrorString(e));
    return PURO_ERR_LAUNCH;
  }
  return PURO_OK;
}

// CTA pairs unless the output has at most 128 rows; PURO_MX_PAIR=0 or 1 forces one of them
// (read once per process).
bool mx_use_pair(int64_t M) {
  static const int mode = [] {
    const char *e = std::getenv("PURO_MX_PAIR");
    return e == nullptr ? -1 : std::atoi(e);
  }();
  if (mode == 0) return false;
  if (mode == 1) return true;
  return M > BM;
}

template <int LAYOUT>
int launch_mx_layout(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs, uint16_t *C,
                     int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
  return mx_use_pair(M) ? launch_mx<LAYOUT, true>(Aq, As, Bq, Bs, C, M, N, K, stream)
                        : launch_mx<LAYOUT, false>(Aq, As, Bq, Bs, C, M, N, K, stream);
}

}  // namespace

int launch_gemm_mx(const uint8_t *Aq, const uint8_t *As, const uint8_t *Bq, const uint8_t *Bs, uint16_t *C,
                   int64_t M, int64_t N, int64_t K, int layout, cudaStream_t stream) {
  switch (layout) {
    case PURO_FPROP: return launch_mx_layout<PURO_FPROP>(Aq, As, Bq, Bs, C, M, N, K, stream);
    case PURO_DGRAD: return launch_mx_layout<PURO_DGRAD>(Aq, As, Bq, Bs, C, M, N, K, stream);
    case PURO_WGRAD: return launch_mx_layout<PURO_WGRAD>(Aq, As, Bq, Bs, C, M, N, K, stream);
    default: return PURO_ERR_LAYOUT;
  }
}

int read_and_clear_mx_status(cudaStream_t stream, int *status_out) {
  int host = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_mx_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_mx_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return PURO_ERR_CUDA;
  *status_out = host;
  return PURO_OK;
}

}  // namespace puro

#ifdef PURO_TEST_HOOKS
extern "C" __attribute__((visibility("default"))) int puro_test_set_mx_skip_sf(int on) {
  return cudaMemcpyToSymbol(puro::g_test_mx_skip_sf, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
