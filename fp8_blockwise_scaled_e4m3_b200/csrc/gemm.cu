// Blockwise-FP8 GEMM for sm_100a: TMA -> swizzled shared memory -> tcgen05 MMA (E4M3,
// FP32 accumulate in TMEM) -> FP32 scale promotion on CUDA cores -> BF16.
//
// "Paper walkthrough: Puro-2B ...", section "Lever 2: use blockwise FP8 from step zero":
// the linear-layer GEMMs run in FP8 with local scales, one per 128 elements along the
// reduction dimension for activations and gradients and one per 128x128 block for
// weights. The scales change every 128 elements of K, so each 128-wide K block is
// accumulated on its own by the tensor cores (FP32 partial in TMEM) and added into the
// running FP32 sum with its two scales:
//     C[m, n] = sum_kb  sA(kb, m) * sB(kb, n) * P_kb[m, n],   P_kb = Aq[m, kb] . Bq[n, kb]
//
// One persistent CTA per SM, tiles of 128 x 256, warp-specialised:
//   warp 0      TMA producer: A and B tiles of one K block per ring stage (3 stages)
//   warps 1, 3  MMA issuers, one per TMEM buffer: warp 1 takes the even K blocks (buffer
//               0), warp 3 the odd ones (buffer 1); each issues 4 x tcgen05.mma (K = 32
//               each) per K block into its 256-column buffer, committed to the stage's
//               "empty" barrier and the buffer's "full" barrier. One issuing thread
//               sustains only about 880 clk per K block (4 MMAs + its loop), against 511 of
//               tensor work; two issue at the full rate. Warp 1 also owns the TMEM allocation.
//   warp 2      scale loader: for every K block, the tile's 128 row scales of A and its
//               column scales of B (one per 128-column block, or one per column for
//               wgrad) are copied with cp.async into a shared-memory ring (16-byte copies
//               where the scale rows are 16-byte aligned), so the promotion never waits
//               on a global load
//   warps 4..11 promotion + epilogue: warp w owns TMEM lanes 32*(w%4) .. +31 (output rows)
//               and columns 128*((w-4)/4) .. +127; partial * (sA * sB) is added into FP32
//               registers with packed FP32x2 FMAs (fprop/dgrad: one row per thread, read
//               in the 32x32b shape; wgrad: 4 rows x 32 columns per thread, read in the
//               16x256b shape, see below); at the end of the tile each warp rounds its
//               sums to BF16 into a 128B-swizzled staging buffer and hands it to TMA
//               tensor stores, so the warps go straight back to the next tile (stores
//               outside M x N are clipped by the TMA unit).
// Every mbarrier wait is bounded (wall-clock limit plus an iteration cap). A wait that
// gives up raises a CTA-wide abort flag and the device status word; all warps then
// leave their loops, in-flight copies and MMAs are waited for (bounded), and TMEM is
// freed before the CTA exits.

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
#include "quant_math.cuh"

namespace puro {
namespace {

constexpr int BM = 128;
constexpr int BK = 128;                  // one scale block of K per stage
constexpr int SC_STAGES = 4;  // scale-ring slots of KPS K blocks each
constexpr int EPI_WARPS = 8;
constexpr int EPI_FIRST_WARP = 4;               // warps 0-3 form warpgroup 0
constexpr int THREADS = 32 * (EPI_FIRST_WARP + EPI_WARPS);  // 384: three warpgroups
// Register split. The CTA is launched with LAUNCH_REGS per thread (what ptxas gets for
// 384 threads and one CTA per SM); warpgroup 0 (TMA, MMA, scale loader, one idle warp) gives
// registers back and the two promotion warpgroups take them:
//   128 * producer + 256 * consumer == 384 * LAUNCH_REGS  (64512)
// and per SM sub-partition (one warp of each warpgroup) 32 * (producer + 2 * consumer)
// <= 16384. Every promotion thread holds 128 FP32 sums.
constexpr int LAUNCH_REGS = 168;
template <int LAYOUT>
struct RegSplit {
  static constexpr int producer = 56;
  static constexpr int consumer = 224;
  static_assert(128 * producer + 256 * consumer == THREADS * LAUNCH_REGS,
                "register split must add up to the launch allocation");
  static_assert(32 * (producer + 2 * consumer) <= 16384, "per sub-partition register file");
};
constexpr int A_BYTES = BM * BK;          // 16 KB
constexpr int STG_BOX_BYTES = 32 * 128;   // 32 rows x 64 BF16 columns, 128B-swizzled

// Tile width TN (256 or 128) sets the rest. TMEM holds 512 FP32 columns, i.e.
// 512 / TN partial buffers; each promotion warp owns TN / 2 columns of one lane quadrant.
// PAIR: a cluster of two CTAs computes a 256 x TN tile with cta_group::2 MMAs. Each CTA
// holds its own 128 rows of A and half (TN / 2 rows) of B in shared memory and receives
// its 128 rows x TN columns of the product in its TMEM, so per output element each SM
// stages and reads half as many B bytes as a single CTA does.
template <int LAYOUT, int TN, bool PAIR>
struct Cfg {
  static constexpr int BN = TN;
  static constexpr int NBUF = 512 / TN;            // TMEM partial buffers
  static constexpr int WCOLS = TN / 2;             // columns per promotion warp
  static constexpr int B_ROWS = PAIR ? TN / 2 : TN;  // rows of B this CTA stages
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGES = PAIR ? (TN == 128 ? 6 : 4) : (TN == 256 ? 3 : 5);
  // Scale-ring slot, KPS K blocks: KPS x 128 row scales of A, then KPS x SB_STRIDE
  // scales of B (TN column scales for wgrad, one per 128-column block otherwise).
  static constexpr int SB_STRIDE = LAYOUT == PURO_WGRAD ? TN : 4;
  // K blocks of scales per slot (wgrad's 256 column scales per K block fill shared
  // memory faster, so its slots are half as deep)
  static constexpr int KPS = LAYOUT == PURO_WGRAD ? 2 : 4;
  static constexpr int SC_SLOT_FLOATS = KPS * (BM + SB_STRIDE);
  static constexpr int SC_SLOT_BYTES = SC_SLOT_FLOATS * 4;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC = idesc_e4m3_f32(PAIR ? 2 * BM : BM, TN);
  static constexpr int STG_WARP_BYTES = (WCOLS / 64) * STG_BOX_BYTES;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_STG = OFF_B + STAGES * B_BYTES;  // output staging, one per warp
  static constexpr int OFF_SC = OFF_STG + EPI_WARPS * STG_WARP_BYTES;
  static constexpr int OFF_BAR = OFF_SC + SC_STAGES * SC_SLOT_BYTES;
  static constexpr int N_BARS = 2 * STAGES + 2 * NBUF + 2 * SC_STAGES + 2;  // + a drain barrier per MMA issuer
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(OFF_STG % 1024 == 0, "swizzled staging must be 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Tile widths: 128 x 256 for single CTAs and 256 x 256 for CTA pairs, in every layout (two
// 256-column TMEM buffers). Measured on B200 and set aside: 128-wide tiles with four
// buffers, 25-30% slower for single CTAs (shared-memory bandwidth) and 12-17% slower as
// 256 x 128 pair tiles (MMA issue rate and shared-memory bandwidth).
template <int LAYOUT, bool PAIR>
struct TileFor {
  static constexpr int TN = 256;
};

// One GEMM of a launch. A launch serves up to G of them (the same layout): their tiles are
// numbered one after the other, problem p owning tiles [tile_begin, tile_begin + num_m *
// num_n), and the persistent CTAs walk that joint sequence.
struct GemmArgs {
  const float *As;
  const float *Bs;
  uint16_t *C;
  int M, N, K;
  int num_m, num_n, kblocks, m_fastest;
  int vec_a;  // As rows are 16-byte aligned (As aligned, M % 4 == 0): 16-byte scale copies
  int vec_b;  // wgrad: Bs rows are 16-byte aligned (Bs aligned; N % 8 == 0 always)
  uint8_t *Cq;  // QOUT: 1x128 codes of the BF16 output along N, [M, N] dense
  float *Cs;    // QOUT: their scales, [N/128, M]
  int tile_begin;
};

// Kernel parameters: the problems' tensor maps (A, B and C of problem p at index p) and
// arguments, passed by value as a __grid_constant__ (the TMA unit reads the maps from the
// parameter space).
template <int G>
struct alignas(64) GemmParams {
  CUtensorMap tmA[G], tmB[G], tmC[G];
  GemmArgs prob[G];
  int count;  // problems in use
  int tiles;  // tiles of all problems
  unsigned long long timeout_ns;
  int *status;
};
constexpr int GROUP_MAX = 4;  // problems per grouped launch

__device__ int g_status;  // non-zero: a bounded wait gave up since the last read

#ifdef PURO_TEST_HOOKS
// Test builds only, never libpuro_fp8.so: while set, the promotion warps do not hand TMEM
// buffer 0 back after its first use, so the MMA warp's bounded wait for it runs out. The
// failure-detection test uses this to check that a give-up inside the GEMM reaches the
// status word and that the kernel drains and exits with the context intact.
__device__ int g_test_skip_release;
#define PURO_SKIP_RELEASE(use) (g_test_skip_release != 0 && (use) == 0)
#else
#define PURO_SKIP_RELEASE(use) false
#endif

// Problem p of global tile `tile` and the tile's coordinates within that problem.
template <int G>
__device__ __forceinline__ int locate_tile(int tile, const GemmParams<G> &prm, int &mt, int &nt);

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs &a, int &mt, int &nt) {
  if (a.m_fastest) {
    mt = tile % a.num_m;
    nt = tile / a.num_m;
  } else {
    nt = tile % a.num_n;
    mt = tile / a.num_n;
  }
}

template <int G>
__device__ __forceinline__ int locate_tile(int tile, const GemmParams<G> &prm, int &mt, int &nt) {
  int p = 0;  // problems are numbered in tile order: count the ones that begin at or before `tile`
#pragma unroll
  for (int q = 1; q < G; ++q) p += (q < prm.count && tile >= prm.prob[q].tile_begin) ? 1 : 0;
  tile_coords(tile - prm.prob[p].tile_begin, prm.prob[p], mt, nt);
  return p;
}

__device__ __forceinline__ void raise_abort(volatile int *abort, int *status) {
  *abort = 1;
  atomicOr(status, 1);
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// ACC32: instead of storing BF16, add the FP32 result into an FP32 C (main-gradient
// accumulation of wgrad) with TMA reduce-add.
// QOUT (fprop/dgrad): the epilogue also quantises the BF16 output row-wise, 1x128 along N:
// a promotion thread holds one output row x 128 columns, exactly one group, so the group's
// amax, scale and codes come from the thread's own registers (the same arithmetic as the
// separate 1x128 quantiser, applied to the same BF16 values).
template <int LAYOUT, int TN, bool ACC32, bool PAIR, bool QOUT, int G>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_blockwise(const __grid_constant__ GemmParams<G> prm) {
  using C = Cfg<LAYOUT, TN, PAIR>;
  constexpr int BN = C::BN, NBUF = C::NBUF, STAGES = C::STAGES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int OFF_A = C::OFF_A, OFF_B = C::OFF_B, OFF_STG = C::OFF_STG, OFF_SC = C::OFF_SC;
  constexpr int OFF_BAR = C::OFF_BAR, OFF_MISC = C::OFF_MISC, N_BARS = C::N_BARS;
  constexpr int KPS = C::KPS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + NBUF + b); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 * NBUF + s); };
  auto sempty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 * NBUF + SC_STAGES + s); };
  auto drain_bar = [&](int issuer) { return bar0 + 8u * (N_BARS - 2 + issuer); };
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  const float *sc_smem = reinterpret_cast<const float *>(smem + OFF_SC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // PAIR: rank 0 of the cluster is the leader (it issues the MMAs for both CTAs and holds
  // the barriers they report to); tiles are walked per cluster.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int first_tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // first output row of this CTA in tile row mt
  auto row_base = [&](int mt) { return PAIR ? mt * 2 * BM + static_cast<int>(rank) * BM : mt * BM; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PAIR ? 2 * EPI_WARPS : EPI_WARPS);  // PAIR: both CTAs' warps
    }
    for (int s = 0; s < SC_STAGES; ++s) {
      mbar_init(sfull_bar(s), 32);  // one cp.async completion arrival per loader lane
      mbar_init(sempty_bar(s), EPI_WARPS);
    }
    mbar_init(drain_bar(0), 1);
    mbar_init(drain_bar(1), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane < prm.count) {
    prefetch_tensormap(&prm.tmA[lane]);
    prefetch_tensormap(&prm.tmB[lane]);
    prefetch_tensormap(&prm.tmC[lane]);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
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

  const int tiles = prm.tiles;
  const uint64_t tmo = prm.timeout_ns;

  if (warp < EPI_FIRST_WARP) {
    // Each role's code sits inside the branch that set its register limit, so ptxas
    // allocates the promotion path with the consumer share and this one with the producer's.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<LAYOUT>::producer));
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage bit masks
      bool ok = true;
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
        int mt, nt;
        const int p = locate_tile(tile, prm, mt, nt);
        const CUtensorMap *tmA = &prm.tmA[p];
        const CUtensorMap *tmB = &prm.tmB[p];
        const int kblocks = prm.prob[p].kblocks;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(s), ph ^ 1u, tmo, abort)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            // Both CTAs' loads are counted on the leader's barrier, which the leader arms
            // with the pair's bytes. A peer's load for the next use of a stage can only
            // start after the MMA that read the stage completed (the empty barrier), so
            // it never lands in the leader's barrier before the previous phase is over.
            const uint32_t fb = map_to_rank(full_bar(s), 0);
            if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * (A_BYTES + B_BYTES));
            tma_load_2d_pair(sbase + OFF_A + s * A_BYTES, tmA, fb, kb * BK, row_base(mt));
            tma_load_2d_pair(sbase + OFF_B + s * B_BYTES, tmB, fb, kb * BK,
                             nt * BN + static_cast<int>(rank) * C::B_ROWS);
          } else {
            mbar_arrive_expect_tx(full_bar(s), A_BYTES + B_BYTES);
            tma_load_2d(sbase + OFF_A + s * A_BYTES, tmA, full_bar(s), kb * BK, mt * BM);
            tma_load_2d(sbase + OFF_B + s * B_BYTES, tmB, full_bar(s), kb * BK, nt * BN);
          }
          issued |= 1u << s;
          issued_parity = (issued_parity & ~(1u << s)) | (ph << s);
          if (++s == STAGES) s = 0, ph ^= 1u;
        }
      }
      if (!ok) {
        raise_abort(abort, prm.status);
        // Let every issued tensor load land before the CTA can exit. (A peer's loads are
        // counted on the leader's barriers, which the leader drains; the peer stays alive
        // until then through the cluster barrier at the end of the kernel.)
        if (leader)
          for (int i = 0; i < STAGES; ++i)
            if ((issued >> i) & 1u) mbar_wait(full_bar(i), (issued_parity >> i) & 1u, tmo, nullptr);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    static_assert(NBUF % 2 == 0, "two MMA issuers take alternate K blocks");
    if (lane == 0 && leader) {  // PAIR: the leader issues for both CTAs
      const uint32_t mine = warp == 1 ? 0u : 1u;  // the parity of this issuer's K blocks
      uint32_t use = 0;                            // K blocks of this CTA so far, both issuers
      bool ok = true;
      for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
        int mt, nt;
        const int kblocks = prm.prob[locate_tile(tile, prm, mt, nt)].kblocks;
        for (int kb = 0; kb < kblocks; ++kb, ++use) {
          if ((use & 1u) != mine) continue;
          const int s = static_cast<int>(use % STAGES);
          const uint32_t ph = (use / STAGES) & 1u;
          const uint32_t b = use % NBUF;
          // The stage's operands are normally in long before its TMEM buffer is free, so
          // that wait comes first and its cost overlaps the promotion still draining the
          // buffer.
          if (!mbar_wait(full_bar(s), ph, tmo, abort) ||
              !mbar_wait(tempty_bar(b), ((use / NBUF) & 1u) ^ 1u, tmo, abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d = tmem + b * BN;
          const uint32_t a_addr = sbase + OFF_A + s * A_BYTES;
          const uint32_t b_addr = sbase + OFF_B + s * B_BYTES;
          if constexpr (PAIR) {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_e4m3_pair(d, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k), C::IDESC,
                            k > 0 ? 1u : 0u);
            mma_commit_pair_mc(empty_bar(s), 0x3);  // both CTAs' stage s is free again
            mma_commit_pair_mc(tfull_bar(b), 0x3);  // both CTAs' partial is in TMEM
          } else {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_e4m3(d, sdesc_k_sw128(a_addr + 32 * k), sdesc_k_sw128(b_addr + 32 * k), C::IDESC,
                       k > 0 ? 1u : 0u);
            mma_commit(empty_bar(s));
            mma_commit(tfull_bar(b));
          }
        }
      }
      if (!ok) {
        raise_abort(abort, prm.status);
        // arrives once every MMA this thread issued has finished
        if constexpr (PAIR)
          mma_commit_pair(drain_bar(mine));
        else
          mma_commit(drain_bar(mine));
        mbar_wait(drain_bar(mine), 0, tmo, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale loader
    // Scales outside the matrix are zero-filled, so the promotion needs no bounds checks.
    int ss = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
      int mt, nt;
      const GemmArgs &args = prm.prob[locate_tile(tile, prm, mt, nt)];
      const int kblocks = args.kblocks;
      const int nb_total = (args.N + 127) / 128;
      const int m_first = row_base(mt);
      for (int kb0 = 0; kb0 < kblocks; kb0 += KPS) {
        if (!mbar_wait(sempty_bar(ss), sph ^ 1u, tmo, abort)) {
          ok = false;
          break;
        }
        const uint32_t dst = sbase + OFF_SC + ss * C::SC_SLOT_BYTES;
        const int nk = kblocks - kb0 < KPS ? kblocks - kb0 : KPS;
        for (int q = 0; q < nk; ++q) {
          const int kb = kb0 + q;
          const float *a_row = args.As + static_cast<int64_t>(kb) * args.M;
          if (args.vec_a) {
            // one 16-byte copy per lane: rows 4 * lane .. +3 of the tile
            const int m0 = m_first + 4 * lane;
            const int valid = min(max(args.M - m0, 0), 4);
            cp_async_16(dst + 4 * (q * BM) + 16 * lane, valid > 0 ? a_row + m0 : args.As, 4 * valid);
          } else {
#pragma unroll 1
            for (int i = lane; i < BM; i += 32) {
              const int m = m_first + i;
              const bool v = m < args.M;
              cp_async_4(dst + 4 * (q * BM + i), v ? a_row + m : args.As, v);
            }
          }
          const uint32_t dsb = dst + 4 * (KPS * BM + q * C::SB_STRIDE);
          if (LAYOUT == PURO_WGRAD) {
            const float *b_row = args.Bs + static_cast<int64_t>(kb) * args.N;
            if (args.vec_b) {
#pragma unroll
              for (int h = 0; h < BN / 128; ++h) {
                const int i = 4 * (lane + 32 * h);
                const int n0 = nt * BN + i;
                const int valid = min(max(args.N - n0, 0), 4);
                cp_async_16(dsb + 4 * i, valid > 0 ? b_row + n0 : args.Bs, 4 * valid);
              }
            } else {
#pragma unroll 1
              for (int i = lane; i < BN; i += 32) {
                const int n = nt * BN + i;
                const bool v = n < args.N;
                cp_async_4(dsb + 4 * i, v ? b_row + n : args.Bs, v);
              }
            }
          } else if (lane < BN / 128) {
            const int nb = nt * (BN / 128) + lane;
            const bool v = nb < nb_total;
            const float *src = LAYOUT == PURO_FPROP
                                   ? args.Bs + static_cast<int64_t>(nb) * kblocks + kb
                                   : args.Bs + static_cast<int64_t>(kb) * nb_total + nb;
            cp_async_4(dsb + 4 * lane, v ? src : args.Bs, v);
          }
        }
        cp_async_mbar_arrive_noinc(sfull_bar(ss));
        if (++ss == SC_STAGES) ss = 0, sph ^= 1u;
      }
    }
    if (!ok) raise_abort(abort, prm.status);
    cp_async_wait_all();  // no copy may land after the CTA has exited
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<LAYOUT>::consumer));
    // ------------------------------------------------------------ promotion + epilogue
    constexpr int WCOLS = C::WCOLS;
    const int quad = warp & 3;
    const int half = (warp - EPI_FIRST_WARP) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t use = 0;
    int ss = 0;
    uint32_t sph = 0;
    bool ok = true;
    // PAIR: the TMEM buffer goes back to the leader's MMA issuer, which waits for both CTAs
    const uint32_t tempty_target0 = PAIR ? map_to_rank(tempty_bar(0), 0) : tempty_bar(0);
    for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
      int kblocks;
      {
        int mt, nt;
        kblocks = prm.prob[locate_tile(tile, prm, mt, nt)].kblocks;
      }
      uint64_t acc[WCOLS / 2];
#pragma unroll
      for (int i = 0; i < WCOLS / 2; ++i) acc[i] = 0;
      float fq[KPS];  // fprop/dgrad: the slot's factors sA * sB, K block kb's first

      for (int kb = 0; kb < kblocks; ++kb, ++use) {
        const uint32_t b = use % NBUF;
        // Scales come KPS K blocks per ring slot, well ahead of the partials: one wait at
        // the slot's first K block, one release after its last.
        const int kq = kb % KPS;
        if (kq == 0 && !mbar_wait(sfull_bar(ss), sph, tmo, abort)) {
          ok = false;
          break;
        }
        const float *slot = sc_smem + ss * C::SC_SLOT_FLOATS;
        const bool slot_done = kq == KPS - 1 || kb == kblocks - 1;
        auto release_slot = [&]() {
          if (slot_done) {
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty_bar(ss));
            if (++ss == SC_STAGES) ss = 0, sph ^= 1u;
          }
        };
        if constexpr (LAYOUT != PURO_WGRAD) {
          // One scalar factor per thread and K block: partial * (sA * sB). All KPS factors
          // of a slot are read at its first K block (one shared-memory latency per slot,
          // off the per-K-block chain) and the slot goes back to the loader at once.
          static_assert(WCOLS == 128 || WCOLS == 64, "fprop/dgrad promotion: 64 or 128 columns per warp");
          if (kq == 0) {
            const int sbi = (half * WCOLS) / 128;
#pragma unroll
            for (int q = 0; q < KPS; ++q) fq[q] = slot[q * BM + row] * slot[KPS * BM + q * C::SB_STRIDE + sbi];
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty_bar(ss));
            if (++ss == SC_STAGES) ss = 0, sph ^= 1u;
          }
          const uint64_t s2 = pack2(fq[0], fq[0]);
#pragma unroll
          for (int q = 0; q + 1 < KPS; ++q) fq[q] = fq[q + 1];
          if (!mbar_wait(tfull_bar(b), (use / NBUF) & 1u, tmo, abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t taddr = tmem + lane_base + b * BN + half * WCOLS;
          // 64-column TMEM loads, one wait each; the buffer goes back to the MMA issuer once
          // the last chunk is in registers, before that chunk's FMAs. (With 32-column loads,
          // each chunk's FMAs overlapping the next chunk's load, it measured 1-2% slower.)
#pragma unroll
          for (int c = 0; c < WCOLS / 64; ++c) {
            uint32_t r[64];
            tmem_ld_64cols(taddr + 64 * c, r);
            tmem_wait_ld_dep(r);
            if (c == WCOLS / 64 - 1) {
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0 && !PURO_SKIP_RELEASE(use)) {
                if constexpr (PAIR)
                  mbar_arrive_cluster(tempty_target0 + 8u * b);
                else
                  mbar_arrive(tempty_bar(b));
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[32 * c + i] =
                  ffma2(pack2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), s2, acc[32 * c + i]);
          }
        } else {
          // wgrad: a factor per element, sA[row] * sB[column]. The partials are read in the
          // 16x256b shape, so a thread holds 4 rows x 32 columns of its warp's 32 x 128
          // block (rows g, g+8, g+16, g+24 with g = lane / 4; columns 8p + c, 8p + c + 1
          // with c = 2 * (lane % 4)) and needs 4 row scales and 32 column scales per K
          // block instead of 1 and 128: a quarter of the shared-memory traffic.
          static_assert(WCOLS == 128, "wgrad promotion reads 128 columns per warp");
          const int g = lane >> 2, c = 2 * (lane & 3);
          const float *sav = slot + kq * BM + quad * 32 + g;
          const float sa0 = sav[0], sa1 = sav[8], sa2 = sav[16], sa3 = sav[24];
          const float *sbv = slot + KPS * BM + kq * C::SB_STRIDE + half * WCOLS + c;
          uint64_t sbp[16];  // column pairs 8p + c, 8p + c + 1
#pragma unroll
          for (int p = 0; p < 16; ++p) sbp[p] = *reinterpret_cast<const uint64_t *>(sbv + 8 * p);
          release_slot();
          if (!mbar_wait(tfull_bar(b), (use / NBUF) & 1u, tmo, abort)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t taddr = tmem + lane_base + b * BN + half * WCOLS;
          const uint64_t s0 = pack2(sa0, sa0), s1 = pack2(sa1, sa1);
          const uint64_t s2 = pack2(sa2, sa2), s3 = pack2(sa3, sa3);
          // 4 loads of 16 lanes x 64 columns: q = 2 * column half + lane half;
          // double-buffered. (8 loads of 32 columns measured 2-3% slower.)
          auto apply = [&](int q, const uint32_t (&r)[32]) {
            const int lh = q & 1, ch = q >> 1;
            const uint64_t sx = lh ? s2 : s0, sy = lh ? s3 : s1;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int p = 8 * ch + j;
              acc[(2 * lh) * 16 + p] = ffma2(pack2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])),
                                             fmul2(sx, sbp[p]), acc[(2 * lh) * 16 + p]);
              acc[(2 * lh + 1) * 16 + p] =
                  ffma2(pack2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])),
                        fmul2(sy, sbp[p]), acc[(2 * lh + 1) * 16 + p]);
            }
          };
          auto issue = [&](int q, uint32_t (&r)[32]) {
            tmem_ld_16x256b_x8(taddr + (static_cast<uint32_t>(16 * (q & 1)) << 16) + 64 * (q >> 1), r);
          };
          uint32_t ra[32], rb[32];
          issue(0, ra);
          tmem_wait_ld_dep(ra);
#pragma unroll
          for (int q = 0; q < 4; q += 2) {
            issue(q + 1, rb);
            apply(q, ra);
            tmem_wait_ld_dep(rb);
            if (q + 2 < 4) {
              issue(q + 2, ra);
            } else {
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0 && !PURO_SKIP_RELEASE(use)) {
                if constexpr (PAIR)
                  mbar_arrive_cluster(tempty_target0 + 8u * b);
                else
                  mbar_arrive(tempty_bar(b));
              }
            }
            apply(q + 1, rb);
            if (q + 2 < 4) tmem_wait_ld_dep(ra);
          }
        }
      }
      if (!ok) break;
      // The tile's problem and position, looked up again only now (registers are scarce
      // during the K loop).
      int mt, nt;
      const int p = locate_tile(tile, prm, mt, nt);
      const GemmArgs &args = prm.prob[p];
      const CUtensorMap *tmC = &prm.tmC[p];
      const int m_first = row_base(mt);
      const int n_base = nt * BN + half * WCOLS;  // first column of this warp
      // Stage this warp's 32 rows x WCOLS columns as BF16 (64-column boxes, 16-byte
      // chunk c of row r at chunk position c ^ (r % 8)) and store them with the TMA unit.
      const uint32_t stg = sbase + OFF_STG + (warp - EPI_FIRST_WARP) * C::STG_WARP_BYTES;
      if (lane == 0) bulk_wait_group_read<0>();  // the previous tile's stores left the buffer
      __syncwarp();
      if constexpr (ACC32) {
        // FP32 out: four boxes of 32 rows x 32 columns (128-byte rows, 16-byte chunk k of
        // row r at position k ^ (r % 8)), staged two at a time in the warp's 8 KB and
        // added into C by the TMA unit.
        static_assert(LAYOUT == PURO_WGRAD && WCOLS == 128, "FP32 accumulation is the wgrad epilogue");
        const int g = lane >> 2, c = 2 * (lane & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1) {
            if (lane == 0) bulk_wait_group_read<0>();  // the first two boxes left the buffer
            __syncwarp();
          }
#pragma unroll
          for (int bb = 0; bb < 2; ++bb) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int p = 4 * (2 * h + bb) + q;  // acc pair: columns 8p + c, 8p + c + 1
                const int r = g + 8 * x;
                const int k16 = 2 * q + (c >> 2);
                const uint32_t addr = stg + bb * STG_BOX_BYTES + r * 128 + ((k16 ^ (r & 7)) << 4) + 4 * (c & 3);
                float lo, hi;
                unpack2(acc[16 * x + p], lo, hi);
                asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(lo), "f"(hi) : "memory");
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int row0 = m_first + quad * 32;
            if (row0 < args.M) {
#pragma unroll
              for (int bb = 0; bb < 2; ++bb) {
                const int col = n_base + 32 * (2 * h + bb);
                if (col < args.N) tma_reduce_add_2d(tmC, stg + bb * STG_BOX_BYTES, col, row0);
              }
            }
            bulk_commit_group();
          }
        }
      } else {
      if constexpr (LAYOUT != PURO_WGRAD) {
        // thread = row `lane`, columns in order
        uint32_t w[WCOLS / 2];  // the row's BF16 pairs
#pragma unroll
        for (int j = 0; j < WCOLS / 8; ++j) {
          float v[8];
          unpack2(acc[4 * j], v[0], v[1]);
          unpack2(acc[4 * j + 1], v[2], v[3]);
          unpack2(acc[4 * j + 2], v[4], v[5]);
          unpack2(acc[4 * j + 3], v[6], v[7]);
          w[4 * j] = bf16x2_bits(v[0], v[1]);
          w[4 * j + 1] = bf16x2_bits(v[2], v[3]);
          w[4 * j + 2] = bf16x2_bits(v[4], v[5]);
          w[4 * j + 3] = bf16x2_bits(v[6], v[7]);
          const uint32_t addr =
              stg + (j >> 3) * STG_BOX_BYTES + lane * 128 + (((j & 7) ^ (lane & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[4 * j]),
                       "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                       : "memory");
        }
        if constexpr (QOUT) {
          static_assert(WCOLS == 128, "one 1x128 group per thread");
          const int grow = m_first + row;
          if (grow < args.M && n_base < args.N) {
            // amax over the 128 BF16 values (exact), in four independent chains
            uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < WCOLS / 2; ++i) m4[i & 3] = bf16x2_absmax(m4[i & 3], w[i]);
            const float amax =
                bf16x2_absmax_to_f32(bf16x2_absmax(bf16x2_absmax(m4[0], m4[1]), bf16x2_absmax(m4[2], m4[3])));
            float sq;
            BlockDivider dq;
            bool fast;
            block_scale_fast(amax, sq, dq, fast);
            if (!fast) block_scale(amax, sq, dq);  // tiny, infinite or NaN amax
            const uint64_t nr2 = pack2(-dq.r, -dq.r), s2q = pack2(dq.s, dq.s);
            uint8_t *qrow = args.Cq + static_cast<int64_t>(grow) * args.N + n_base;
#pragma unroll
            for (int k = 0; k < WCOLS / 16; ++k) {
              uint32_t q[4];
#pragma unroll
              for (int t = 0; t < 4; ++t)
                q[t] = fast ? block_codes4_fast(w[8 * k + 2 * t], w[8 * k + 2 * t + 1], nr2, s2q)
                            : block_codes4(w[8 * k + 2 * t], w[8 * k + 2 * t + 1], dq);
              asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(qrow + 16 * k), "r"(q[0]),
                           "r"(q[1]), "r"(q[2]), "r"(q[3])
                           : "memory");
            }
            args.Cs[static_cast<int64_t>(n_base / 128) * args.M + grow] = sq;
          }
        }
      } else {
        // 16x256b ownership: acc[8x + j] is row g + 8x, columns 8j + c, 8j + c + 1; one
        // 4-byte BF16 pair per store, bank-conflict free under the swizzle.
        const int g = lane >> 2, c = 2 * (lane & 3);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            float lo, hi;
            unpack2(acc[16 * x + p], lo, hi);
            const int r = g + 8 * x, j = p & 7;
            const uint32_t addr = stg + (p >> 3) * STG_BOX_BYTES + r * 128 + ((j ^ (r & 7)) << 4) + 2 * c;
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(bf16x2_bits(lo, hi)) : "memory");
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int row0 = m_first + quad * 32;
        if (row0 < args.M) {
#pragma unroll
          for (int box = 0; box < WCOLS / 64; ++box)
            if (n_base + 64 * box < args.N)
              tma_store_2d(tmC, stg + box * STG_BOX_BYTES, n_base + 64 * box, row0);
        }
        bulk_commit_group();
      }
      }  // BF16 store
    }
    if (lane == 0) bulk_wait_group_all();  // stores complete before the CTA exits
    if (!ok) raise_abort(abort, prm.status);
  }

  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync();  // neither CTA leaves while the other may still use its shared memory or TMEM
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
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

// Row-major [rows, cols] matrix of `elem` bytes per element, box [box_rows, box_cols].
bool make_map(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem,
              uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
              CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

// Device address of g_status on the current device (looked up once per device).
int *device_status_ptr() {
  static PerDevice<int *> cache;
  int *p = nullptr;
  if (!cache.get(p, [](int, int *&v) {
        return cudaGetSymbolAddress(reinterpret_cast<void **>(&v), g_status) == cudaSuccess;
      }))
    return nullptr;
  return p;
}

// Which kernel shape serves a GEMM: the CTA-pair kernel (256-row tiles) unless the output
// has at most 128 rows. PURO_GEMM_PAIR=0 or 1 forces one of them (read once per process).
bool use_pair(int64_t M) {
  static const int mode = [] {
    const char *e = std::getenv("PURO_GEMM_PAIR");
    return e == nullptr ? -1 : std::atoi(e);
  }();
  if (mode == 0) return false;
  if (mode == 1) return true;
  return M > BM;
}

// One GEMM as the host hands it over: operands, outputs and sizes.
struct HostProblem {
  const uint8_t *Aq, *Bq;
  const float *As, *Bs;
  void *C;                // BF16 [M, N], or FP32 for ACC32
  uint8_t *Cq;            // QOUT only
  float *Cs;              // QOUT only
  int64_t M, N, K;
};

template <int LAYOUT, bool ACC32, bool PAIR, bool QOUT, int G>
int launch_kernel(const HostProblem *probs, int count, int sms, cudaStream_t stream) {
  constexpr int TN = TileFor<LAYOUT, PAIR>::TN;
  using CF = Cfg<LAYOUT, TN, PAIR>;
  constexpr int SMEM_BYTES = CF::SMEM_BYTES;
  static_assert(sizeof(GemmParams<G>) <= 32000, "kernel parameters");
  GemmParams<G> prm{};
  int *status = device_status_ptr();
  if (status == nullptr) return PURO_ERR_CUDA;
  prm.count = count;
  prm.timeout_ns = wait_timeout_ns();
  prm.status = status;
  const int tile_rows = PAIR ? 2 * BM : BM;
  int64_t tiles = 0;
  for (int p = 0; p < count; ++p) {
    const HostProblem &h = probs[p];
    if (!make_map(&prm.tmA[p], h.Aq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h.M, h.K, BM, BK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&prm.tmB[p], h.Bq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, h.N, h.K, CF::B_ROWS, BK,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !(ACC32 ? make_map(&prm.tmC[p], h.C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, h.M, h.N, 32, 32,
                           CU_TENSOR_MAP_SWIZZLE_128B)
                : make_map(&prm.tmC[p], h.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h.M, h.N, 32, 64,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
      return PURO_ERR_CUDA;
    GemmArgs &a = prm.prob[p];
    a.As = h.As;
    a.Bs = h.Bs;
    a.C = static_cast<uint16_t *>(h.C);
    a.Cq = h.Cq;
    a.Cs = h.Cs;
    a.M = static_cast<int>(h.M);
    a.N = static_cast<int>(h.N);
    a.K = static_cast<int>(h.K);
    a.kblocks = static_cast<int>(h.K / BK);
    // Walk the smaller operand fastest so that it stays resident in L2 while the larger
    // one streams through once.
    a.m_fastest = h.M <= h.N ? 1 : 0;
    a.vec_a = (reinterpret_cast<uintptr_t>(h.As) % 16 == 0 && h.M % 4 == 0) ? 1 : 0;
    a.vec_b = (reinterpret_cast<uintptr_t>(h.Bs) % 16 == 0) ? 1 : 0;  // used by wgrad only
    a.num_m = static_cast<int>((h.M + tile_rows - 1) / tile_rows);
    a.num_n = static_cast<int>((h.N + TN - 1) / TN);
    a.tile_begin = static_cast<int>(tiles);
    tiles += static_cast<int64_t>(a.num_m) * a.num_n;
  }
  if (tiles > (1ll << 31) - (1ll << 16)) return PURO_ERR_SHAPE;
  prm.tiles = static_cast<int>(tiles);
  auto kern = k_gemm_blockwise<LAYOUT, TN, ACC32, PAIR, QOUT, G>;
  // Once per device: the register split inside the kernel assumes exactly LAUNCH_REGS per
  // thread at launch (with any other count the promotion warps' setmaxnreg.inc could wait
  // forever), the kernel needs its dynamic shared memory opted in, and a pair kernel's
  // grid is sized by the clusters that can be resident at once (a persistent grid with
  // more would leave the extra clusters to run after the others).
  static PerDevice<int> prepared;  // PURO_OK or an error; for PAIR, the resident clusters
  int prep = PURO_ERR_CUDA;
  if (!prepared.get(prep, [&](int, int &v) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
        if (fa.numRegs != LAUNCH_REGS || fa.maxThreadsPerBlock < THREADS) {
          std::fprintf(stderr, "puro_fp8: GEMM kernel built with %d registers (expected %d); not launched\n",
                       fa.numRegs, LAUNCH_REGS);
          v = PURO_ERR_LAUNCH;
          return true;
        }
        const cudaError_t se = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (se != cudaSuccess) {
          std::fprintf(stderr, "puro_fp8: cudaFuncSetAttribute: %s\n", cudaGetErrorString(se));
          return false;
        }
        v = PURO_OK;
        if constexpr (PAIR) {
          cudaLaunchConfig_t cfg{};
          cudaLaunchAttribute attr[1];
          attr[0].id = cudaLaunchAttributeClusterDimension;
          attr[0].val.clusterDim.x = 2;
          attr[0].val.clusterDim.y = 1;
          attr[0].val.clusterDim.z = 1;
          cfg.gridDim = dim3(2 * (sms / 2));
          cfg.blockDim = dim3(THREADS);
          cfg.dynamicSmemBytes = SMEM_BYTES;
          cfg.attrs = attr;
          cfg.numAttrs = 1;
          int clusters = 0;
          if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
            std::fprintf(stderr, "puro_fp8: no CTA pair of the GEMM kernel fits on this device\n");
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
    const int64_t clusters = tiles < prep ? tiles : prep;
    grid = static_cast<int>(2 * clusters);
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, prm);
    if (e == cudaSuccess) e = cudaGetLastError();
  } else {
    grid = static_cast<int>(tiles < sms ? tiles : sms);
    kern<<<grid, THREADS, SMEM_BYTES, stream>>>(prm);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, kern);
    std::fprintf(stderr,
                 "puro_fp8: GEMM launch (grid %d, %d threads, %d B smem, %s): %s "
                 "[kernel: %d regs, max %d threads/block, max dyn smem %d]\n",
                 grid, THREADS, SMEM_BYTES, PAIR ? "CTA pairs" : "single CTAs", cudaGetErrorString(e),
                 fa.numRegs, fa.maxThreadsPerBlock, fa.maxDynamicSharedSizeBytes);
    return PURO_ERR_LAUNCH;
  }
  return PURO_OK;
}

// Single problems (G = 1) and groups of up to GROUP_MAX, on CTA pairs unless some problem
// has at most 128 output rows.
template <int LAYOUT, bool ACC32, bool QOUT = false>
int launch_layout(const HostProblem *probs, int count, cudaStream_t stream) {
  int sms = 0;
  if (!sm_count(sms)) return PURO_ERR_CUDA;
  bool pair = true;
  for (int p = 0; p < count; ++p) pair = pair && use_pair(probs[p].M);
  if (count == 1)
    return pair ? launch_kernel<LAYOUT, ACC32, true, QOUT, 1>(probs, 1, sms, stream)
                : launch_kernel<LAYOUT, ACC32, false, QOUT, 1>(probs, 1, sms, stream);
  if constexpr (!ACC32 && !QOUT) {
    return pair ? launch_kernel<LAYOUT, false, true, false, GROUP_MAX>(probs, count, sms, stream)
                : launch_kernel<LAYOUT, false, false, false, GROUP_MAX>(probs, count, sms, stream);
  }
  return PURO_ERR_LAYOUT;
}

}  // namespace

int launch_gemm_blockwise(const uint8_t *Aq, const float *As, const uint8_t *Bq, const float *Bs,
                          uint16_t *C, int64_t M, int64_t N, int64_t K, int layout,
                          cudaStream_t stream) {
  const HostProblem h{Aq, Bq, As, Bs, C, nullptr, nullptr, M, N, K};
  switch (layout) {
    case PURO_FPROP: return launch_layout<PURO_FPROP, false>(&h, 1, stream);
    case PURO_DGRAD: return launch_layout<PURO_DGRAD, false>(&h, 1, stream);
    case PURO_WGRAD: return launch_layout<PURO_WGRAD, false>(&h, 1, stream);
    default: return PURO_ERR_LAYOUT;
  }
}

int launch_gemm_blockwise_grouped(const GroupedProblem *problems, int count, int layout,
                                  cudaStream_t stream) {
  if (count < 1 || count > GROUP_MAX) return PURO_ERR_SHAPE;
  HostProblem h[GROUP_MAX];
  for (int p = 0; p < count; ++p)
    h[p] = HostProblem{problems[p].Aq, problems[p].Bq, problems[p].As, problems[p].Bs, problems[p].C,
                       nullptr, nullptr, problems[p].M, problems[p].N, problems[p].K};
  // The longest tiles (most K blocks) first, so the shorter ones fill the last wave.
  for (int a = 1; a < count; ++a)
    for (int b = a; b > 0 && h[b].K > h[b - 1].K; --b) {
      const HostProblem t = h[b];
      h[b] = h[b - 1];
      h[b - 1] = t;
    }
  switch (layout) {
    case PURO_FPROP: return launch_layout<PURO_FPROP, false>(h, count, stream);
    case PURO_DGRAD: return launch_layout<PURO_DGRAD, false>(h, count, stream);
    case PURO_WGRAD: return launch_layout<PURO_WGRAD, false>(h, count, stream);
    default: return PURO_ERR_LAYOUT;
  }
}

int launch_gemm_blockwise_quant(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                                const float *Bs, uint16_t *C, uint8_t *Cq, float *Cs, int64_t M,
                                int64_t N, int64_t K, int layout, cudaStream_t stream) {
  const HostProblem h{Aq, Bq, As, Bs, C, Cq, Cs, M, N, K};
  switch (layout) {
    case PURO_FPROP: return launch_layout<PURO_FPROP, false, true>(&h, 1, stream);
    case PURO_DGRAD: return launch_layout<PURO_DGRAD, false, true>(&h, 1, stream);
    default: return PURO_ERR_LAYOUT;
  }
}

int launch_gemm_wgrad_acc_f32(const uint8_t *Aq, const float *As, const uint8_t *Bq,
                              const float *Bs, float *C, int64_t M, int64_t N, int64_t K,
                              cudaStream_t stream) {
  const HostProblem h{Aq, Bq, As, Bs, C, nullptr, nullptr, M, N, K};
  return launch_layout<PURO_WGRAD, true>(&h, 1, stream);
}

int read_and_clear_device_status(cudaStream_t stream, int *status_out) {
  int host = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return PURO_ERR_CUDA;
  *status_out = host;
  return PURO_OK;
}

}  // namespace puro

#ifdef PURO_TEST_HOOKS
extern "C" __attribute__((visibility("default"))) int puro_test_set_skip_release(int on) {
  return cudaMemcpyToSymbol(puro::g_test_skip_release, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
