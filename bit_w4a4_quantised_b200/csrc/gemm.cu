// Block-scaled NVFP4 GEMM on 5th-generation tensor cores (tcgen05, sm_100a),
// with the ASP low-rank branch and the bias folded into the same accumulator
// and epilogue.
//
//   acc[m, n] = sum_k e2m1(A[m,k]) sa[m,k/16] * e2m1(B[n,k]) sb[n,k/16]   (FP4 MMA)
//             + sum_j u'[m,j] L[n,j]                                     (bf16 MMA)
//   y[m, n]   = bf16( acc * g_a * g_b + bias[n] )
//
// u' is the activation branch operand already divided by g_a * g_b, so both
// MMA kinds accumulate in the same units into one TMEM accumulator and the
// single epilogue multiply restores the scale ("FastWAM UR3 3-task — 4-bit
// quantisations", section "What ASP is...": y = (x~V)(W~V)^T + NVFP4GEMM(...) +
// bias; branch kept in bf16).
//
// Persistent kernel, one CTA per SM, tiles of 128 x BN, K in stages of KS
// elements (KS / 2 bytes of packed E2M1 per row: one 128B- or 64B-swizzle
// atom), K64 per MMA.  A stage is one box each of A, B, the A scales and the B
// scales (every 128-row block of the tile in one 3-D box), all issued by
// different lanes of one instruction: on this part a lane's TMA boxes run one
// after another at a roughly fixed cost per box, while boxes from different
// lanes overlap.
// Roles:
//   producer warps  one per ring slot (a TMA instruction holds its warp for
//                   several hundred cycles); the first stage's weight boxes go
//                   out before the wait on the kernel that writes A.
//   MMA warp        owns TMEM; issues only tcgen05.mma (bf16 branch, then FP4).
//   copy warps      four; move each stage's scale blocks from shared memory
//                   into a four-slot TMEM scale ring (tcgen05.cp; one warp's
//                   copies run one after another, so four warps share them).
//   epilogue warps  eight, two per TMEM lane quarter (column halves).  Stage
//                   the tile's bias in shared memory, drain the accumulator
//                   to registers, release it to the next tile, round to bf16,
//                   stage through 128B-swizzled smem and store with TMA
//                   (ragged M / N are clipped by the tensor map).
// Split-K (small M): the splits of an output tile form one cluster (split
// fastest in the grid, one work item per CTA).  Once every split's MMAs are
// done, each pushes its fp32 accumulator rows to the CTA that owns them (a
// 128 / splits row slice) through distributed shared memory, into the owner's
// now idle operand ring; the owner sums the splits in order and writes y.
// Every mbarrier wait is bounded.  No TMA multicast.
#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace qwam {
namespace {

constexpr int kBM = 128;
constexpr int kEpiWarps = 8;
constexpr int kCopyWarps = 4;
constexpr int kScaleSlots = 4;  // TMEM scale ring, one stage per slot

// F8: the FP8 W8A8 arm (E4M3 operands, kind::f8f6f4, one byte per element, no
// block scales); otherwise NVFP4 (packed E2M1, E4M3 scale per 16 in TMEM).
// NB: no low-rank branch (r = 0): no room for the branch tiles.  CTA pairs
// keep five operand stages (the stage ring is bound by its round trip, not by
// the tensor core: more bytes in flight is more throughput), which just fit
// beside the branch tiles too.
template <int BN, int KS, bool PAIR = false, bool F8 = false, bool NB = false>
struct Cfg {
  static constexpr int TM = PAIR ? 2 * kBM : kBM;          // rows of an output tile
  static constexpr int HB = PAIR ? BN / 2 : BN;             // B (and L) rows held by one CTA
  static constexpr int ROWB = F8 ? KS : KS / 2;             // operand bytes per row per stage
  static constexpr int KM = F8 ? KS / 32 : KS / 64;         // MMAs per stage (K 32 for FP8, 64 for FP4)
  static constexpr int K64 = KS / 64;                       // K64 steps of a stage (FP4 scale blocks)
  static constexpr uint32_t SWZ = ROWB == 128 ? 2u : 4u;    // UMMA layout: 128B / 64B swizzle
  static constexpr int STAGES = PAIR ? 5 : (ROWB == 128 ? (BN == 256 ? 3 : 4) : (BN == 256 ? 6 : 8));
  static constexpr int NSFB = F8 ? 0 : BN / 128;            // 128-row scale blocks of B
  static constexpr int SF_BLK = F8 ? 0 : K64 * 512;         // one 128-row scale block of a stage
  static constexpr int NBOX = F8 ? 2 : 4;                   // boxes per stage: A, B (, A scales, B scales)
  // producer warps, taking stages in turn (three keep the CTA at 16 warps, so
  // the epilogue keeps 128 registers)
  static constexpr int NPROD = STAGES < 3 ? STAGES : 3;
  static constexpr int MMA_WARP = NPROD;
  static constexpr int CP_WARP0 = NPROD + 1;
  static constexpr int EPI_WARP0 = CP_WARP0 + kCopyWarps;
  static constexpr int THREADS = 32 * (EPI_WARP0 + kEpiWarps);
  static constexpr int REG_OTHER = 96, REG_EPI = 160;       // per thread after setmaxnreg
  static constexpr int A_BYTES = kBM * ROWB;
  static constexpr int B_BYTES = HB * ROWB;
  static constexpr int SF_BYTES = F8 ? 0 : (1 + NSFB) * SF_BLK;
  static constexpr int STAGE_TX = A_BYTES + B_BYTES + SF_BYTES;
  static constexpr int U_BYTES = NB ? 0 : kBM * 64;
  static constexpr int L_BYTES = NB ? 0 : HB * 64;
  static constexpr int SCOLS = PAIR ? 32 : 64;              // columns of one y store box
  static constexpr int STG_BYTES = 32 * SCOLS * 2;          // per epilogue warp: 32 rows x SCOLS bf16
  static constexpr int BIAS_BYTES = BN;                     // per epilogue warp: BN / 2 bf16
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_U = OFF_SF + STAGES * SF_BYTES;
  static constexpr int OFF_L = OFF_U + U_BYTES;
  static constexpr int OFF_STG = OFF_L + L_BYTES;
  static constexpr int OFF_BIAS = OFF_STG + kEpiWarps * STG_BYTES;
  static constexpr int OFF_BAR = OFF_BIAS + kEpiWarps * BIAS_BYTES;
  static constexpr int NBAR = 2 * STAGES + 2 * kScaleSlots + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  // TMEM columns: accumulator [0, BN), then kScaleSlots scale slots, each K64
  // steps of A (4 columns) then of B (BN / 32 columns).
  static constexpr int SF_A_COLS = K64 * 4;
  static constexpr int SF_COLS = SF_A_COLS + K64 * (BN / 32);
  static constexpr int TMEM_USED = BN + (F8 ? 0 : kScaleSlots * SF_COLS);
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(NBOX <= 32, "one lane per box");
  static_assert(PAIR || kBM * BN * 4 <= STAGES * (A_BYTES + B_BYTES), "split-K receive area fits in the operand ring");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return pack2(bf16_bits_rn(a), bf16_bits_rn(b));
}

struct TileCoord {
  int m0, n0, split;
};

// Tiles run M-fastest so consecutive CTAs reuse the same weight tile from L2;
// with split-K the split index is fastest (a tile's splits are one cluster).
// m0 is the first row of the tile (tm rows).
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n, int tm, int bn, int splits) {
  const int sp = t % splits;
  const int rest = t / splits;
  return {(rest % tiles_m) * tm, (rest / tiles_m % tiles_n) * bn, sp};
}

template <int BN, int KS, int EPI, bool PAIR, bool F8, bool NB>
__global__ void __launch_bounds__(Cfg<BN, KS, PAIR, F8, NB>::THREADS, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL,
                    const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmSA,
                    const __grid_constant__ CUtensorMap tmSB, const GemmParams p) {
  using C = Cfg<BN, KS, PAIR, F8, NB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // [STAGES] operands and scales landed
  uint64_t* empty = full + C::STAGES;                               // [STAGES] MMAs done with the slot
  uint64_t* sf_ready = empty + C::STAGES;                           // [kScaleSlots] scales copied into TMEM
  uint64_t* sf_tfree = sf_ready + kScaleSlots;                      // [kScaleSlots] MMAs done with the TMEM slot
  uint64_t* branch_full = sf_tfree + kScaleSlots;
  uint64_t* branch_empty = branch_full + 1;
  uint64_t* acc_full = branch_empty + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  constexpr bool kClusterK = EPI == static_cast<int>(GemmEpilogue::SplitK);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  const int tiles_m = (p.M + C::TM - 1) / C::TM;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int n_tiles = tiles_m * tiles_n * p.splits;
  const int k64_total = p.K / (F8 ? 32 : 64);  // MMA K steps over the whole K
  // CTA pair: rank 0 issues the MMAs and the scale copies for both CTAs; each
  // CTA loads its own 128 rows of A and its half of the B rows, and every load
  // of either CTA counts its bytes on rank 0's barrier.
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  auto coord = [&](int t) {
    TileCoord tc = tile_coord(t, tiles_m, tiles_n, C::TM, BN, p.splits);
    tc.m0 += static_cast<int>(rank) * kBM;  // this CTA's rows
    return tc;
  };
  // barrier addresses as the pair-wide forms take them
  auto lead = [&](uint64_t* b) { return PAIR ? dsmem_addr(smem_u32(b), 0u) : smem_u32(b); };
  // tcgen05 commits: to rank 0 only, or to the same barrier in both CTAs
  auto commit_lead = [&](uint64_t* b) {
    if constexpr (PAIR) tc_commit_pair(dsmem_addr(smem_u32(b), 0u));
    else tc_commit(b);
  };
  auto commit_both = [&](uint64_t* b) {
    if constexpr (PAIR) {
      tc_commit_pair(dsmem_addr(smem_u32(b), 0u));
      tc_commit_pair(dsmem_addr(smem_u32(b), 1u));
    } else {
      tc_commit(b);
    }
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kScaleSlots; ++i) {
      mbar_init(&sf_ready[i], kCopyWarps);
      mbar_init(&sf_tfree[i], 1);
    }
    mbar_init(branch_full, 1);
    mbar_init(branch_empty, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps * (PAIR ? 2 : 1));
    fence_barrier_init();
  }
  if (warp == C::MMA_WARP) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // both CTAs' barriers are initialised before either signals the other's
    cluster_arrive();
    cluster_wait();
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the next kernel in the stream may start its own set-up now
  griddep_launch_dependents();
  // Split-K cluster barriers: A0 (every split CTA runs), R (every split's MMAs
  // are done, so its operand ring may take remote stores), P (all rows pushed).
  // Up to 64 rows the pushed rows fit in the epilogue staging area, which the
  // split-K epilogue does not otherwise use, and R is not needed.
  const bool rx_stg = p.M <= 64 && kBM / 2 * BN * 4 <= kEpiWarps * C::STG_BYTES;
  if constexpr (kClusterK) cluster_arrive();  // A0
  // every role other than the epilogue ends with the same cluster barriers
  auto cluster_tail = [&]() {
    if constexpr (kClusterK) {
      cluster_wait();  // A0
      if (!rx_stg) {
        cluster_arrive();  // R
        cluster_wait();
      }
      cluster_arrive();  // P
      cluster_wait();
    }
  };

  // A split's K range: stages [s_begin, s_begin + n_st) (balanced: every split
  // gets at least one stage when splits <= k_stages), K64 steps
  // [k64_begin, k64_begin + n_k64).
  struct Range {
    int s_begin, n_st, k64_begin, n_k64;
  };
  auto range_of = [&](int split) {
    Range r;
    r.s_begin = split * p.k_stages / p.splits;
    r.n_st = (split + 1) * p.k_stages / p.splits - r.s_begin;
    r.k64_begin = r.s_begin * C::KM;
    r.n_k64 = min(r.n_st * C::KM, k64_total - r.k64_begin);
    return r;
  };

  // Warps [0, EPI_WARP0) are two warpgroups (producers + MMA, copy warps) that
  // need few registers; the two epilogue warpgroups hold a column half of the
  // accumulator as packed bf16.  setmaxnreg moves registers between them:
  // 256 x REG_OTHER + 256 x REG_EPI = 512 x 128, the launch's total.  It is
  // the first instruction of each branch (warpgroup-wide).
  static_assert(C::EPI_WARP0 == 8 && C::THREADS == 512, "two warpgroups each side");
  static_assert(256 * (C::REG_OTHER + C::REG_EPI) <= 512 * 128, "register split");
  if (warp < C::EPI_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_OTHER));
  if (warp < C::NPROD) {
    // ------------------------------------------------ producers: warp w issues stages g = w mod NPROD
    if (lane == 0 && warp == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      tma_prefetch_desc(&tmSA);
      tma_prefetch_desc(&tmSB);
      if (!NB && p.has_branch) {
        tma_prefetch_desc(&tmU);
        tma_prefetch_desc(&tmL);
      }
    }
    // this lane's box of a stage: 0 A, 1 B, 2 A scales, 3 B scales; weight
    // boxes (B and its scales) do not depend on the kernel before this one
    const bool weight_box = lane == 1 || lane == 3;
    const CUtensorMap* map = lane == 0 ? &tmA : (lane == 1 ? &tmB : (lane == 2 ? &tmSA : &tmSB));
    const int dst_base = lane == 0 ? C::OFF_A : (lane == 1 ? C::OFF_B : C::OFF_SF + (lane - 2) * C::SF_BLK);
    const int dst_step = lane == 0 ? C::A_BYTES : (lane == 1 ? C::B_BYTES : C::SF_BYTES);
    int g = 0;  // stage counter of this CTA
    int last = -1, nbranch = 0;
    bool ok = true;
    bool dep_done = false;  // griddep_wait() done: A, its scales and U may be read
    for (int t = unit; ok && t < n_tiles; t += n_units) {
      const TileCoord tc = coord(t);
      const Range rg = range_of(tc.split);
      if (!NB && p.has_branch && tc.split == 0 && warp == C::NPROD - 1) {
        // branch operands of this tile, once the previous tile's branch MMAs are done
        int bok = 1;
        if (lane == 0) {
          bok = (nbranch == 0 || mbar_wait(branch_empty, (nbranch - 1) & 1, p.err, DEVERR_PRODUCER_WAIT, wlim)) ? 1 : 0;
          if (bok && leader)
            mbar_arrive_expect_tx(branch_full, static_cast<uint32_t>((PAIR ? 2 : 1) * (kBM + C::HB) * p.branch_k * 2));
        }
        bok = __shfl_sync(0xffffffffu, bok, 0);
        if (!bok) break;
        // L (weights) may load before the activation producer has finished; U not
        const int l_row = tc.n0 + static_cast<int>(rank) * C::HB;
        if (lane == 1) {
          if constexpr (PAIR) tma_load_2d_pair(smem + C::OFF_L, &tmL, lead(branch_full), 0, l_row);
          else tma_load_2d(smem + C::OFF_L, &tmL, branch_full, 0, l_row);
        }
        if (!dep_done) {
          griddep_wait();
          dep_done = true;
        }
        if (lane == 0) {
          if constexpr (PAIR) tma_load_2d_pair(smem + C::OFF_U, &tmU, lead(branch_full), 0, tc.m0);
          else tma_load_2d(smem + C::OFF_U, &tmU, branch_full, 0, tc.m0);
        }
        ++nbranch;
      }
      for (int i = 0; i < rg.n_st; ++i, ++g) {
        if (g % C::NPROD != warp) continue;
        const int st = g % C::STAGES;
        const uint32_t ph = (g / C::STAGES) & 1;
        uint8_t* const dst = smem + dst_base + st * dst_step;
        int wok = 1;
        if (lane == 0) wok = mbar_wait(&empty[st], ph ^ 1u, p.err, DEVERR_PRODUCER_WAIT, wlim) ? 1 : 0;
        wok = __shfl_sync(0xffffffffu, wok, 0);
        if (!wok) {
          ok = false;
          break;
        }
        const int kst = rg.s_begin + i;
        // operands: x = byte column, y = row, z = 0; scales (256-byte rows, two
        // per K64 step of a 128-row block): x = 0, y = 2 * step, z = block
        int cx = 0, cy, cz = 0;
        if (lane < 2) {
          cx = kst * C::ROWB;
          cy = lane ? tc.n0 + static_cast<int>(rank) * C::HB : tc.m0;
        } else {
          cy = 2 * kst * C::K64;
          cz = lane == 2 ? tc.m0 / kBM : tc.n0 / 128;
        }
        if (lane == 0 && leader)
          mbar_arrive_expect_tx(&full[st], (PAIR ? 2 : 1) * C::STAGE_TX + (g == 0 ? p.withheld_bytes : 0u));
        __syncwarp();
        auto load = [&]() {
          if constexpr (PAIR) tma_load_3d_pair(dst, map, lead(&full[st]), cx, cy, cz);
          else tma_load_3d(dst, map, &full[st], cx, cy, cz);
        };
        if (dep_done) {
          if (lane < C::NBOX) load();
        } else {
          // the weight boxes first, then A and its scales once the kernel
          // writing them has finished
          if (weight_box && lane < C::NBOX) load();
          griddep_wait();
          dep_done = true;
          if (!weight_box) {
            if (lane < C::NBOX) load();
          }
        }
        last = g;
      }
    }
    // every copy this warp started must land before the CTA exits (in a pair
    // rank 0 counts them; every MMA commit to this CTA's barriers must arrive)
    if (lane == 0) {
      if (leader && last >= 0) mbar_wait(&full[last % C::STAGES], (last / C::STAGES) & 1, p.err, DEVERR_DRAIN_WAIT, wlim);
      if (leader && nbranch > 0) mbar_wait(branch_full, (nbranch - 1) & 1, p.err, DEVERR_DRAIN_WAIT, wlim);
      if (PAIR && last >= 0) mbar_wait(&empty[last % C::STAGES], (last / C::STAGES) & 1, p.err, DEVERR_DRAIN_WAIT, wlim);
      if (PAIR && nbranch > 0) mbar_wait(branch_empty, (nbranch - 1) & 1, p.err, DEVERR_DRAIN_WAIT, wlim);
    }
    __syncwarp();
    cluster_tail();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------ MMA issuer (rank 0 of a pair)
    if (lane == 0 && leader) {
      const uint32_t idesc_fp4 = F8 ? idesc_f8e4m3(C::TM, BN) : idesc_mxf4(C::TM, BN);
      const uint32_t idesc_br = idesc_bf16(C::TM, BN);
      const uint32_t layout = p.branch_k == 32 ? 4u : 6u;  // 64B / 32B swizzle
      const uint32_t sbo = 8u * p.branch_k * 2u;
      const uint32_t us = smem_u32(smem + C::OFF_U), ls = smem_u32(smem + C::OFF_L);
      int g = 0, tl = 0, nbranch = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units, ++tl) {
        const TileCoord tc = coord(t);
        const Range rg = range_of(tc.split);
        // the epilogue must have drained the previous tile's accumulator
        if (!mbar_wait(acc_empty, (tl & 1) ^ 1u, p.err, DEVERR_MMA_WAIT, wlim)) break;
        tc_fence_after();
        uint32_t accum = 0;
        if (!NB && p.has_branch && tc.split == 0) {
          if (!mbar_wait(branch_full, nbranch & 1, p.err, DEVERR_BRANCH_WAIT, wlim)) break;
          tc_fence_after();
          for (int kk = 0; kk < p.branch_k / 16; ++kk) {
            const uint64_t ud = smem_desc(us + kk * 32, 16, sbo, layout), ld = smem_desc(ls + kk * 32, 16, sbo, layout);
            if constexpr (PAIR) mma_bf16_pair(tmem, ud, ld, idesc_br, accum);
            else mma_bf16(tmem, ud, ld, idesc_br, accum);
            accum = 1;
          }
          commit_both(branch_empty);
          ++nbranch;
        }
        for (int i = 0; i < rg.n_st; ++i, ++g) {
          const int st = g % C::STAGES, sl = g % kScaleSlots;
          if (!mbar_wait(&full[st], (g / C::STAGES) & 1, p.err, DEVERR_MMA_WAIT, wlim) ||
              (!F8 && !mbar_wait(&sf_ready[sl], (g / kScaleSlots) & 1, p.err, DEVERR_MMA_WAIT, wlim))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = smem_u32(smem + C::OFF_A + st * C::A_BYTES);
          const uint32_t b_s = smem_u32(smem + C::OFF_B + st * C::B_BYTES);
          const uint32_t sfa = tmem + BN + sl * C::SF_COLS, sfb = sfa + C::SF_A_COLS;
          const int nk = min(C::KM, rg.n_k64 - i * C::KM);
          for (int kk = 0; kk < nk; ++kk) {
            // one MMA takes 32 bytes of each operand row (K 64 FP4 / K 32 FP8)
            const uint64_t ad = smem_desc(a_s + kk * 32, 16, 8 * C::ROWB, C::SWZ);
            const uint64_t bd = smem_desc(b_s + kk * 32, 16, 8 * C::ROWB, C::SWZ);
            if constexpr (F8) {
              if constexpr (PAIR) mma_f8_pair(tmem, ad, bd, idesc_fp4, accum);
              else mma_f8(tmem, ad, bd, idesc_fp4, accum);
            } else {
              if constexpr (PAIR) mma_mxf4nvf4_pair(tmem, ad, bd, idesc_fp4, sfa + kk * 4, sfb + kk * (BN / 32), accum);
              else mma_mxf4nvf4(tmem, ad, bd, idesc_fp4, sfa + kk * 4, sfb + kk * (BN / 32), accum);
            }
            accum = 1;
          }
          commit_both(&empty[st]);
          if constexpr (!F8) commit_lead(&sf_tfree[sl]);
        }
        if (!ok) break;
        commit_both(acc_full);
      }
    }
    __syncwarp();
    cluster_tail();
  } else {
    // ------------------------------------------------ scale copies: smem stage -> TMEM slot (rank 0 of a pair)
    const int cw = warp - C::CP_WARP0;
    if (!F8 && lane == 0 && leader) {  // FP8 operands carry no block scales
      int g = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units) {
        const Range rg = range_of(coord(t).split);
        for (int i = 0; i < rg.n_st; ++i, ++g) {
          const int st = g % C::STAGES, sl = g % kScaleSlots;
          if (!mbar_wait(&full[st], (g / C::STAGES) & 1, p.err, DEVERR_SCALE_WAIT, wlim) ||
              (g >= kScaleSlots &&
               !mbar_wait(&sf_tfree[sl], ((g / kScaleSlots) & 1) ^ 1u, p.err, DEVERR_SCALE_WAIT, wlim))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(C::K64, rg.n_k64 - i * C::K64);
          const uint32_t src = smem_u32(smem + C::OFF_SF + st * C::SF_BYTES);
          const uint32_t col0 = BN + sl * C::SF_COLS;
          for (int c = cw; c < C::K64 * (1 + C::NSFB); c += kCopyWarps) {
            const int blk = c / C::K64, kk = c % C::K64;
            if (kk >= nk) continue;
            const uint32_t col = blk == 0 ? col0 + kk * 4 : col0 + C::SF_A_COLS + kk * (BN / 32) + (blk - 1) * 4;
            const uint64_t sd = smem_desc(src + blk * C::SF_BLK + kk * 512, 0, 128, 0);
            if constexpr (PAIR) tmem_cp_32x128b_x4_pair(tmem + col, sd);
            else tmem_cp_32x128b_x4(tmem + col, sd);
          }
          commit_lead(&sf_ready[sl]);
        }
      }
    }
    __syncwarp();
    cluster_tail();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_EPI));
    // ------------------------------------------------ epilogue
    const int ew = warp - C::EPI_WARP0;  // 0..7
    const int qd = warp & 3;             // TMEM lane quarter this warp may access
    const int half = ew >> 2;            // column half [half*BN/2, (half+1)*BN/2)
    const int et = threadIdx.x - 32 * C::EPI_WARP0;
    constexpr int HC = BN / 2;           // columns per thread
    griddep_wait();  // g_a is written by the kernel before this one
    const float gs = __fmul_rn(p.g_a_ptr ? *p.g_a_ptr : p.g_a, p.g_b);
    const uint16_t* bias = static_cast<const uint16_t*>(p.bias);
    // staging: a 32-row block per warp, the four blocks of a column half
    // stacked in lane-quarter order (128 rows: one TMA store box)
    uint8_t* stg = smem + C::OFF_STG + (half * 4 + qd) * C::STG_BYTES;
    uint8_t* const stg_half = smem + C::OFF_STG + half * 4 * C::STG_BYTES;
    const bool store_issuer = qd == 0 && lane == 0;  // one thread per column half
    uint4* bias_s = reinterpret_cast<uint4*>(smem + C::OFF_BIAS + ew * C::BIAS_BYTES);  // this warp's HC bf16
    int tl = 0;
    bool alive = true;
    for (int t = unit; t < n_tiles; t += n_units, ++tl) {
      const TileCoord tc = coord(t);
      const int row = tc.m0 + qd * 32 + lane;
      const int c0 = tc.n0 + half * HC;
      if constexpr (EPI == static_cast<int>(GemmEpilogue::Bf16)) {
        // this warp's bias columns, fetched while the tile accumulates
        if (lane < HC / 8) {
          uint4 braw = make_uint4(0u, 0u, 0u, 0u);
          if (bias && c0 + 8 * lane < p.N) braw = __ldg(reinterpret_cast<const uint4*>(bias + c0 + 8 * lane));
          bias_s[lane] = braw;
        }
        __syncwarp();
      }
      // after one wait has run out, the accumulator of later tiles never comes
      const bool ok = alive && mbar_wait(acc_full, tl & 1, p.err, DEVERR_EPILOGUE_WAIT, wlim);
      alive = ok;
      __syncwarp();
      tc_fence_after();
      if constexpr (EPI == static_cast<int>(GemmEpilogue::Bf16)) {
        // drain: y = bf16(acc * gs + bias).  The whole column half is read out
        // of TMEM and packed to bf16 pairs in registers first, so the
        // accumulator goes back to the MMA warp before any store is issued
        // (a TMA store can hold its thread while the engine is busy with the
        // operand loads).  Then the four warps of a column half stage SCOLS
        // columns of their 128 rows at a time (128B swizzle for 64 columns,
        // 64B for 32) and one thread stores them with one TMA box.  The half's
        // named barrier is reached by all four warps on every path.
        constexpr int NH = HC / C::SCOLS, CPR = C::SCOLS / 8;  // store rounds, 16-byte chunks per row
        const uint32_t taddr = tmem + (static_cast<uint32_t>(qd * 32) << 16) + half * HC;
        auto chunk = [&](int k) {
          const int sw = C::SCOLS == 64 ? (lane & 7) : ((lane >> 1) & 3);
          return reinterpret_cast<uint4*>(stg + lane * (2 * C::SCOLS) + ((k ^ sw) << 4));
        };
        // 8 columns (qq * 32 + 8 j ..) of a 32-column TMEM load -> 4 bf16 pairs
        auto convert = [&](const uint32_t* r, int qq, int j) {
          const uint4 bw = bias_s[qq * 4 + j];
          return make_uint4(fma_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1]), gs, bw.x),
                            fma_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]), gs, bw.y),
                            fma_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]), gs, bw.z),
                            fma_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]), gs, bw.w));
        };
        auto half_sync = [&]() { named_bar(1 + half, 128); };
        // two 32-column loads in flight per wait (the round trip, not the
        // bytes, sets the drain time; four serial rounds held the accumulator
        // ~1.4 us per tile)
        static_assert((HC / 32) % 2 == 0, "column pairs of 32");
        uint4 v[HC / 8];
#pragma unroll
        for (int qq = 0; qq < HC / 32; qq += 2) {
          uint32_t r[32], r1[32];
          tmem_ld_32x32b_x32(taddr + qq * 32, r);
          tmem_ld_32x32b_x32(taddr + (qq + 1) * 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j) v[4 * qq + j] = convert(r, qq, j);
#pragma unroll
          for (int j = 0; j < 4; ++j) v[4 * (qq + 1) + j] = convert(r1, qq + 1, j);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(lead(acc_empty));
          else mbar_arrive(acc_empty);
        }
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          if (store_issuer) bulk_wait_read<0>();  // the staging blocks are free
          half_sync();
#pragma unroll
          for (int k = 0; k < CPR; ++k) *chunk(k) = v[CPR * hh + k];
          fence_proxy_async();
          half_sync();
          if (store_issuer && ok) {
            tma_store_2d(&tmY, stg_half, c0 + hh * C::SCOLS, tc.m0);
            bulk_commit();
          }
        }
      } else if constexpr (EPI == static_cast<int>(GemmEpilogue::RawF32)) {
        // fp32 out: direct row stores
#pragma unroll 1
        for (int qq = 0; qq < HC / 32; ++qq) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(qd * 32) << 16) + half * HC + qq * 32, r);
          tmem_ld_wait();
          const int n = c0 + qq * 32;
          if (!ok || row >= p.M || n >= p.N) continue;
          float4* d4 = reinterpret_cast<float4*>(p.out_f32 + static_cast<size_t>(row) * p.N + n);
          const int nv = min(32, p.N - n) / 4;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k < nv)
              d4[k] = make_float4(__fmul_rn(__uint_as_float(r[4 * k]), gs), __fmul_rn(__uint_as_float(r[4 * k + 1]), gs),
                                  __fmul_rn(__uint_as_float(r[4 * k + 2]), gs),
                                  __fmul_rn(__uint_as_float(r[4 * k + 3]), gs));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(lead(acc_empty));
          else mbar_arrive(acc_empty);
        }
      } else {
        // Split-K: this tile's MMAs are done (acc_full), so this CTA's operand
        // ring is idle.  Push accumulator rows to their owner's ring, laid out
        // [split][row in slice][BN]; the owner sums them in split order.
        const int SLR = (rx_stg ? kBM / 2 : kBM) / p.splits;  // rows per owner
        float* ring = reinterpret_cast<float*>(smem + (rx_stg ? C::OFF_STG : C::OFF_A));
        cluster_wait();  // A0
        if (!rx_stg) {
          cluster_arrive();  // R
          cluster_wait();
        }
        const int rloc = qd * 32 + lane;
        const uint32_t dst = dsmem_addr(smem_u32(ring + (tc.split * SLR + rloc % SLR) * BN + half * HC),
                                        static_cast<uint32_t>(min(rloc / SLR, p.splits - 1)));
#pragma unroll 1
        for (int qq = 0; qq < HC / 32; ++qq) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(qd * 32) << 16) + half * HC + qq * 32, r);
          tmem_ld_wait();
          if (ok && row < p.M) {  // rows >= M are not pushed (rx_stg: M <= 64 rows)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dsmem_st_f4(dst + static_cast<uint32_t>((qq * 32 + 4 * k) * 4),
                          make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                      __uint_as_float(r[4 * k + 2]), __uint_as_float(r[4 * k + 3])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        cluster_arrive();  // P
        cluster_wait();
        uint16_t* y = static_cast<uint16_t*>(p.y);
        for (int it = et; it < SLR * (BN / 4); it += 32 * kEpiWarps) {
          const int srow = it / (BN / 4), c4 = it % (BN / 4);
          const int m = tc.m0 + tc.split * SLR + srow, n = tc.n0 + 4 * c4;
          if (m >= p.M || n >= p.N) continue;
          float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int sp = 0; sp < p.splits; ++sp) {
            const float4 v = *reinterpret_cast<const float4*>(ring + (sp * SLR + srow) * BN + 4 * c4);
            sacc.x = __fadd_rn(sacc.x, v.x);
            sacc.y = __fadd_rn(sacc.y, v.y);
            sacc.z = __fadd_rn(sacc.z, v.z);
            sacc.w = __fadd_rn(sacc.w, v.w);
          }
          float b4[4] = {0.f, 0.f, 0.f, 0.f};
          if (bias) {
            const uint2 braw = __ldg(reinterpret_cast<const uint2*>(bias + n));
            b4[0] = __uint_as_float(braw.x << 16);
            b4[1] = __uint_as_float(braw.x & 0xffff0000u);
            b4[2] = __uint_as_float(braw.y << 16);
            b4[3] = __uint_as_float(braw.y & 0xffff0000u);
          }
          *reinterpret_cast<uint2*>(y + static_cast<size_t>(m) * p.N + n) =
              make_uint2(pack_bf16x2(__fmaf_rn(sacc.x, gs, b4[0]), __fmaf_rn(sacc.y, gs, b4[1])),
                         pack_bf16x2(__fmaf_rn(sacc.z, gs, b4[2]), __fmaf_rn(sacc.w, gs, b4[3])));
        }
      }
    }
    if constexpr (EPI == static_cast<int>(GemmEpilogue::Bf16)) {
      if (lane == 0) bulk_wait<0>();
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // neither CTA leaves while the other may still signal its barriers
    cluster_arrive();
    cluster_wait();
  }
  if (warp == C::MMA_WARP) {
    __syncwarp();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int KS, int EPI, bool PAIR, bool F8, bool NB = false>
cudaError_t launch_t(const GemmMaps& m, const GemmParams& p, cudaStream_t st) {
  using C = Cfg<BN, KS, PAIR, F8, NB>;
  auto kern = fp4_gemm_kernel<BN, KS, EPI, PAIR, F8, NB>;
  if (NB && p.has_branch) return cudaErrorInvalidValue;
  static const cudaError_t smem_attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (smem_attr != cudaSuccess) return smem_attr;
  int dev = 0, sms = p.sms;
  cudaGetDevice(&dev);
  if (sms <= 0) {
    const cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  if (p.k_stages != (p.K + KS - 1) / KS) return cudaErrorInvalidValue;
  const int tiles = ((p.M + C::TM - 1) / C::TM) * ((p.N + BN - 1) / BN) * p.splits;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (EPI == static_cast<int>(GemmEpilogue::SplitK)) {
    // one work item per CTA; the splits of a tile are one cluster
    if (PAIR || p.splits < 2 || p.splits > 8 || (p.splits & (p.splits - 1)) || p.splits > p.k_stages)
      return cudaErrorInvalidValue;
    cfg.gridDim = dim3(tiles, 1, 1);
    attr[1].val.clusterDim.x = p.splits;
    cfg.numAttrs = 2;
  } else if (PAIR) {
    // persistent CTA pairs: as many as can be resident at once (a GPC with an
    // odd number of free SMs leaves one idle)
    if (p.splits != 1) return cudaErrorInvalidValue;
    attr[1].val.clusterDim.x = 2;
    cfg.numAttrs = 2;
    static int pairs_per_dev[64] = {};
    int pairs = dev >= 0 && dev < 64 ? pairs_per_dev[dev] : 0;
    if (pairs <= 0) {
      cfg.gridDim = dim3(sms & ~1, 1, 1);
      if (cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg) != cudaSuccess || pairs <= 0) {
        (void)cudaGetLastError();
        pairs = sms / 2;
      }
      pairs = std::min(pairs, sms / 2);
      if (dev >= 0 && dev < 64) pairs_per_dev[dev] = pairs;
    }
    cfg.gridDim = dim3(2 * std::min(tiles, pairs), 1, 1);
  } else {
    if (p.splits != 1) return cudaErrorInvalidValue;
    cfg.gridDim = dim3(std::min(tiles, sms), 1, 1);
  }
  return cudaLaunchKernelEx(&cfg, kern, m.a, m.b, m.u, m.l, m.y, m.sfa, m.sfb, p);
}

// registers per thread at launch: the split's total over the 512 threads
template <int BN, int KS, int EPI, bool PAIR, bool F8, bool NB = false>
bool split_ok(char* msg, size_t n) {
  using C = Cfg<BN, KS, PAIR, F8, NB>;
  constexpr int want = (256 * C::REG_OTHER + 256 * C::REG_EPI) / C::THREADS;
  cudaFuncAttributes a{};
  const cudaError_t e = cudaFuncGetAttributes(&a, fp4_gemm_kernel<BN, KS, EPI, PAIR, F8, NB>);
  if (e != cudaSuccess) {
    snprintf(msg, n, "cudaFuncGetAttributes(fp4_gemm_kernel<%d,%d,%d,%d,%d>) failed: %s", BN, KS, EPI, int(PAIR),
             int(F8), cudaGetErrorString(e));
    return false;
  }
  if ((a.numRegs + 7) / 8 * 8 != want) {
    snprintf(msg, n,
             "fp4_gemm_kernel<%d,%d,%d,%d,%d> was compiled to %d registers per thread; its warpgroup register "
             "split assumes %d",
             BN, KS, EPI, int(PAIR), int(F8), a.numRegs, want);
    return false;
  }
  return true;
}

template <int BN, int KS, bool PAIR, bool F8>
cudaError_t launch_bn(const GemmMaps& m, const GemmParams& p, GemmEpilogue epi, cudaStream_t st) {
  switch (epi) {
    case GemmEpilogue::Bf16:
      if constexpr (PAIR)
        if (!p.has_branch) return launch_t<BN, KS, 0, PAIR, F8, true>(m, p, st);
      return launch_t<BN, KS, 0, PAIR, F8>(m, p, st);
    case GemmEpilogue::RawF32:
      if constexpr (PAIR)
        if (!p.has_branch) return launch_t<BN, KS, 1, PAIR, F8, true>(m, p, st);
      return launch_t<BN, KS, 1, PAIR, F8>(m, p, st);
    case GemmEpilogue::SplitK:
      if constexpr (PAIR) return cudaErrorInvalidValue;
      else return launch_t<BN, KS, 2, false, F8>(m, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

template <bool F8, int KB, int KS>  // KB: K per stage of the large-M tiles, KS of the small-M ones
bool format_split_ok(char* msg, size_t n) {
  return split_ok<256, KB, 0, true, F8>(msg, n) && split_ok<256, KB, 1, true, F8>(msg, n) &&
         split_ok<256, KB, 0, true, F8, true>(msg, n) && split_ok<256, KB, 1, true, F8, true>(msg, n) &&
         split_ok<256, KB, 0, false, F8>(msg, n) && split_ok<256, KB, 1, false, F8>(msg, n) &&
         split_ok<256, KB, 2, false, F8>(msg, n) && split_ok<128, KB, 0, false, F8>(msg, n) &&
         split_ok<128, KB, 1, false, F8>(msg, n) && split_ok<128, KB, 2, false, F8>(msg, n) &&
         split_ok<128, KS, 0, false, F8>(msg, n) && split_ok<128, KS, 1, false, F8>(msg, n) &&
         split_ok<128, KS, 2, false, F8>(msg, n);
}

bool gemm_register_split_ok(char* msg, size_t n) {
  return format_split_ok<false, 256, 128>(msg, n) && format_split_ok<true, 128, 64>(msg, n);
}

GemmShape gemm_shape(int M, int N, bool fp8) {
  GemmShape s;
  s.bn = (M <= kBM || N < 256) ? 128 : 256;
  // operand rows of one 128B (large M) or 64B swizzle atom per stage
  s.ks = (M <= kBM ? 128 : 256) / (fp8 ? 2 : 1);
  s.pair = s.bn == 256;
  s.fp8 = fp8;
  return s;
}

cudaError_t launch_gemm(const GemmMaps& maps, const GemmParams& p, GemmShape shape, GemmEpilogue epi,
                        cudaStream_t st) {
  const int kb = shape.fp8 ? 128 : 256, ksm = shape.fp8 ? 64 : 128;  // K per stage: large / small M
  if (shape.pair) {
    if (shape.bn != 256 || shape.ks != kb) return cudaErrorInvalidValue;
    return shape.fp8 ? launch_bn<256, 128, true, true>(maps, p, epi, st)
                     : launch_bn<256, 256, true, false>(maps, p, epi, st);
  }
  if (shape.bn == 256 && shape.ks == kb)
    return shape.fp8 ? launch_bn<256, 128, false, true>(maps, p, epi, st)
                     : launch_bn<256, 256, false, false>(maps, p, epi, st);
  if (shape.bn == 128 && shape.ks == kb)
    return shape.fp8 ? launch_bn<128, 128, false, true>(maps, p, epi, st)
                     : launch_bn<128, 256, false, false>(maps, p, epi, st);
  if (shape.bn == 128 && shape.ks == ksm)
    return shape.fp8 ? launch_bn<128, 64, false, true>(maps, p, epi, st)
                     : launch_bn<128, 128, false, false>(maps, p, epi, st);
  return cudaErrorInvalidValue;
}

}  // namespace qwam
