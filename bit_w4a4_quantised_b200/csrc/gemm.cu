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
// CTA = 6 warps: warp 0 issues TMA (tiles) and bulk copies (scales) into a
// STAGES-deep shared-memory ring, warp 1 owns TMEM and issues tcgen05.cp (scales
// -> TMEM) and tcgen05.mma, warps 2-5 drain the accumulator (tcgen05.ld).  Tile
// 128 x BN, 256 K per stage (128 bytes of packed E2M1 per row = one 128B-swizzle
// atom), K64 per MMA.  Split-K (small M): each split stores fp32 partials, the
// last split to finish a tile (atomic ticket) sums them in split order and runs
// the epilogue.  No TMA multicast.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwam {
namespace {

constexpr int kBM = 128;
constexpr int kStageBytes = 128;    // bytes per row per stage
constexpr int kThreads = 192;

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 256 ? 3 : 4;
  static constexpr int A_BYTES = kBM * kStageBytes;
  static constexpr int B_BYTES = BN * kStageBytes;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
  static constexpr int U_BYTES = kBM * 64;
  static constexpr int L_BYTES = BN * 64;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
  static constexpr int OFF_U = OFF_SFB + STAGES * SFB_BYTES;
  static constexpr int OFF_L = OFF_U + U_BYTES;
  static constexpr int OFF_BAR = OFF_L + L_BYTES;
  static constexpr int NBAR = 2 * STAGES + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  // TMEM columns: accumulator [0, BN), then per stage 4 K64 steps of scale
  // factors: A needs 4 columns per step (128 rows), B needs BN/32.
  static constexpr int SF_COLS = 4 * 4 + 4 * (BN / 32);
  static constexpr int TMEM_USED = BN + STAGES * SF_COLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
  static_assert(TMEM_USED <= 512, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return pack2(bf16_bits_rn(a), bf16_bits_rn(b));
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL,
                    const GemmParams p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::STAGES;
  uint64_t* branch_full = empty + C::STAGES;
  uint64_t* acc_full = branch_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  uint32_t* last_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM, split = blockIdx.z;
  const int s_begin = split * p.stages_per_split;
  const int s_end = min(s_begin + p.stages_per_split, p.k_stages);
  const int n_st = max(0, s_end - s_begin);
  const int k64_total = p.K / 64;
  const bool do_branch = p.has_branch && split == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(branch_full, 1);
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- producer ----------------
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (do_branch) {
      tma_prefetch_desc(&tmU);
      tma_prefetch_desc(&tmL);
      mbar_arrive_expect_tx(branch_full, static_cast<uint32_t>((kBM + BN) * p.branch_k * 2));
      tma_load_2d(smem + C::OFF_U, &tmU, branch_full, 0, m0);
      tma_load_2d(smem + C::OFF_L, &tmL, branch_full, 0, n0);
    }
    int issued = 0;
    for (int i = 0; i < n_st; ++i) {
      const int st = i % C::STAGES;
      const uint32_t ph = (i / C::STAGES) & 1;
      if (!mbar_wait(&empty[st], ph ^ 1u, p.err, DEVERR_PRODUCER_WAIT)) break;
      const int s = s_begin + i;
      const int nk = min(4, k64_total - 4 * s);
      const uint32_t sfb = static_cast<uint32_t>(nk) * 512u;
      mbar_arrive_expect_tx(&full[st], C::A_BYTES + C::B_BYTES + sfb * (1 + BN / 128));
      tma_load_2d(smem + C::OFF_A + st * C::A_BYTES, &tmA, &full[st], s * kStageBytes, m0);
      tma_load_2d(smem + C::OFF_B + st * C::B_BYTES, &tmB, &full[st], s * kStageBytes, n0);
      bulk_load(smem + C::OFF_SFA + st * C::SFA_BYTES,
                p.sfa + (static_cast<size_t>(m0 / 128) * k64_total + 4 * s) * 512, sfb, &full[st]);
#pragma unroll
      for (int j = 0; j < BN / 128; ++j)
        bulk_load(smem + C::OFF_SFB + st * C::SFB_BYTES + j * 2048,
                  p.sfb + (static_cast<size_t>(n0 / 128 + j) * k64_total + 4 * s) * 512, sfb, &full[st]);
      ++issued;
    }
    // every copy this CTA started must land before it exits
    for (int i = max(0, issued - C::STAGES); i < issued; ++i)
      mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1, p.err, DEVERR_DRAIN_WAIT);
    if (do_branch) mbar_wait(branch_full, 0, p.err, DEVERR_DRAIN_WAIT);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                               (static_cast<uint32_t>(kBM >> 4) << 24);
    uint32_t accum = 0;
    bool ok = true;
    if (do_branch) {
      ok = mbar_wait(branch_full, 0, p.err, DEVERR_BRANCH_WAIT);
      if (ok) {
        tc_fence_after();
        const uint32_t idesc_bf16 = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                    (static_cast<uint32_t>(kBM >> 4) << 24);
        const uint32_t layout = p.branch_k == 32 ? 4u : 6u;  // 64B / 32B swizzle
        const uint32_t sbo = 8u * p.branch_k * 2u;
        const uint32_t us = smem_u32(smem + C::OFF_U), ls = smem_u32(smem + C::OFF_L);
        for (int kk = 0; kk < p.branch_k / 16; ++kk) {
          mma_bf16(tmem, smem_desc(us + kk * 32, 16, sbo, layout), smem_desc(ls + kk * 32, 16, sbo, layout),
                   idesc_bf16, accum);
          accum = 1;
        }
      }
    }
    for (int i = 0; ok && i < n_st; ++i) {
      const int st = i % C::STAGES;
      const uint32_t ph = (i / C::STAGES) & 1;
      if (!mbar_wait(&full[st], ph, p.err, DEVERR_MMA_WAIT)) break;
      tc_fence_after();
      const int s = s_begin + i;
      const int nk = min(4, k64_total - 4 * s);
      const uint32_t sfa_col = BN + st * C::SF_COLS;
      const uint32_t sfb_col = sfa_col + 16;
      const uint32_t sfa_s = smem_u32(smem + C::OFF_SFA + st * C::SFA_BYTES);
      const uint32_t sfb_s = smem_u32(smem + C::OFF_SFB + st * C::SFB_BYTES);
      for (int kk = 0; kk < nk; ++kk) {
        tmem_cp_32x128b_x4(tmem + sfa_col + kk * 4, smem_desc(sfa_s + kk * 512, 0, 128, 0));
#pragma unroll
        for (int j = 0; j < BN / 128; ++j)
          tmem_cp_32x128b_x4(tmem + sfb_col + kk * (BN / 32) + j * 4,
                             smem_desc(sfb_s + j * 2048 + kk * 512, 0, 128, 0));
      }
      const uint32_t a_s = smem_u32(smem + C::OFF_A + st * C::A_BYTES);
      const uint32_t b_s = smem_u32(smem + C::OFF_B + st * C::B_BYTES);
      for (int kk = 0; kk < nk; ++kk) {
        mma_mxf4nvf4(tmem, smem_desc(a_s + kk * 32, 16, 1024, 2), smem_desc(b_s + kk * 32, 16, 1024, 2), idesc_fp4,
                     tmem + sfa_col + kk * 4, tmem + sfb_col + kk * (BN / 32), accum);
        accum = 1;
      }
      tc_commit(&empty[st]);
    }
    tc_commit(acc_full);
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int qd = warp & 3;  // TMEM lane quarter this warp may access
    const bool ok = mbar_wait(acc_full, 0, p.err, DEVERR_EPILOGUE_WAIT);
    __syncwarp();
    tc_fence_after();
    const int row = m0 + qd * 32 + lane;
    const float gs = __fmul_rn(p.g_a_ptr ? *p.g_a_ptr : p.g_a, p.g_b);
    const uint16_t* bias = static_cast<const uint16_t*>(p.bias);
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(qd * 32) << 16) + c * 32, r);
        tmem_ld_wait();
        const int n = n0 + c * 32;
        if (row >= p.M || n >= p.N) continue;
        const int nvalid = min(32, p.N - n);  // 16 or 32 (N % 16 == 0)
        if constexpr (EPI == static_cast<int>(GemmEpilogue::Bf16)) {
          uint16_t* y = static_cast<uint16_t*>(p.y) + static_cast<size_t>(row) * p.N + n;
          for (int h = 0; h < nvalid / 16; ++h) {
            float bv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) bv[j] = bias ? bf16_bits_to_float(__ldg(bias + n + 16 * h + j)) : 0.0f;
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              o[j] = pack_bf16x2(__fmaf_rn(__uint_as_float(r[16 * h + 2 * j]), gs, bv[2 * j]),
                                 __fmaf_rn(__uint_as_float(r[16 * h + 2 * j + 1]), gs, bv[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(y + 16 * h);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
        } else {
          float* dst = (EPI == static_cast<int>(GemmEpilogue::RawF32))
                           ? p.out_f32 + static_cast<size_t>(row) * p.N + n
                           : p.partial + (static_cast<size_t>(split) * p.M + row) * p.N + n;
          const float sc = (EPI == static_cast<int>(GemmEpilogue::RawF32)) ? gs : 1.0f;
          for (int j = 0; j < nvalid; j += 4)
            *reinterpret_cast<float4*>(dst + j) =
                make_float4(__fmul_rn(__uint_as_float(r[j]), sc), __fmul_rn(__uint_as_float(r[j + 1]), sc),
                            __fmul_rn(__uint_as_float(r[j + 2]), sc), __fmul_rn(__uint_as_float(r[j + 3]), sc));
        }
      }
    }
    if constexpr (EPI == static_cast<int>(GemmEpilogue::SplitK)) {
      __threadfence();
      epi_bar();
      const int tile = blockIdx.y * gridDim.x + blockIdx.x;
      if (threadIdx.x == 64) {
        const uint32_t prev = atomicAdd(&p.counters[tile], 1u);
        *last_flag = (prev == static_cast<uint32_t>(p.splits - 1)) ? 1u : 0u;
      }
      epi_bar();
      if (*last_flag) {
        __threadfence();
        const int t = threadIdx.x - 64;
        const int rows_v = min(kBM, p.M - m0), cols_v = min(BN, p.N - n0);
        const int c4 = cols_v / 4;
        uint16_t* y = static_cast<uint16_t*>(p.y);
        for (int idx = t; idx < rows_v * c4; idx += 128) {
          const int m = m0 + idx / c4, n = n0 + (idx % c4) * 4;
          float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int sp = 0; sp < p.splits; ++sp) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p.partial + (static_cast<size_t>(sp) * p.M + m) * p.N + n));
            s.x = __fadd_rn(s.x, v.x);
            s.y = __fadd_rn(s.y, v.y);
            s.z = __fadd_rn(s.z, v.z);
            s.w = __fadd_rn(s.w, v.w);
          }
          float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
          if (bias) {
            b0 = bf16_bits_to_float(__ldg(bias + n));
            b1 = bf16_bits_to_float(__ldg(bias + n + 1));
            b2 = bf16_bits_to_float(__ldg(bias + n + 2));
            b3 = bf16_bits_to_float(__ldg(bias + n + 3));
          }
          *reinterpret_cast<uint2*>(y + static_cast<size_t>(m) * p.N + n) =
              make_uint2(pack_bf16x2(__fmaf_rn(s.x, gs, b0), __fmaf_rn(s.y, gs, b1)),
                         pack_bf16x2(__fmaf_rn(s.z, gs, b2), __fmaf_rn(s.w, gs, b3)));
        }
        if (t == 0) p.counters[tile] = 0u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, int EPI>
cudaError_t launch_t(const GemmMaps& m, const GemmParams& p, cudaStream_t st) {
  using C = Cfg<BN>;
  auto kern = fp4_gemm_kernel<BN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + BN - 1) / BN, (p.M + kBM - 1) / kBM, p.splits);
  kern<<<grid, kThreads, C::SMEM, st>>>(m.a, m.b, m.u, m.l, p);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const GemmMaps& m, const GemmParams& p, GemmEpilogue epi, cudaStream_t st) {
  switch (epi) {
    case GemmEpilogue::Bf16: return launch_t<BN, 0>(m, p, st);
    case GemmEpilogue::RawF32: return launch_t<BN, 1>(m, p, st);
    case GemmEpilogue::SplitK: return launch_t<BN, 2>(m, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t gemm_smem_bytes(int bn) { return bn == 256 ? Cfg<256>::SMEM : Cfg<128>::SMEM; }

cudaError_t launch_gemm(const GemmMaps& maps, const GemmParams& p, int bn, GemmEpilogue epi, cudaStream_t st) {
  if (bn == 256) return launch_bn<256>(maps, p, epi, st);
  if (bn == 128) return launch_bn<128>(maps, p, epi, st);
  return cudaErrorInvalidValue;
}

}  // namespace qwam
