// INT4 group-64 W4A4 GEMM of the SVDQuant arm on 5th-generation tensor cores
// (tcgen05, sm_100a).  "FastWAM UR3 3-task — 4-bit quantisations", top table,
// SVDQuant column: INT4 elements at group 64 on weights and activations, the
// products on integer tensor cores, exact for 4-bit codes.
//
//   P_g[m, n] = sum over the 64 k of group g of qa[m, k] qb[n, k]      (exact)
//   y[m, n]   = bf16( sum_g P_g[m, n] (sa[m, g] sb[n, g]) + sum_j u'[m, j] L[n, j] + bias[n] )
//
// The INT4 levels (-8..7) reach the tensor core as E4M3 bytes, which hold every
// level exactly; kind::f8f6f4 forms the exact products and the group sums (at
// most 64 * 64 in magnitude) are exact in its fp32 accumulator, so P_g is the
// integer an INT8 tensor core would give, read out of TMEM as fp32 with no
// conversion.  The scale sa sb changes from group to group, so it cannot stay
// in the accumulator: each group's P_g goes to one of four TMEM buffers in turn
// (the MMA warp runs up to three groups ahead of the barrier round trip that
// frees a buffer) and sixteen rescale warps fold it into an fp32 accumulator in
// registers,
// acc = fma(P_g, RN(sa * sb), acc) in group order (sa * sb is exact in fp32:
// both are fp16 values), while the MMA warp fills the other buffers.  The bf16
// branch product u' L^T comes last, as one more group with scale 1.
//
// CTA = one 128 x 128 output tile (one K split of it), 18 warps:
//   warp 0    TMA producer.  A stage is K 128 (two groups): the A and B level
//             boxes (128 rows x 128 bytes, 128B swizzle) and the two groups'
//             fp32 scales of the tile's rows and of its columns; U and L once.
//             The weight boxes of the first stage go out before the wait on
//             the kernel that writes A.
//   warp 1    TMEM owner and MMA issuer: two MMAs (K 32) per group into
//             buffer g % 4.
//   warps 2-17 rescale and epilogue: warp w reads TMEM lane quarter w % 4,
//             columns [32 h, 32 h + 32), h = (w - 2) / 4: one thread = one
//             output row x 32 columns.  The rescale is a chain of dependent
//             loads and packed FMAs per group; four such warps per scheduler
//             keep its issue slots busy where two left them idle two thirds of
//             the time.
// Split K (few output tiles): each split writes its fp32 partial tile and a
// second kernel sums the splits in order, adds the bias and rounds to bf16.
// Every mbarrier wait is bounded.  No TMA multicast.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwam {
namespace {

constexpr int kTile = 128;
constexpr int kStages = 5;
constexpr int kOffA = 0;
constexpr int kOffB = 16384;
constexpr int kOffSA = 32768;   // [2 groups][128 rows] fp32
constexpr int kOffSB = 33792;   // [2 groups][128 columns] fp32
constexpr int kStageBytes = 34816;
constexpr int kOffU = kStages * kStageBytes;  // u' tile: 128 rows x r bf16 (r <= 32)
constexpr int kOffL = kOffU + 8192;           // L tile: 128 rows x r bf16
constexpr int kOffBar = kOffL + 8192;
constexpr int kSmem = kOffBar + 256 + 1024;
constexpr int kRescaleWarp0 = 2;
constexpr int kRescaleWarps = 16;
constexpr int kCols = kTile * 4 / kRescaleWarps;  // output columns per rescale thread
static_assert(kCols == 32, "one 32-column TMEM load per group per rescale thread");
constexpr int kThreads = 32 * (kRescaleWarp0 + kRescaleWarps);
constexpr int kBufs = 4;             // 128-column TMEM group buffers
constexpr uint32_t kTmemCols = 128 * kBufs;

// acc0/1 += P0/1 * RN(w0/1 * a): two packed fp32 operations (RN(w a) is exact
// here: w and a are fp16 values), written as one block so the pairs are formed
// in registers once.
__device__ __forceinline__ void rescale2(float& acc0, float& acc1, uint32_t p0, uint32_t p1, float w0, float w1,
                                         float a) {
  asm("{\n\t.reg .b64 pp, ww, aa, cc;\n\t"
      "mov.b64 pp, {%2, %3};\n\t"
      "mov.b64 ww, {%4, %5};\n\t"
      "mov.b64 aa, {%6, %6};\n\t"
      "mov.b64 cc, {%0, %1};\n\t"
      "mul.rn.f32x2 ww, ww, aa;\n\t"
      "fma.rn.f32x2 cc, pp, ww, cc;\n\t"
      "mov.b64 {%0, %1}, cc;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "r"(p0), "r"(p1), "f"(w0), "f"(w1), "f"(a));
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
static_assert(kSmem <= 227 * 1024, "shared memory budget");
static_assert(kStageBytes % 1024 == 0, "128B-swizzled boxes stay 1024-byte aligned");

__global__ void __launch_bounds__(kThreads, 1)
    group_gemm_kernel(const __grid_constant__ GroupGemmMaps maps, const GroupGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [kStages] levels and scales landed
  uint64_t* empty = full + kStages;                               // [kStages] MMAs done with the levels
  uint64_t* sc_free = empty + kStages;                            // [kStages] rescale warps done with the scales
  uint64_t* acc_full = sc_free + kStages;                         // [kBufs] a group's P in the buffer
  uint64_t* acc_empty = acc_full + kBufs;                         // [kBufs] the buffer read out
  uint64_t* branch_full = acc_empty + kBufs;
  uint64_t* mma_done = branch_full + 1;  // every MMA of this CTA complete (before TMEM is freed)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  const int n0 = static_cast<int>(blockIdx.x) * kTile;
  const int m0 = static_cast<int>(blockIdx.y) * kTile;
  const int split = static_cast<int>(blockIdx.z);
  const int k_stages = p.K / 128;
  const int s_begin = split * k_stages / p.splits;
  const int n_st = (split + 1) * k_stages / p.splits - s_begin;
  const bool branch = p.branch_k > 0 && split == 0;
  const int n_groups = 2 * n_st + (branch ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&sc_free[i], kRescaleWarps);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kRescaleWarps);
    }
    mbar_init(branch_full, 1);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();  // the next kernel may start its set-up

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&maps.a);
      tma_prefetch_desc(&maps.b);
      tma_prefetch_desc(&maps.sa);
      tma_prefetch_desc(&maps.sb);
      if (branch) {
        tma_prefetch_desc(&maps.u);
        tma_prefetch_desc(&maps.l);
        mbar_arrive_expect_tx(branch_full, 2u * kTile * static_cast<uint32_t>(p.branch_k) * 2u);
        tma_load_2d(smem + kOffL, &maps.l, branch_full, 0, n0);  // a layer constant
      }
      bool ok = true, dep = false;
      int last = -1;
      for (int s = 0; ok && s < n_st; ++s) {
        const int st = s % kStages;
        const int use = s / kStages;
        if (use > 0) {
          const uint32_t par = static_cast<uint32_t>(use - 1) & 1u;
          ok = mbar_wait(&empty[st], par, p.err, DEVERR_PRODUCER_WAIT, wlim) &&
               mbar_wait(&sc_free[st], par, p.err, DEVERR_PRODUCER_WAIT, wlim);
          if (!ok) break;
        }
        uint8_t* base = smem + st * kStageBytes;
        const int kst = s_begin + s;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
        tma_load_3d(base + kOffB, &maps.b, &full[st], kst * 128, n0, 0);
        tma_load_2d(base + kOffSB, &maps.sb, &full[st], n0, 2 * kst);
        if (!dep) {
          // A, its scales and u' are written by the kernel before this one
          griddep_wait();
          dep = true;
          if (branch) tma_load_2d(smem + kOffU, &maps.u, branch_full, 0, m0);
        }
        tma_load_3d(base + kOffA, &maps.a, &full[st], kst * 128, m0, 0);
        tma_load_2d(base + kOffSA, &maps.sa, &full[st], m0, 2 * kst);
        last = s;
      }
      if (!dep) {
        griddep_wait();
        if (branch && ok) tma_load_2d(smem + kOffU, &maps.u, branch_full, 0, m0);
      }
      // every copy issued lands before the CTA exits
      if (last >= 0) mbar_wait(&full[last % kStages], static_cast<uint32_t>(last / kStages) & 1u, p.err,
                               DEVERR_DRAIN_WAIT, wlim);
      if (branch) mbar_wait(branch_full, 0, p.err, DEVERR_DRAIN_WAIT, wlim);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f8e4m3(kTile, kTile);
      bool ok = true;
      // buffer g % kBufs read out by the rescale warps since its last group
      auto take = [&](int g) {
        const int use = g / kBufs;
        return use == 0 || mbar_wait(&acc_empty[g % kBufs], static_cast<uint32_t>(use - 1) & 1u, p.err,
                                     DEVERR_MMA_WAIT, wlim);
      };
      int g = 0;
      for (int s = 0; ok && s < n_st; ++s) {
        const int st = s % kStages;
        if (!mbar_wait(&full[st], static_cast<uint32_t>(s / kStages) & 1u, p.err, DEVERR_MMA_WAIT, wlim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_s = smem_u32(smem + st * kStageBytes + kOffA);
        const uint32_t b_s = smem_u32(smem + st * kStageBytes + kOffB);
        for (int j = 0; j < 2; ++j, ++g) {
          if (!take(g)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + 128u * static_cast<uint32_t>(g % kBufs);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // 32 bytes of each operand row per MMA (K 32), inside the 128-byte swizzle atom
            const uint64_t ad = smem_desc(a_s + j * 64 + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_s + j * 64 + kk * 32, 16, 1024, 2);
            mma_f8(d, ad, bd, idesc, kk ? 1u : 0u);
          }
          tc_commit(&acc_full[g % kBufs]);
        }
        tc_commit(&empty[st]);
      }
      if (ok && branch && take(g) && mbar_wait(branch_full, 0, p.err, DEVERR_BRANCH_WAIT, wlim)) {
        tc_fence_after();
        const uint32_t layout = p.branch_k == 32 ? 4u : 6u;  // 64B / 32B swizzle
        const uint32_t sbo = 8u * static_cast<uint32_t>(p.branch_k) * 2u;
        const uint32_t us = smem_u32(smem + kOffU), ls = smem_u32(smem + kOffL);
        const uint32_t d = tmem + 128u * static_cast<uint32_t>(g % kBufs);
        for (int kk = 0; kk < p.branch_k / 16; ++kk)
          mma_bf16(d, smem_desc(us + kk * 32, 16, sbo, layout), smem_desc(ls + kk * 32, 16, sbo, layout),
                   idesc_bf16(kTile, kTile), kk ? 1u : 0u);
        tc_commit(&acc_full[g % kBufs]);
      }
      // on every path (an expired wait included) no MMA may still be writing
      // TMEM when it is freed
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, p.err, DEVERR_DRAIN_WAIT, wlim);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ rescale and epilogue
    const int ew = warp - kRescaleWarp0;  // 0..15
    const int qd = warp & 3;              // TMEM lane quarter this warp may access
    const int h = ew >> 2;                // column quarter
    const int row_l = qd * 32 + lane;
    const int row = m0 + row_l;
    const int c0 = n0 + h * kCols;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(qd * 32) << 16) + static_cast<uint32_t>(h * kCols);
    float acc[kCols];
#pragma unroll
    for (int q = 0; q < kCols; ++q) acc[q] = 0.0f;
    griddep_wait();  // y / the partial tiles may still be read by the kernel before this one
    bool alive = true;
    for (int g = 0; alive && g < n_groups; ++g) {
      const int b = g % kBufs;
      // warp-uniform outcome: the TMEM loads below are warp-collective
      alive = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], static_cast<uint32_t>(g / kBufs) & 1u, p.err,
                                                DEVERR_EPILOGUE_WAIT, wlim));
      if (!alive) break;
      tc_fence_after();
      uint32_t r0[32];
      tmem_ld_32x32b_x32(taddr + 128u * static_cast<uint32_t>(b), r0);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
      if (g < 2 * n_st) {
        const int s = g >> 1, j = g & 1, st = s % kStages;
        // the stage's TMA writes (the scales) are complete and visible
        if (j == 0)
          alive = __all_sync(0xffffffffu, mbar_wait(&full[st], static_cast<uint32_t>(s / kStages) & 1u, p.err,
                                                     DEVERR_EPILOGUE_WAIT, wlim));
        const uint32_t sbase = smem_u32(smem + st * kStageBytes);
        const uint32_t sa = sbase + kOffSA + 4u * static_cast<uint32_t>(j * kTile);
        const uint32_t sb = sbase + kOffSB + 4u * static_cast<uint32_t>(j * kTile + h * kCols);
        const float a = lds_f32(sa + 4u * static_cast<uint32_t>(row_l));
#pragma unroll
        for (int q = 0; q < kCols / 4; ++q) {
          const float4 w4 = lds_f32x4(sb + 16u * q);
          rescale2(acc[4 * q], acc[4 * q + 1], r0[4 * q], r0[4 * q + 1], w4.x, w4.y, a);
          rescale2(acc[4 * q + 2], acc[4 * q + 3], r0[4 * q + 2], r0[4 * q + 3], w4.z, w4.w, a);
        }
        __syncwarp();
        if (j == 1 && lane == 0) mbar_arrive(&sc_free[st]);
      } else {
        // the branch u' L^T, scale 1
#pragma unroll
        for (int q = 0; q < kCols; ++q) acc[q] = __fadd_rn(acc[q], __uint_as_float(r0[q]));
      }
    }
    if (alive && row < p.M) {
      if (p.y) {
        // y = bf16(acc + bias), 16 bytes per store
        const uint16_t* bias = static_cast<const uint16_t*>(p.bias);
        uint16_t* yrow = static_cast<uint16_t*>(p.y) + static_cast<size_t>(row) * p.N;
#pragma unroll
        for (int q8 = 0; q8 < kCols / 8; ++q8) {
          const int n = c0 + 8 * q8;
          if (n >= p.N) break;
          const uint4 bw = bias ? __ldg(reinterpret_cast<const uint4*>(bias + n)) : make_uint4(0u, 0u, 0u, 0u);
          const float* a8 = acc + 8 * q8;
          const uint4 o = make_uint4(fma_bf16x2(a8[0], a8[1], 1.0f, bw.x), fma_bf16x2(a8[2], a8[3], 1.0f, bw.y),
                                     fma_bf16x2(a8[4], a8[5], 1.0f, bw.z), fma_bf16x2(a8[6], a8[7], 1.0f, bw.w));
          *reinterpret_cast<uint4*>(yrow + n) = o;
        }
      } else {
        float* prow = p.partial + (static_cast<size_t>(split) * p.M + row) * p.N;
#pragma unroll
        for (int q4 = 0; q4 < kCols / 4; ++q4) {
          const int n = c0 + 4 * q4;
          if (n >= p.N) break;
          *reinterpret_cast<float4*>(prow + n) = make_float4(acc[4 * q4], acc[4 * q4 + 1], acc[4 * q4 + 2], acc[4 * q4 + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// y[m, n .. n + 7] = bf16(sum_s partial[s][m][n ..] + bias[n ..]), the splits
// added in order (fp32), one thread per 8 columns.
__global__ void splitk_finalize_kernel(const float* __restrict__ partial, int splits, int M, int N,
                                       const uint16_t* __restrict__ bias, uint16_t* __restrict__ y) {
  griddep_wait();
  griddep_launch_dependents();
  const size_t n8 = static_cast<size_t>(N / 8);
  const size_t total = static_cast<size_t>(M) * n8;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t m = i / n8, c = (i % n8) * 8;
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = 0.0f;
    for (int s = 0; s < splits; ++s) {
      const float4* src = reinterpret_cast<const float4*>(partial + (static_cast<size_t>(s) * M + m) * N + c);
      const float4 a = src[0], b = src[1];
      v[0] = __fadd_rn(v[0], a.x); v[1] = __fadd_rn(v[1], a.y); v[2] = __fadd_rn(v[2], a.z); v[3] = __fadd_rn(v[3], a.w);
      v[4] = __fadd_rn(v[4], b.x); v[5] = __fadd_rn(v[5], b.y); v[6] = __fadd_rn(v[6], b.z); v[7] = __fadd_rn(v[7], b.w);
    }
    const uint4 bw = bias ? *reinterpret_cast<const uint4*>(bias + c) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(y + m * N + c) =
        make_uint4(fma_bf16x2(v[0], v[1], 1.0f, bw.x), fma_bf16x2(v[2], v[3], 1.0f, bw.y),
                   fma_bf16x2(v[4], v[5], 1.0f, bw.z), fma_bf16x2(v[6], v[7], 1.0f, bw.w));
  }
}

cudaError_t launch_pdl(const void* kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace

cudaError_t launch_group_gemm(const GroupGemmMaps& maps, const GroupGemmParams& p, cudaStream_t st) {
  if (p.K <= 0 || p.K % 128 || p.splits < 1 || p.splits > p.K / 128 || p.M <= 0 || p.N <= 0 || p.N % 16 ||
      (p.branch_k != 0 && p.branch_k != 16 && p.branch_k != 32) || (!p.y && !p.partial) || (p.y && p.splits != 1))
    return cudaErrorInvalidValue;
  static const cudaError_t smem_attr =
      cudaFuncSetAttribute(group_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (smem_attr != cudaSuccess) return smem_attr;
  const dim3 grid((p.N + kTile - 1) / kTile, (p.M + kTile - 1) / kTile, p.splits);
  GroupGemmMaps m = maps;
  GroupGemmParams q = p;
  void* args[] = {&m, &q};
  return launch_pdl(reinterpret_cast<const void*>(group_gemm_kernel), grid, dim3(kThreads), kSmem, st, args);
}

cudaError_t launch_splitk_finalize(const float* partial, int splits, int M, int N, const void* bias, void* y,
                                   cudaStream_t st) {
  if (M <= 0 || N <= 0 || N % 8 || splits < 1) return cudaErrorInvalidValue;
  const size_t items = static_cast<size_t>(M) * (N / 8);
  const int blocks = static_cast<int>(std::min<size_t>((items + 255) / 256, 148 * 8));
  const float* pp = partial;
  int s = splits, mm = M, nn = N;
  const uint16_t* bb = static_cast<const uint16_t*>(bias);
  uint16_t* yy = static_cast<uint16_t*>(y);
  void* args[] = {&pp, &s, &mm, &nn, &bb, &yy};
  return launch_pdl(reinterpret_cast<const void*>(splitk_finalize_kernel), dim3(blocks), dim3(256), 0, st, args);
}

}  // namespace qwam
