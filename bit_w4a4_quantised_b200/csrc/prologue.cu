// Activation prologue and weight prepare: one row pipeline for both sides of
// the deflated ASP layer ("FastWAM UR3 3-task — 4-bit quantisations", section
// "What ASP is, and what the deflated form means"):
//
//   T~ = (T * chan) H           per-channel scale, block FWHT (one thread = one row)
//   c  = T~ V                   rank-r coordinates, tcgen05 bf16 MMA into TMEM
//   Z  = T~ - c V^T             deflation, tcgen05 bf16 MMA into TMEM
//   amax(Z) -> g, quantise(Z)   NVFP4 codes + 128x4-tiled E4M3 scales
//   branch operand              bf16(c)  (weight side: W~V)  or
//                               bf16(c / (g_x g_w))  (activation side)
//
// T = x and chan = 1/s on the activation side, T = W and chan = s on the weight
// side.  Both rank-r products run on the tensor cores with a hi/lo bf16 split of
// each operand (three MMAs per K step; plain bf16 flips ~0.2 % of the FP4 codes
// against a float64 reference, the split keeps it below 0.01 %).
//
// CTA = 128 rows (one TMEM lane per row) x `chunks` 128-column chunks, 7 warps:
//   warps 0-3  row threads: read their row of x from a TMA-filled ring, scale,
//              FWHT in registers, write T~ (hi/lo) as the MMA A operand, read
//              u and Z from TMEM, reduce amax, quantise in registers;
//   warps 4, 6 TMA producers (x tiles, V tiles, chan), one per ring slot;
//   warp 5     TMEM owner and MMA issuer.
// The CTAs of a row tile form a cluster along K: partial c is summed across it
// through distributed shared memory in rank order (deterministic).
//
// Modes: Fused (rows <= 128: the cluster holds the whole tensor, so amax is a
// cluster reduction and one launch finishes the job), Stats (c to global,
// atomic amax) and Quantise (reads c and amax, recomputes Z bit-identically from
// the same code and data, quantises).  Every wait on an mbarrier is bounded.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace cg = cooperative_groups;

namespace qwam {
namespace {

constexpr int kRows = 128;
constexpr int kChunk = 128;
constexpr int kThreads = 224;  // 4 row warps, producer warps 4 and 6, MMA warp 5

template <int R, int MODE>
struct PCfg {
  static constexpr bool kMMA = R > 0;
  static constexpr bool kProj = R > 0 && MODE != 2;        // sweep computing c
  static constexpr bool kA = MODE != 2 && R > 0;           // cluster exchange of c
  static constexpr bool kB = MODE == 0;                    // cluster exchange of amax
  static constexpr bool kC = kA || kB;                     // keep smem alive for peers
  static constexpr int X_BYTES = kRows * kChunk * 2;       // two 64-column SW128 boxes
  static constexpr int V_BYTES = 512 * R;                  // V^T hi/lo (sweep 1) or V hi/lo
  static constexpr int CH_BYTES = kChunk * 4;
  static constexpr int SLOT = (X_BYTES + V_BYTES + CH_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_XT = 2 * SLOT;                  // T~ hi/lo as MMA A, 4 x 16 KB
  static constexpr int XT_BYTES = kProj ? 4 * 16384 : 0;
  static constexpr int OFF_UA = OFF_XT + XT_BYTES;         // c hi/lo as MMA A
  static constexpr int UA_BYTES = kMMA ? 512 * R : 0;
  static constexpr int OFF_BAR = OFF_UA + UA_BYTES;
  static constexpr int OFF_MISC = OFF_BAR + 128;
  static constexpr int SMEM = OFF_MISC + 64 + 1024;
  static constexpr int UP_STRIDE = R + 4;                  // fp32 partial c rows (aliases T~)
  static constexpr uint32_t TMEM_COLS = kMMA ? (MODE == 2 ? 128u : 256u) : 32u;
  static_assert(!kProj || kRows * UP_STRIDE * 4 <= 32768, "partial and parked c must fit in the T~ area");
};

__device__ __forceinline__ void unpack8(uint4 w, float* o) {
  o[0] = __uint_as_float(w.x << 16); o[1] = __uint_as_float(w.x & 0xffff0000u);
  o[2] = __uint_as_float(w.y << 16); o[3] = __uint_as_float(w.y & 0xffff0000u);
  o[4] = __uint_as_float(w.z << 16); o[5] = __uint_as_float(w.z & 0xffff0000u);
  o[6] = __uint_as_float(w.w << 16); o[7] = __uint_as_float(w.w & 0xffff0000u);
}

// This thread's row of one chunk: x (bf16, SW128 TMA tile) * chan, then the
// block FWHT in registers (Sylvester order, butterflies (lo+hi, lo-hi)), then
// the 1/sqrt(b) scale.  Identical code and op order in every sweep.
__device__ __forceinline__ void rotate_row(const uint8_t* slot, const float* chan, int t, int b, float hscale,
                                           float (&v)[kChunk]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint8_t* rowp = slot + h * 16384 + t * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((j ^ (t & 7)) << 4));
      unpack8(w, v + h * 64 + j * 8);
    }
  }
#pragma unroll
  for (int i = 0; i < kChunk; i += 4) {
    const float4 c = *reinterpret_cast<const float4*>(chan + i);
    v[i] = __fmul_rn(v[i], c.x);
    v[i + 1] = __fmul_rn(v[i + 1], c.y);
    v[i + 2] = __fmul_rn(v[i + 2], c.z);
    v[i + 3] = __fmul_rn(v[i + 3], c.w);
  }
#pragma unroll
  for (int s = 0; s < 7; ++s) {
    const int hh = 1 << s;
    if (hh < b) {
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        if (!(i & hh)) {
          const float a = v[i], c = v[i + hh];
          v[i] = __fadd_rn(a, c);
          v[i + hh] = __fsub_rn(a, c);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kChunk; ++i) v[i] = __fmul_rn(v[i], hscale);
}

// Row t of a K-major bf16 operand tile with W-byte rows (one swizzle atom wide):
// write 8 consecutive elements (16 bytes) as logical chunk j.
__device__ __forceinline__ void put16(uint8_t* tile, int t, int j, int W, uint4 w) {
  *reinterpret_cast<uint4*>(tile + t * W + (swz_chunk(t, j, W) << 4)) = w;
}

__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint16_t h0, l0, h1, l1;
    split_bf16(v[2 * k], h0, l0);
    split_bf16(v[2 * k + 1], h1, l1);
    h[k] = pack2(h0, h1);
    l[k] = pack2(l0, l1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Quantise this thread's 128 values of row `row`, columns [col, col+128).
__device__ __forceinline__ void quantise_row(const PrologueParams& p, const float (&v)[kChunk], int row, int col,
                                             float g) {
  uint32_t cw[16];
  uint32_t sfw[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float blk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) blk[e] = v[16 * k + e];
    uint32_t c2[2];
    const uint32_t S = quant_block16(blk, g, c2);
    cw[2 * k] = c2[0];
    cw[2 * k + 1] = c2[1];
    sfw[k >> 2] |= S << (8 * (k & 3));
  }
  uint4* dst = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * (p.K / 2) + col / 2);
#pragma unroll
  for (int k = 0; k < 4; ++k) dst[k] = make_uint4(cw[4 * k], cw[4 * k + 1], cw[4 * k + 2], cw[4 * k + 3]);
  *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, col / 16, p.K)) = sfw[0];
  *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, col / 16 + 4, p.K)) = sfw[1];
  if (p.z_out) {
    float4* z = reinterpret_cast<float4*>(p.z_out + static_cast<size_t>(row) * p.K + col);
#pragma unroll
    for (int k = 0; k < kChunk / 4; ++k) z[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  }
}

template <int R>
__device__ __forceinline__ void write_branch(const PrologueParams& p, const float (&u)[R > 0 ? R : 1], int row,
                                             float g) {
  if constexpr (R > 0) {
    const float gs = __fmul_rn(g, p.g_other);
    uint32_t w[R / 2];
#pragma unroll
    for (int j = 0; j < R / 2; ++j) {
      float a = u[2 * j], b = u[2 * j + 1];
      if (p.branch_mode == 1) {
        a = __fdiv_rn(a, gs);
        b = __fdiv_rn(b, gs);
      }
      w[j] = pack2(bf16_bits_rn(a), bf16_bits_rn(b));
    }
    uint4* dst = reinterpret_cast<uint4*>(p.branch + static_cast<size_t>(row) * R);
#pragma unroll
    for (int j = 0; j < R / 8; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    if (p.u_out) {
      float4* o = reinterpret_cast<float4*>(p.u_out + static_cast<size_t>(row) * R);
#pragma unroll
      for (int j = 0; j < R / 4; ++j) o[j] = make_float4(u[4 * j], u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
    }
  }
}

template <int R, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prologue_kernel(const __grid_constant__ ProMaps maps, const PrologueParams p) {
  using C = PCfg<R, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* xs_full = bars;      // [2] TMA landed
  uint64_t* xs_free = bars + 2;  // [2] rows (and MMA) done with the slot
  uint64_t* xt_full = bars + 4;  // rows wrote T~ for the next projection
  uint64_t* xt_free = bars + 5;  // projection MMAs done with T~
  uint64_t* u_full = bars + 6;   // all projection MMAs done
  uint64_t* ua_full = bars + 7;  // rows wrote c hi/lo
  uint64_t* d2_full = bars + 8;  // deflation MMAs done
  uint64_t* d2_free = bars + 9;  // rows read the deflation result
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  float* red = reinterpret_cast<float*>(smem + C::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x;
  const int m0 = blockIdx.y * kRows;
  const int nch = p.chunks;
  const int col0 = part * nch * kChunk;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xs_full[i], 1);
      mbar_init(&xs_free[i], kRows + (C::kMMA ? 1 : 0));
    }
    mbar_init(xt_full, kRows);
    mbar_init(xt_free, 1);
    mbar_init(u_full, 1);
    mbar_init(ua_full, kRows);
    mbar_init(d2_full, 1);
    mbar_init(d2_free, kRows);
    fence_barrier_init();
  }
  if constexpr (C::kMMA) {
    if (warp == 5) {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C::kMMA ? *tmem_slot : 0u;
  const uint32_t d2_tmem = tmem;
  const uint32_t u_tmem = tmem + 128;

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ producers
    // A TMA instruction occupies its warp for a fixed ~600 cycles whatever its
    // size: every slot has its own producer warp (4: even loads, 6: odd loads)
    // and a slot's tiles (x, V^T or V) go out as one converged instruction.
    const int my_slot = warp == 4 ? 0 : 1;
    int i = 0, last = -1;
    auto load = [&](int c, bool proj) {
      const int slot = i & 1;
      if (slot != my_slot) {
        ++i;
        return true;
      }
      int ok = 1;
      if (lane == 0 && i >= 2)
        ok = mbar_wait(&xs_free[slot], ((i >> 1) & 1) ^ 1u, p.err, DEVERR_PRODUCER_WAIT) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      uint8_t* s = smem + slot * C::SLOT;
      const int col = col0 + c * kChunk;
      if (lane == 0) mbar_arrive_expect_tx(&xs_full[slot], C::X_BYTES + C::V_BYTES + C::CH_BYTES);
      __syncwarp();
      const CUtensorMap* m = nullptr;
      uint8_t* dst = s;
      int x = 0, y = 0;
      if (lane < 2) {
        m = &maps.x; dst = s + lane * 16384; x = col + 64 * lane; y = m0;
      } else if (R > 0 && proj && lane < 6) {
        const int pp = (lane - 2) >> 1, kb = (lane - 2) & 1;
        m = pp ? &maps.vt_lo : &maps.vt_hi; dst = s + C::X_BYTES + (pp * 2 + kb) * R * 128; x = col + kb * 64; y = 0;
      } else if (R > 0 && !proj && lane < 4) {
        const int pp = lane - 2;
        m = pp ? &maps.v_lo : &maps.v_hi; dst = s + C::X_BYTES + pp * 256 * R; x = 0; y = col;
      }
      if (m) tma_load_2d(dst, m, &xs_full[slot], x, y);
      if (lane == 0) bulk_load(s + C::X_BYTES + C::V_BYTES, p.chan + col, C::CH_BYTES, &xs_full[slot]);
      last = i;
      ++i;
      return true;
    };
    bool ok = true;
    if (lane == 0 && warp == 4) {
      tma_prefetch_desc(&maps.x);
      if constexpr (R > 0) {
        tma_prefetch_desc(&maps.vt_hi); tma_prefetch_desc(&maps.vt_lo);
        tma_prefetch_desc(&maps.v_hi); tma_prefetch_desc(&maps.v_lo);
      }
    }
    __syncwarp();
    if constexpr (C::kA) cluster_arrive();
    if constexpr (C::kProj)
      for (int c = 0; ok && c < nch; ++c) ok = load(c, true);
    for (int c = 0; ok && c < nch; ++c) ok = load(c, false);
    __syncwarp();
    if constexpr (C::kA) cluster_wait();
    if constexpr (C::kB) {
      cluster_arrive();
      for (int c = 0; ok && c < nch; ++c) ok = load(c, false);
      __syncwarp();
    }
    if (lane == 0 && last >= 0) mbar_wait(&xs_full[last & 1], (last >> 1) & 1, p.err, DEVERR_DRAIN_WAIT);
    __syncwarp();
    if constexpr (C::kB) cluster_wait();
    if constexpr (C::kC) {
      cluster_arrive();
      cluster_wait();
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (C::kMMA) {
      int i = 0, j = 0;
      bool ok = true;
      const uint32_t sbo_u = 8u * 2u * R;
      const uint32_t swz_u = umma_swizzle_code(2 * R);
      // deflation of one chunk: D2[128 x 128] = c (hi/lo) . V_chunk^T (hi/lo)
      auto deflate_chunk = [&]() {
        const int slot = i & 1;
        if (!mbar_wait(&xs_full[slot], (i >> 1) & 1, p.err, DEVERR_MMA_WAIT)) return false;
        if (!mbar_wait(d2_free, (j & 1) ^ 1u, p.err, DEVERR_MMA_WAIT)) return false;
        tc_fence_after();
        const uint32_t vs = smem_u32(smem + slot * C::SLOT + C::X_BYTES);
        const uint32_t ua = smem_u32(smem + C::OFF_UA);
#pragma unroll
        for (int k = 0; k < R / 16; ++k) {
          const uint64_t ah = smem_desc(ua + k * 32, 16, sbo_u, swz_u);
          const uint64_t al = smem_desc(ua + 256 * R + k * 32, 16, sbo_u, swz_u);
          const uint64_t bh = smem_desc(vs + k * 32, 16, sbo_u, swz_u);
          const uint64_t bl = smem_desc(vs + 256 * R + k * 32, 16, sbo_u, swz_u);
          mma_bf16(d2_tmem, al, bh, idesc_bf16(128, 128), k > 0 ? 1u : 0u);
          mma_bf16(d2_tmem, ah, bl, idesc_bf16(128, 128), 1u);
          mma_bf16(d2_tmem, ah, bh, idesc_bf16(128, 128), 1u);
        }
        tc_commit(d2_full);
        tc_commit(&xs_free[slot]);
        ++i;
        ++j;
        return true;
      };
      if constexpr (C::kProj) {
        if (lane == 0) {
          uint32_t acc = 0;
          for (int c = 0; ok && c < nch; ++c) {
            const int slot = i & 1;
            ok = mbar_wait(&xs_full[slot], (i >> 1) & 1, p.err, DEVERR_MMA_WAIT) &&
                 mbar_wait(xt_full, c & 1, p.err, DEVERR_MMA_WAIT);
            if (!ok) break;
            tc_fence_after();
            const uint32_t vs = smem_u32(smem + slot * C::SLOT + C::X_BYTES);
            const uint32_t xt = smem_u32(smem + C::OFF_XT);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ah = smem_desc(xt + kb * 16384 + k * 32, 16, 1024, 2);
                const uint64_t al = smem_desc(xt + (2 + kb) * 16384 + k * 32, 16, 1024, 2);
                const uint64_t bh = smem_desc(vs + kb * R * 128 + k * 32, 16, 1024, 2);
                const uint64_t bl = smem_desc(vs + (2 + kb) * R * 128 + k * 32, 16, 1024, 2);
                mma_bf16(u_tmem, al, bh, idesc_bf16(128, R), acc);
                mma_bf16(u_tmem, ah, bl, idesc_bf16(128, R), 1u);
                mma_bf16(u_tmem, ah, bh, idesc_bf16(128, R), 1u);
                acc = 1u;
              }
            tc_commit(xt_free);
            tc_commit(&xs_free[slot]);
            ++i;
          }
          tc_commit(u_full);
        }
        __syncwarp();
      }
      if constexpr (C::kA) cluster_arrive();
      if (lane == 0) {
        ok = ok && mbar_wait(ua_full, 0, p.err, DEVERR_MMA_WAIT);
        for (int c = 0; ok && c < nch; ++c) ok = deflate_chunk();
      }
      __syncwarp();
      if constexpr (C::kA) cluster_wait();
      if constexpr (C::kB) {
        cluster_arrive();
        if (lane == 0)
          for (int c = 0; ok && c < nch; ++c) ok = deflate_chunk();
        __syncwarp();
        cluster_wait();
      }
    } else {
      if constexpr (C::kB) cluster_sync_all();
    }
    if constexpr (C::kC) {
      cluster_arrive();
      cluster_wait();
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int t = threadIdx.x;  // 0..127 = TMEM lane = row within the tile
    const int row = m0 + t;
    const bool valid = row < p.rows;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float v[kChunk];
    float u[R > 0 ? R : 1];
#pragma unroll
    for (int k = 0; k < (R > 0 ? R : 1); ++k) u[k] = 0.0f;
    int i = 0, j = 0;

    if constexpr (C::kProj) {
      for (int c = 0; c < nch; ++c) {
        const int slot = i & 1;
        mbar_wait(&xs_full[slot], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
        const uint8_t* s = smem + slot * C::SLOT;
        rotate_row(s, reinterpret_cast<const float*>(s + C::X_BYTES + C::V_BYTES), t, p.b, p.hscale, v);
        mbar_arrive(&xs_free[slot]);
        mbar_wait(xt_free, (c & 1) ^ 1u, p.err, DEVERR_EPILOGUE_WAIT);
        uint8_t* xt = smem + C::OFF_XT;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint4 hi, lo;
            split8(v + kb * 64 + q * 8, hi, lo);
            put16(xt + kb * 16384, t, q, 128, hi);
            put16(xt + (2 + kb) * 16384, t, q, 128, lo);
          }
        fence_proxy_async();
        mbar_arrive(xt_full);
        ++i;
      }
      // c of this CTA's K range -> shared memory -> sum over the cluster
      mbar_wait(u_full, 0, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
      tc_fence_after();
      {
        uint32_t r32[32];
        tmem_ld_32x32b_x32(u_tmem + lane_base, r32);
        tmem_ld_wait();
        float* up = reinterpret_cast<float*>(smem + C::OFF_XT) + t * C::UP_STRIDE;
#pragma unroll
        for (int k = 0; k < R; k += 4)
          *reinterpret_cast<float4*>(up + k) = make_float4(__uint_as_float(r32[k]), __uint_as_float(r32[k + 1]),
                                                           __uint_as_float(r32[k + 2]), __uint_as_float(r32[k + 3]));
      }
      cluster_arrive();
      cluster_wait();
      cg::cluster_group cluster = cg::this_cluster();
      const int nranks = static_cast<int>(cluster.num_blocks());
      for (int rk = 0; rk < nranks; ++rk) {
        const float* rp = cluster.map_shared_rank(reinterpret_cast<float*>(smem + C::OFF_XT), rk) + t * C::UP_STRIDE;
#pragma unroll
        for (int k = 0; k < R; k += 4) {
          const float4 a = *reinterpret_cast<const float4*>(rp + k);
          u[k] = __fadd_rn(u[k], a.x);
          u[k + 1] = __fadd_rn(u[k + 1], a.y);
          u[k + 2] = __fadd_rn(u[k + 2], a.z);
          u[k + 3] = __fadd_rn(u[k + 3], a.w);
        }
      }
      if (MODE == 1 && part == 0 && valid) {
        float4* o = reinterpret_cast<float4*>(p.u_glob + static_cast<size_t>(row) * R);
#pragma unroll
        for (int k = 0; k < R / 4; ++k) o[k] = make_float4(u[4 * k], u[4 * k + 1], u[4 * k + 2], u[4 * k + 3]);
      }
    }
    if constexpr (MODE == 2 && R > 0) {
      if (valid) {
        const float4* src = reinterpret_cast<const float4*>(p.u_glob + static_cast<size_t>(row) * R);
#pragma unroll
        for (int k = 0; k < R / 4; ++k) {
          const float4 a = src[k];
          u[4 * k] = a.x; u[4 * k + 1] = a.y; u[4 * k + 2] = a.z; u[4 * k + 3] = a.w;
        }
        if (part == 0) write_branch<R>(p, u, row, global_scale_from_amax(__uint_as_float(*p.amax_glob)));
      }
    }
    if constexpr (MODE == 0 && R > 0) {
      // park the cluster-summed c in the (now idle) T~ area until g is known
      float* uf = reinterpret_cast<float*>(smem + C::OFF_XT + 32768) + t * C::UP_STRIDE;
#pragma unroll
      for (int k = 0; k < R; k += 4) *reinterpret_cast<float4*>(uf + k) = make_float4(u[k], u[k + 1], u[k + 2], u[k + 3]);
    }
    if constexpr (C::kMMA) {
      uint8_t* ua = smem + C::OFF_UA;
#pragma unroll
      for (int q = 0; q < R / 8; ++q) {
        uint4 hi, lo;
        split8(u + q * 8, hi, lo);
        put16(ua, t, q, 2 * R, hi);
        put16(ua + 256 * R, t, q, 2 * R, lo);
      }
      fence_proxy_async();
      mbar_arrive(ua_full);
    }

    // Z sweeps: Z = T~ - c V^T per chunk, then amax and / or quantisation.
    auto z_chunk = [&](int c) {
      const int slot = i & 1;
      mbar_wait(&xs_full[slot], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      const uint8_t* s = smem + slot * C::SLOT;
      rotate_row(s, reinterpret_cast<const float*>(s + C::X_BYTES + C::V_BYTES), t, p.b, p.hscale, v);
      mbar_arrive(&xs_free[slot]);
      if constexpr (C::kMMA) {
        mbar_wait(d2_full, j & 1, p.err, DEVERR_EPILOGUE_WAIT);
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t r32[32];
          tmem_ld_32x32b_x32(d2_tmem + lane_base + q * 32, r32);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[q * 32 + k] = __fsub_rn(v[q * 32 + k], __uint_as_float(r32[k]));
        }
        tc_fence_before();
        mbar_arrive(d2_free);
        ++j;
      }
      ++i;
    };
    float g = 1.0f;
    if constexpr (MODE == 2) g = global_scale_from_amax(__uint_as_float(*p.amax_glob));
    float amax = 0.0f;
    for (int c = 0; c < nch; ++c) {
      z_chunk(c);
      if constexpr (MODE == 2) {
        if (valid) quantise_row(p, v, row, col0 + c * kChunk, g);
      } else {
#pragma unroll
        for (int k = 0; k < kChunk; ++k) amax = fmaxf(amax, fabsf(v[k]));
      }
    }
    if constexpr (MODE != 2) {
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      if (lane == 0) red[warp] = __uint_as_float(wmax);
      named_bar(1, kRows);
      const float cmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      if constexpr (MODE == 1) {
        if (t == 0) atomicMax(p.amax_glob, __float_as_uint(cmax));
      } else {
        if (t == 0) red[4] = cmax;
      }
    }
    if constexpr (MODE == 0) {
      // red[4] is published by the cluster barrier B.
      cluster_arrive();
      cluster_wait();
      cg::cluster_group cluster = cg::this_cluster();
      const int nranks = static_cast<int>(cluster.num_blocks());
      float A = 0.0f;
      for (int rk = 0; rk < nranks; ++rk) A = fmaxf(A, cluster.map_shared_rank(red, rk)[4]);
      g = global_scale_from_amax(A);
      if constexpr (R > 0) {
        if (part == 0 && valid) {
          const float* uf = reinterpret_cast<const float*>(smem + C::OFF_XT + 32768) + t * C::UP_STRIDE;
#pragma unroll
          for (int k = 0; k < R; ++k) u[k] = uf[k];
          write_branch<R>(p, u, row, g);
        }
      }
      if (part == 0 && t == 0 && blockIdx.y == 0) *p.g_out = g;
      for (int c = 0; c < nch; ++c) {
        z_chunk(c);
        if (valid) quantise_row(p, v, row, col0 + c * kChunk, g);
      }
    }
    if constexpr (MODE == 2) {
      if (part == 0 && t == 0 && blockIdx.y == 0) *p.g_out = g;
    }
    if constexpr (C::kC) {
      cluster_arrive();
      cluster_wait();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C::kMMA) {
    if (warp == 5) {
      __syncwarp();
      tmem_dealloc(tmem, C::TMEM_COLS);
    }
  }
}

template <int R, int MODE>
cudaError_t launch_one(const ProMaps& maps, const PrologueParams& p, int parts, cudaStream_t st) {
  using C = PCfg<R, MODE>;
  auto kern = prologue_kernel<R, MODE>;
  static const cudaError_t smem_attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (smem_attr != cudaSuccess) return smem_attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(parts, (p.rows + kRows - 1) / kRows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = 0;
  if (C::kC) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = parts;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

template <int MODE>
cudaError_t launch_mode(const ProMaps& maps, const PrologueParams& p, int r, int parts, cudaStream_t st) {
  switch (r) {
    case 0: return launch_one<0, MODE>(maps, p, parts, st);
    case 16: return launch_one<16, MODE>(maps, p, parts, st);
    case 32: return launch_one<32, MODE>(maps, p, parts, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_prologue(const ProMaps& maps, const PrologueParams& p, int r, PrologueMode mode, int parts,
                            cudaStream_t st) {
  switch (mode) {
    case PrologueMode::Fused: return launch_mode<0>(maps, p, r, parts, st);
    case PrologueMode::Stats: return launch_mode<1>(maps, p, r, parts, st);
    case PrologueMode::Quantise: return launch_mode<2>(maps, p, r, parts, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qwam
