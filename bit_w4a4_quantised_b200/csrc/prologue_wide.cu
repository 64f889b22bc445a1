// Activation prologue for rank r = 0 and more than 128 rows: the plain
// smoothed and rotated NVFP4 path of the layer ("FastWAM UR3 3-task — 4-bit
// quantisations", section "What ASP is, and what the deflated form means":
// x~ = (x / s) H, quantised to NVFP4; with no protected subspace the deflation
// is the identity).
//
// The per-channel scale folds into the rotation's other operand:
//
//   x~[m, n] = sum_k x[m, k] * B[n, k],   B[n, k] = chan[k] H_b[k, n] / sqrt(b)
//
// over each 128-column chunk (H is block-diagonal with blocks b <= 128, so a
// chunk's x~ needs only that chunk's x).  x is exact in bf16; B is split into
// bf16 hi and lo parts (B ~= B_hi + B_lo to ~2^-17 relative), so x~ = x B_hi +
// x B_lo is two chains of bf16 tensor-core products accumulated in fp32 TMEM,
// and no CUDA-core work is spent on the rotation.
//
// Grid: chunks x G CTAs.  CTA (c, g) owns chunk c and the 128-row tiles
// t = g, g + G, ...; it builds its B once in shared memory.  Per tile: one TMA
// load of the 128 x 128 bf16 x tile into a four-slot ring, 16 MMAs
// (128 x 128 x 16, hi then lo) into one of two TMEM buffers, and sixteen row
// warps (four per TMEM lane quarter, 32 columns each) read Z back:
//   Stats     max |Z| over the tile -> one atomicMax per warp on the amax word
//   Quantise  NVFP4 codes and tiled E4M3 scales with g from that amax
// Both launches issue the same MMA sequence on the same operands, so Z is
// bit-identical in both.  Every mbarrier wait is bounded; no multicast.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace qwam {
namespace {

constexpr int kTile = 128;
constexpr int kSlots = 4;
constexpr int kRowWarps = 16;
constexpr int kRowWarp0 = 4;                     // warps 0 producer, 1 MMA, 2-3 help build B
constexpr int kThreads = 32 * (kRowWarp0 + kRowWarps);
constexpr int kXBytes = kTile * kTile * 2;       // two 64-column boxes, 128B swizzle
constexpr int kOffB = 0;                         // B_hi, then B_lo: the x tile's layout, rows = n
constexpr int kOffX = kOffB + 2 * kXBytes;
constexpr int kOffBar = kOffX + kSlots * kXBytes;
constexpr int kSmem = kOffBar + 256 + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory budget");

template <int MODE>  // 1: Stats, 2: Quantise
__global__ void __launch_bounds__(kThreads, 1)
    wide_prologue_kernel(const __grid_constant__ CUtensorMap tmx, const PrologueParams p, int groups) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                 // [kSlots] x tile landed
  uint64_t* empty = bars + kSlots;       // [kSlots] MMAs done with the slot
  uint64_t* zfull = bars + 2 * kSlots;   // [2] Z of a tile in TMEM buffer d
  uint64_t* zfree = zfull + 2;           // [2] row warps read buffer d
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(zfree + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunks = p.K / kTile;
  const int c = blockIdx.x % chunks;
  const int g0 = blockIdx.x / chunks;
  const int tiles = (p.rows + kTile - 1) / kTile;
  const int col0 = c * kTile;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&zfull[i], 1);
      mbar_init(&zfree[i], kRowWarps);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // B = diag(chan / sqrt(b)) H_b of this chunk, split into bf16 hi / lo, in the
  // K-major 128B-swizzled layout of the x tile (row n, 16-byte chunk j of the
  // 64-column half kb).  p.chan holds chan / sqrt(b) (a layer constant, so this
  // runs before the wait on the previous kernel).
  {
    const float* ch = p.chan + static_cast<size_t>(c) * 2 * kTile;
    for (int idx = threadIdx.x; idx < 2 * kTile * 8; idx += kThreads) {
      const int kb = idx >> 10, n = (idx >> 3) & 127, j = idx & 7;
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float v[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int k = kb * 64 + 8 * j + e + h;
          const bool in_block = (n ^ k) < p.b;
          const bool neg = (__popc(n & k & (p.b - 1)) & 1) != 0;
          v[h] = in_block ? (neg ? -ch[k] : ch[k]) : 0.0f;
        }
        hw[e / 2] = bf16x2_rn(v[0], v[1]);
        lw[e / 2] = bf16x2_rn(__fsub_rn(v[0], __uint_as_float(hw[e / 2] << 16)),
                              __fsub_rn(v[1], __uint_as_float(hw[e / 2] & 0xffff0000u)));
      }
      const int off = kb * 16384 + n * 128 + ((j ^ (n & 7)) << 4);
      *reinterpret_cast<uint4*>(smem + kOffB + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(smem + kOffB + kXBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
  fence_proxy_async();  // B is read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Stats reads x, which the kernel before it may write: wait for it, then let
  // Quantise start (Quantise therefore sees final x without waiting itself).
  if constexpr (MODE == 1) griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) tma_prefetch_desc(&tmx);
    int i = 0, last = -1;
    bool ok = true;
    for (int t = g0; ok && t < tiles; t += groups, ++i) {
      const int slot = i % kSlots;
      int wok = 1;
      if (lane == 0) {
        wok = mbar_wait(&empty[slot], ((i / kSlots) & 1) ^ 1u, p.err, DEVERR_PRODUCER_WAIT) ? 1 : 0;
        if (wok) mbar_arrive_expect_tx(&full[slot], kXBytes);
      }
      wok = __shfl_sync(0xffffffffu, wok, 0);
      if (!wok) {
        ok = false;
        break;
      }
      if (lane < 2)
        tma_load_2d(smem + kOffX + slot * kXBytes + lane * 16384, &tmx, &full[slot], col0 + 64 * lane, t * kTile);
      last = i;
    }
    // every copy this warp started lands before the CTA exits
    if (lane == 0 && last >= 0)
      mbar_wait(&full[last % kSlots], (last / kSlots) & 1, p.err, DEVERR_DRAIN_WAIT);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTile, kTile);
      const uint32_t bs = smem_u32(smem + kOffB);
      int i = 0;
      for (int t = g0; t < tiles; t += groups, ++i) {
        const int slot = i % kSlots, d = i & 1;
        if (!mbar_wait(&full[slot], (i / kSlots) & 1, p.err, DEVERR_MMA_WAIT)) break;
        if (!mbar_wait(&zfree[d], ((i >> 1) & 1) ^ 1u, p.err, DEVERR_MMA_WAIT)) break;
        tc_fence_after();
        const uint32_t xs = smem_u32(smem + kOffX + slot * kXBytes);
#pragma unroll
        for (int part = 0; part < 2; ++part)  // B_hi, then B_lo
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t a = smem_desc(xs + kb * 16384 + k * 32, 16, 1024, 2);
              const uint64_t b = smem_desc(bs + part * kXBytes + kb * 16384 + k * 32, 16, 1024, 2);
              mma_bf16(tmem + 128u * d, a, b, idesc, (part | kb | k) ? 1u : 0u);
            }
        tc_commit(&zfull[d]);
        tc_commit(&empty[slot]);
      }
    }
    __syncwarp();
  } else if (warp >= kRowWarp0) {
    // ------------------------------------------------------------ row warps
    const int rw = warp - kRowWarp0;
    const int q = warp & 3;                 // TMEM lane quarter
    const int cq = rw >> 2;                 // 32-column quarter of the chunk
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    float g = 1.0f, y_g = 1.0f;
    if constexpr (MODE == 2) {
      griddep_wait();  // the amax of Stats, and the workspace's last reader
      g = scale_from_amax(__uint_as_float(*p.amax_glob), p.fmt);
      y_g = rcp_rn(g);
    }
    float amax = 0.0f;
    bool alive = true;
    int i = 0;
    for (int t = g0; t < tiles; t += groups, ++i) {
      const int d = i & 1;
      // after one wait has run out no later tile comes
      alive = alive && mbar_wait(&zfull[d], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
      tc_fence_after();
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + 128u * d + lane_base + 32u * cq, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&zfree[d]);
      const int row = t * kTile + q * 32 + lane;
      if (!alive || row >= p.rows) continue;
      if constexpr (MODE == 1) {
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(__uint_as_float(r[k])));
      } else {
        float z[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) z[k] = __uint_as_float(r[k]);
        if (p.fmt == FMT_FP8)
          quantise_store_fp8<32>(z, row, col0 + 32 * cq, p.K, y_g, p.codes, p.z_out);
        else
          quantise_store<32>(z, row, col0 + 32 * cq, p.K, g, y_g, p.codes, p.sf, p.z_out);
      }
    }
    if constexpr (MODE == 1) {
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      if (lane == 0) atomicMax(p.amax_glob, wmax);
    } else {
      if (blockIdx.x == 0 && rw == 0 && lane == 0) *p.g_out = g;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& x, const PrologueParams& p, int groups, cudaStream_t st) {
  auto kern = wide_prologue_kernel<MODE>;
  static const cudaError_t smem_attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (smem_attr != cudaSuccess) return smem_attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((p.K / kTile) * groups), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, p, groups);
}

}  // namespace

int wide_prologue_groups(int rows, int K, int sms) {
  const int chunks = K / kTile, tiles = (rows + kTile - 1) / kTile;
  int g = sms / chunks;
  if (g < 1) g = 1;
  if (g > tiles) g = tiles;
  return g;
}

cudaError_t launch_prologue_wide(const CUtensorMap& x, const PrologueParams& p, PrologueMode mode, int groups,
                                 cudaStream_t st) {
  if (p.K % kTile || p.rows < 1 || groups < 1 || p.b < 1 || p.b > kTile) return cudaErrorInvalidValue;
  switch (mode) {
    case PrologueMode::Stats: return launch_mode<1>(x, p, groups, st);
    case PrologueMode::Quantise: return launch_mode<2>(x, p, groups, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qwam
