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
constexpr int kOffStage = kOffBar + 256;           // 128 staged channel words for building B
constexpr int kSmem = kOffStage + 512 + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory budget");

// B = diag(chan / sqrt(b)) H_b of chunk c, split into bf16 hi / lo, in the
// K-major 128B-swizzled layout of the x tile (row n, 16-byte chunk j of the
// 64-column half kb): hi at dst, lo at dst + kXBytes.  p.chan holds chan /
// sqrt(b) (a layer constant, so this may run before the wait on the previous
// kernel).  The chunk's 128 values and their hi / lo parts are staged first
// (stage: 128 words, hi in bits 0..15, lo in 16..31); an entry of B is then
// one of them with both signs flipped (bf16 rounding is sign-symmetric, so
// -c splits into -hi, -lo) or zero.  Called by the nthreads builder threads
// (tid 0 .. nthreads - 1, whole warps, nthreads >= 128), which synchronise on
// named barrier kBuildBar.
constexpr int kBuildBar = 2;
constexpr int kBuildWarp0 = 2;  // warps 2 .. end build B; 0 (loads) and 1 (MMA) do not wait for it
constexpr int kBuilders = kThreads - 32 * kBuildWarp0;
__device__ __forceinline__ void build_rotation_operand(uint8_t* dst, uint32_t* stage, const PrologueParams& p, int c,
                                                       int tid, int nthreads) {
  if (tid < kTile) {
    const float v = p.chan[static_cast<size_t>(c) * 2 * kTile + tid];
    const uint32_t hi = bf16_bits_rn(v);
    const uint32_t lo = bf16_bits_rn(__fsub_rn(v, __uint_as_float(hi << 16)));
    stage[tid] = hi | (lo << 16);
  }
  named_bar(kBuildBar, nthreads);
  // An item is the 16-byte chunk of row n holding k = k0 .. k0 + 7 (k0 = 64 kb +
  // 8 j).  The Sylvester sign (-1)^popcount(n & k) over those k is the sign at
  // k0 times the parity pattern of (n & 7) & e, e = 0 .. 7 (bit e of kPar[n & 7]);
  // b-blocks of 8 or more columns hold all 8 entries or none.
  constexpr uint32_t kPar[8] = {0x00u, 0xAAu, 0xCCu, 0x66u, 0xF0u, 0x5Au, 0x3Cu, 0x96u};
  const uint32_t bmask = static_cast<uint32_t>(p.b - 1);
  for (int idx = tid; idx < 2 * kTile * 8; idx += nthreads) {
    const int kb = idx >> 10, n = (idx >> 3) & 127, j = idx & 7;
    const int k0 = kb * 64 + 8 * j;
    const uint32_t s0 = (__popc(static_cast<uint32_t>(n & k0) & bmask) & 1u) ? 0xFFu : 0u;
    const uint32_t negs = s0 ^ kPar[n & 7];
    const uint4 st0 = *reinterpret_cast<const uint4*>(stage + k0);
    const uint4 st1 = *reinterpret_cast<const uint4*>(stage + k0 + 4);
    const uint32_t sw[8] = {st0.x, st0.y, st0.z, st0.w, st1.x, st1.y, st1.z, st1.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = k0 + e + h;
        // within H's b-block of k?  (for b < 8 the block bits of e matter too)
        const bool in_block = ((static_cast<uint32_t>(n ^ k)) & ~bmask) == 0u;
        const uint32_t sgn = (p.b >= 8 ? (negs >> (e + h)) : (__popc(static_cast<uint32_t>(n & k) & bmask))) & 1u;
        w[h] = in_block ? (sw[e + h] ^ (sgn ? 0x80008000u : 0u)) : 0u;
      }
      hw[e / 2] = (w[0] & 0xffffu) | (w[1] << 16);
      lw[e / 2] = (w[0] >> 16) | (w[1] & 0xffff0000u);
    }
    const int off = kb * 16384 + n * 128 + ((j ^ (n & 7)) << 4);
    *reinterpret_cast<uint4*>(dst + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(dst + kXBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// The 16 MMAs of one 128 x 128 tile: x (bf16, at xs) times B_hi then B_lo
// (at bs) into the TMEM accumulator d.
__device__ __forceinline__ void rotate_tile_mma(uint32_t d, uint32_t xs, uint32_t bs) {
  const uint32_t idesc = idesc_bf16(kTile, kTile);
#pragma unroll
  for (int part = 0; part < 2; ++part)
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t a = smem_desc(xs + kb * 16384 + k * 32, 16, 1024, 2);
        const uint64_t b = smem_desc(bs + part * kXBytes + kb * 16384 + k * 32, 16, 1024, 2);
        mma_bf16(d, a, b, idesc, (part | kb | k) ? 1u : 0u);
      }
}

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
  uint64_t* b_ready = zfree + 2;         // the builder warps wrote B
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_ready + 1);

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
    mbar_init(b_ready, kBuilders / 32);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // B is built while the first x tiles are in flight; the MMA warp waits for it
  if (warp >= kBuildWarp0) {
    build_rotation_operand(smem + kOffB, reinterpret_cast<uint32_t*>(smem + kOffStage), p, c,
                           threadIdx.x - 32 * kBuildWarp0, kBuilders);
    fence_proxy_async();  // B is read by the tensor core
    __syncwarp();
    if (lane == 0) mbar_arrive(b_ready);
  }
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
      const uint32_t bs = smem_u32(smem + kOffB);
      int i = 0;
      const bool bok = mbar_wait(b_ready, 0, p.err, DEVERR_MMA_WAIT);
      for (int t = g0; bok && t < tiles; t += groups, ++i) {
        const int slot = i % kSlots, d = i & 1;
        if (!mbar_wait(&full[slot], (i / kSlots) & 1, p.err, DEVERR_MMA_WAIT)) break;
        if (!mbar_wait(&zfree[d], ((i >> 1) & 1) ^ 1u, p.err, DEVERR_MMA_WAIT)) break;
        tc_fence_after();
        rotate_tile_mma(tmem + 128u * d, smem_u32(smem + kOffX + slot * kXBytes), bs);
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

// ---------------------------------------------------------------------------
// One-pass form: one cooperative launch with a bounded grid-wide barrier for the
// amax, for CTAs that hold at most six row tiles of their chunk (4096 rows of
// K = 3072 on 144 CTAs, for instance).  x is read from memory once:
//   phase 1  tiles 0..2: x through a two-slot ring, Z kept in TMEM buffers
//            0..2; tiles 3..5: x kept in shared memory, Z formed in TMEM
//            buffer 3 one after another; max |Z| of every tile -> atomicMax
//   barrier  every CTA has published its maximum (a counter in the workspace
//            header, cleared before the launch; bounded wait)
//   phase 2  tiles 0..2 quantised from TMEM; tiles 3..5 formed again from the
//            kept x (into buffers 3, 0, 1 as they free up) and quantised
// A tile's MMA sequence is the same in both phases, so Z is bit-identical.
constexpr int kOnePassMaxTiles = 6;
constexpr int kOffRing = kOffB + 2 * kXBytes;     // ring slots 0, 1 (tiles 0, 1, then 2)
constexpr int kOffKeep = kOffRing + 2 * kXBytes;  // x of tiles 3, 4, 5, kept for phase 2
constexpr int kOffBar1 = kOffKeep + 3 * kXBytes;
constexpr int kOffStage1 = kOffBar1 + 256;
constexpr int kSmem1 = kOffStage1 + 512 + 1024;
static_assert(kSmem1 <= 227 * 1024, "shared memory budget");
constexpr int kBarCountOffset = 12;               // bytes after the amax word

__device__ __forceinline__ int onepass_buf1(int i) { return i < 3 ? i : 3; }
__device__ __forceinline__ int onepass_buf2(int i) { return i < 3 ? i : (i == 3 ? 3 : i - 4); }
__device__ __forceinline__ int onepass_xslot(int i) {
  return i < 2 ? kOffRing + i * kXBytes : (i == 2 ? kOffRing : kOffKeep + (i - 3) * kXBytes);
}
// phase-1 order: tile 2 reuses ring slot 0, so it comes last
__device__ __forceinline__ int onepass_order(int k) { return k < 2 ? k : (k < 5 ? k + 1 : 2); }

__global__ void __launch_bounds__(kThreads, 1)
    onepass_prologue_kernel(const __grid_constant__ CUtensorMap tmx, const PrologueParams p, int groups) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar1);
  uint64_t* full = bars;                 // [6] x of tile i landed
  uint64_t* ring_free = bars + 6;        // MMAs of tile 0 done with ring slot 0
  uint64_t* zfull = bars + 7;            // [4] Z of a tile in TMEM buffer d
  uint64_t* zfree = bars + 11;           // [4] row warps done with buffer d
  uint64_t* b_ready = bars + 15;         // the builder warps wrote B
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  int* grid_ok = reinterpret_cast<int*>(bars + 17);
  uint32_t* bar_count = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.amax_glob) + kBarCountOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunks = p.K / kTile;
  const int c = blockIdx.x % chunks;
  const int g0 = blockIdx.x / chunks;
  const int tiles = (p.rows + kTile - 1) / kTile;
  const int col0 = c * kTile;
  int n = 0;  // row tiles of this CTA: g0, g0 + groups, ... (the host keeps n <= 6)
  for (int t = g0; t < tiles && n < kOnePassMaxTiles; t += groups) ++n;
  auto tile_row = [&](int i) { return (g0 + i * groups) * kTile; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kOnePassMaxTiles; ++i) mbar_init(&full[i], 1);
    mbar_init(ring_free, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&zfull[i], 1);
      mbar_init(&zfree[i], kRowWarps);
    }
    mbar_init(b_ready, kBuilders / 32);
    *grid_ok = 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // B is built while the first x tiles are in flight; the MMA warp waits for it
  if (warp >= kBuildWarp0) {
    build_rotation_operand(smem + kOffB, reinterpret_cast<uint32_t*>(smem + kOffStage1), p, c,
                           threadIdx.x - 32 * kBuildWarp0, kBuilders);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_ready);
  }
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) tma_prefetch_desc(&tmx);
    uint32_t issued = 0;
    for (int k = 0; k < kOnePassMaxTiles; ++k) {
      const int i = onepass_order(k);
      if (i >= n) continue;
      int ok = 1;
      if (lane == 0) {
        if (i == 2) ok = mbar_wait(ring_free, 0, p.err, DEVERR_PRODUCER_WAIT) ? 1 : 0;
        if (ok) mbar_arrive_expect_tx(&full[i], kXBytes);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane < 2) tma_load_2d(smem + onepass_xslot(i) + lane * 16384, &tmx, &full[i], col0 + 64 * lane, tile_row(i));
      issued |= 1u << i;
    }
    // every copy this warp started lands before the CTA exits
    if (lane == 0)
      for (int i = 0; i < kOnePassMaxTiles; ++i)
        if (issued >> i & 1u) mbar_wait(&full[i], 0, p.err, DEVERR_DRAIN_WAIT);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t bs = smem_u32(smem + kOffB);
      int n3 = 0;  // MMAs issued into buffer 3 so far
      bool ok = mbar_wait(b_ready, 0, p.err, DEVERR_MMA_WAIT);
      for (int k = 0; ok && k < kOnePassMaxTiles; ++k) {  // phase 1
        const int i = onepass_order(k);
        if (i >= n) continue;
        const int d = onepass_buf1(i);
        ok = mbar_wait(&full[i], 0, p.err, DEVERR_MMA_WAIT) &&
             (d != 3 || n3 == 0 || mbar_wait(&zfree[3], (n3 - 1) & 1, p.err, DEVERR_MMA_WAIT));
        if (!ok) break;
        tc_fence_after();
        rotate_tile_mma(tmem + 128u * d, smem_u32(smem + onepass_xslot(i)), bs);
        tc_commit(&zfull[d]);
        if (i == 0) tc_commit(ring_free);
        if (d == 3) ++n3;
      }
      for (int i = 3; ok && i < n; ++i) {  // phase 2: tiles 3.. from the kept x
        const int d = onepass_buf2(i);
        // buffer 3 once the rows read its last phase-1 tile; buffers 0 / 1 once
        // the rows quantised tiles 0 / 1
        ok = d == 3 ? mbar_wait(&zfree[3], (n3 - 1) & 1, p.err, DEVERR_MMA_WAIT)
                    : mbar_wait(&zfree[d], 0, p.err, DEVERR_MMA_WAIT);
        if (!ok) break;
        tc_fence_after();
        rotate_tile_mma(tmem + 128u * d, smem_u32(smem + onepass_xslot(i)), bs);
        tc_commit(&zfull[d]);
        if (d == 3) ++n3;
      }
    }
    __syncwarp();
  } else if (warp >= kRowWarp0) {
    // ------------------------------------------------------------ row warps
    const int rw = warp - kRowWarp0;
    const int q = warp & 3;
    const int cq = rw >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int nfull[4] = {0, 0, 0, 0};  // completions of zfull[d] seen
    bool alive = true;
    float amax = 0.0f;
    uint32_t r[32];
    auto take = [&](int d) {  // Z of buffer d, this warp's 32 columns
      __syncwarp();
      tc_fence_after();
      tmem_ld_32x32b_x32(tmem + 128u * d + lane_base + 32u * cq, r);
      tmem_ld_wait();
    };
    auto release = [&](int d) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&zfree[d]);
    };
    for (int k = 0; k < kOnePassMaxTiles; ++k) {  // phase 1: the maximum
      const int i = onepass_order(k);
      if (i >= n) continue;
      const int d = onepass_buf1(i);
      alive = alive && mbar_wait(&zfull[d], nfull[d] & 1, p.err, DEVERR_EPILOGUE_WAIT);
      ++nfull[d];
      take(d);
      if (d == 3) release(3);
      const int row = tile_row(i) + q * 32 + lane;
      if (alive && row < p.rows) {
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(__uint_as_float(r[e])));
      }
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0) atomicMax(p.amax_glob, wmax);
    __syncwarp();
    named_bar(1, 32 * kRowWarps);  // every row warp of this CTA published
    if (rw == 0 && lane == 0) {
      // the CTA's maxima (ordered before this by the named barrier) are made
      // visible device-wide by a full fence before the arrival; then poll with
      // acquire order until every CTA has arrived
      __threadfence();
      atomicAdd(bar_count, 1u);
      const uint64_t t0 = global_timer_ns();
      for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar_count) : "memory");
        if (v >= gridDim.x) break;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicOr(p.err, DEVERR_GRID_WAIT);
          *grid_ok = 0;
          break;
        }
      }
    }
    __syncwarp();  // the named barrier is warp-aligned: lane 0 rejoins first
    named_bar(1, 32 * kRowWarps);
    alive = alive && *reinterpret_cast<volatile int*>(grid_ok) != 0;
    const float g = scale_from_amax(__uint_as_float(*reinterpret_cast<volatile uint32_t*>(p.amax_glob)), p.fmt);
    const float y_g = rcp_rn(g);
    for (int i = 0; i < n; ++i) {  // phase 2: quantise
      const int d = onepass_buf2(i);
      if (i >= 3) {
        alive = alive && mbar_wait(&zfull[d], nfull[d] & 1, p.err, DEVERR_EPILOGUE_WAIT);
        ++nfull[d];
      }
      take(d);
      if (i < 2 && i + 4 < n) release(d);  // buffer i takes tile i + 4
      const int row = tile_row(i) + q * 32 + lane;
      if (!alive || row >= p.rows) continue;
      float z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = __uint_as_float(r[e]);
      if (p.fmt == FMT_FP8)
        quantise_store_fp8<32>(z, row, col0 + 32 * cq, p.K, y_g, p.codes, p.z_out);
      else
        quantise_store<32>(z, row, col0 + 32 * cq, p.K, g, y_g, p.codes, p.sf, p.z_out);
    }
    if (blockIdx.x == 0 && rw == 0 && lane == 0) *p.g_out = g;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
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

bool onepass_prologue_fits(int rows, int K, int groups, int sms) {
  const int chunks = K / kTile, tiles = (rows + kTile - 1) / kTile;
  return (tiles + groups - 1) / groups <= kOnePassMaxTiles && chunks * groups <= sms;
}

cudaError_t launch_prologue_onepass(const CUtensorMap& x, const PrologueParams& p, int groups, cudaStream_t st) {
  if (p.K % kTile || p.rows < 1 || groups < 1 || p.b < 1 || p.b > kTile) return cudaErrorInvalidValue;
  auto kern = onepass_prologue_kernel;
  static const cudaError_t smem_attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem1);
  if (smem_attr != cudaSuccess) return smem_attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((p.K / kTile) * groups), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem1;
  cfg.stream = st;
  // every CTA of the grid is resident at once (their grid-wide barrier
  // depends on it); the launch fails rather than runs when they do not fit
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, p, groups);
}

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
