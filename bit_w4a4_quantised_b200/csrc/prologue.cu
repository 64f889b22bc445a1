// Activation prologue and weight prepare kernels.
//
// Both sides of the deflated ASP layer ("FastWAM UR3 3-task — 4-bit
// quantisations", section "What ASP is, and what the deflated form means") run
// the same row pipeline:
//
//   T~ = (T * chan) H            per-channel scale, then block-FWHT in registers
//   c  = T~ V                    rank-r coordinates (bf16x3 split warp MMA)
//   Z  = T~ - c V^T              deflation, again bf16x3
//   amax(Z) -> g,  quantise(Z)   NVFP4 codes + tiled E4M3 scales
//   branch operand               bf16(c) (weights: W~V) or bf16(c / (g_x g_w))
//
// Work split: a CTA of 4 warps owns 64 rows x (chunks * 128) columns; warp w
// owns 16 rows.  The CTAs of one row group form a thread-block cluster along
// K; their partial c sums are exchanged through distributed shared memory in a
// fixed rank order (deterministic).  With <= 64 rows one cluster covers the
// whole tensor, so the per-tensor amax is a cluster reduction and the kernel
// finishes in one launch (Fused).  Otherwise a Stats launch writes c and
// atomically maxes amax, and a Quantise launch recomputes Z bit-identically
// (same code path, explicit round-to-nearest intrinsics, same fp32 c) and
// quantises it.
//
// The rank-r products use the legacy m16n8k16 warp MMA with a hi/lo bf16 split
// of both operands (three products per step): plain bf16 flips ~0.2 % of the
// FP4 codes against a float64 reference, the split keeps it below 0.01 %.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace cg = cooperative_groups;

namespace qwam {
namespace {

constexpr int kGroupRows = 64;
constexpr int kChunk = 128;
constexpr int kPad = 8;  // row stride = 8 (mod 32) floats: conflict-free float2 fragment reads

__device__ __forceinline__ uint32_t ldg_u32(const uint16_t* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}

// In-register fast Walsh-Hadamard transform over blocks of b columns; this lane
// holds 4 consecutive columns, partner lanes are reached with xor shuffles.
// Natural (Sylvester) order: (lo, hi) -> (lo + hi, lo - hi).
__device__ __forceinline__ void fwht_lane4(float (&v)[4], int b, int lane) {
  if (b >= 2) {
    const float a0 = __fadd_rn(v[0], v[1]), a1 = __fsub_rn(v[0], v[1]);
    const float a2 = __fadd_rn(v[2], v[3]), a3 = __fsub_rn(v[2], v[3]);
    v[0] = a0; v[1] = a1; v[2] = a2; v[3] = a3;
  }
  if (b >= 4) {
    const float a0 = __fadd_rn(v[0], v[2]), a2 = __fsub_rn(v[0], v[2]);
    const float a1 = __fadd_rn(v[1], v[3]), a3 = __fsub_rn(v[1], v[3]);
    v[0] = a0; v[1] = a1; v[2] = a2; v[3] = a3;
  }
  for (int h = 4; h < b; h <<= 1) {
    const int m = h >> 2;
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
    }
  }
}

// Rotate the warp's 16 rows of one 128-column chunk into shared memory.
// Rows past p.rows read as zero.  Returns this lane's max |T~|.
__device__ __forceinline__ float rotate_rows(const PrologueParams& p, int row0, int col, float* xt, int stride,
                                             int lane) {
  const float4 c = __ldg(reinterpret_cast<const float4*>(p.chan + col) + lane);
  const uint16_t* x = static_cast<const uint16_t*>(p.x);
  float amax = 0.0f;
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int row = row0 + i;
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (row < p.rows) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + static_cast<size_t>(row) * p.K + col) + lane);
      v[0] = __fmul_rn(__uint_as_float(raw.x << 16), c.x);
      v[1] = __fmul_rn(__uint_as_float(raw.x & 0xffff0000u), c.y);
      v[2] = __fmul_rn(__uint_as_float(raw.y << 16), c.z);
      v[3] = __fmul_rn(__uint_as_float(raw.y & 0xffff0000u), c.w);
    }
    fwht_lane4(v, p.b, lane);
    float4 o;
    o.x = __fmul_rn(v[0], p.hscale);
    o.y = __fmul_rn(v[1], p.hscale);
    o.z = __fmul_rn(v[2], p.hscale);
    o.w = __fmul_rn(v[3], p.hscale);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
    *reinterpret_cast<float4*>(xt + i * stride + 4 * lane) = o;
  }
  return amax;
}

__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
  uint16_t ah, al, bh, bl;
  split_bf16(a, ah, al);
  split_bf16(b, bh, bl);
  hi = pack2(ah, bh);
  lo = pack2(al, bl);
}

// c[16 x R] += T~[16 x 128] * V[col.., 0..R) for the warp's rows (C fragments).
template <int R>
__device__ __forceinline__ void project(const PrologueParams& p, const float* xt, int stride, int col, int lane,
                                        float (&u)[R / 8][4]) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll 2
  for (int ks = 0; ks < kChunk / 16; ++ks) {
    const float* r0 = xt + g * stride + ks * 16 + 2 * q;
    const float* r1 = r0 + 8 * stride;
    const float2 x00 = *reinterpret_cast<const float2*>(r0);
    const float2 x10 = *reinterpret_cast<const float2*>(r1);
    const float2 x01 = *reinterpret_cast<const float2*>(r0 + 8);
    const float2 x11 = *reinterpret_cast<const float2*>(r1 + 8);
    uint32_t ahi[4], alo[4];
    split_pair(x00.x, x00.y, ahi[0], alo[0]);
    split_pair(x10.x, x10.y, ahi[1], alo[1]);
    split_pair(x01.x, x01.y, ahi[2], alo[2]);
    split_pair(x11.x, x11.y, ahi[3], alo[3]);
    const int kc = col + ks * 16 + 2 * q;
#pragma unroll
    for (int nt = 0; nt < R / 8; ++nt) {
      const size_t off = static_cast<size_t>(nt * 8 + g) * p.K + kc;
      const uint32_t bh0 = ldg_u32(p.vt_hi + off), bh1 = ldg_u32(p.vt_hi + off + 8);
      const uint32_t bl0 = ldg_u32(p.vt_lo + off), bl1 = ldg_u32(p.vt_lo + off + 8);
      mma16816(u[nt], alo, bh0, bh1);
      mma16816(u[nt], ahi, bl0, bl1);
      mma16816(u[nt], ahi, bh0, bh1);
    }
  }
}

// Z = T~ - c V^T on one 128-column chunk, in place; returns the lane's max |Z|.
template <int R>
__device__ __forceinline__ float deflate(const PrologueParams& p, float* xt, int stride, int col, int lane,
                                         const float (&u)[R / 8][4]) {
  const int g = lane >> 2, q = lane & 3;
  uint32_t ahi[R / 16][4], alo[R / 16][4];
#pragma unroll
  for (int ks = 0; ks < R / 16; ++ks) {
    split_pair(u[2 * ks][0], u[2 * ks][1], ahi[ks][0], alo[ks][0]);
    split_pair(u[2 * ks][2], u[2 * ks][3], ahi[ks][1], alo[ks][1]);
    split_pair(u[2 * ks + 1][0], u[2 * ks + 1][1], ahi[ks][2], alo[ks][2]);
    split_pair(u[2 * ks + 1][2], u[2 * ks + 1][3], ahi[ks][3], alo[ks][3]);
  }
  float amax = 0.0f;
#pragma unroll 4
  for (int nt = 0; nt < kChunk / 8; ++nt) {
    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const size_t vrow = static_cast<size_t>(col + nt * 8 + g) * R;
#pragma unroll
    for (int ks = 0; ks < R / 16; ++ks) {
      const size_t off = vrow + ks * 16 + 2 * q;
      const uint32_t bh0 = ldg_u32(p.v_hi + off), bh1 = ldg_u32(p.v_hi + off + 8);
      const uint32_t bl0 = ldg_u32(p.v_lo + off), bl1 = ldg_u32(p.v_lo + off + 8);
      mma16816(d, alo[ks], bh0, bh1);
      mma16816(d, ahi[ks], bl0, bl1);
      mma16816(d, ahi[ks], bh0, bh1);
    }
    float* p0 = xt + g * stride + nt * 8 + 2 * q;
    float* p1 = p0 + 8 * stride;
    float2 x0 = *reinterpret_cast<float2*>(p0);
    float2 x1 = *reinterpret_cast<float2*>(p1);
    x0.x = __fsub_rn(x0.x, d[0]);
    x0.y = __fsub_rn(x0.y, d[1]);
    x1.x = __fsub_rn(x1.x, d[2]);
    x1.y = __fsub_rn(x1.y, d[3]);
    *reinterpret_cast<float2*>(p0) = x0;
    *reinterpret_cast<float2*>(p1) = x1;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(x0.x), fabsf(x0.y)), fmaxf(fabsf(x1.x), fabsf(x1.y))));
  }
  return amax;
}

// Quantise the warp's 16 rows of one chunk (Z in shared memory): lane l takes
// row l/2 and 64 columns (4 blocks); 32 code bytes and 4 scale bytes per lane.
__device__ __forceinline__ void quantise_rows(const PrologueParams& p, const float* xt, int stride, int row0,
                                              int col, float g, int lane) {
  const int i = lane >> 1, half = lane & 1;
  const int row = row0 + i;
  if (row >= p.rows) return;
  const float* src = xt + i * stride + half * 64;
  const int c0 = col + half * 64;
  uint32_t codes[8];
  uint32_t sf4 = 0;
#pragma unroll
  for (int bb = 0; bb < 4; ++bb) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 t = *reinterpret_cast<const float4*>(src + bb * 16 + 4 * j);
      v[4 * j] = t.x; v[4 * j + 1] = t.y; v[4 * j + 2] = t.z; v[4 * j + 3] = t.w;
    }
    uint32_t c2[2];
    const uint32_t S = quant_block16(v, g, c2);
    codes[2 * bb] = c2[0];
    codes[2 * bb + 1] = c2[1];
    sf4 |= S << (8 * bb);
    if (p.z_out) {
      float4* z = reinterpret_cast<float4*>(p.z_out + static_cast<size_t>(row) * p.K + c0 + bb * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j) z[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * (p.K / 2) + c0 / 2);
  dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
  *reinterpret_cast<uint32_t*>(p.sf + sf_offset(row, c0 / 16, p.K)) = sf4;
}

// Branch operand and optional fp32 export of c for the warp's rows.
template <int R>
__device__ __forceinline__ void write_branch(const PrologueParams& p, int row0, const float (&u)[R / 8][4], float g,
                                             int lane) {
  const int g4 = lane >> 2, q = lane & 3;
  const float gs = __fmul_rn(g, p.g_other);
#pragma unroll
  for (int nt = 0; nt < R / 8; ++nt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = row0 + g4 + 8 * h;
      if (row >= p.rows) continue;
      float a = u[nt][2 * h], b = u[nt][2 * h + 1];
      const size_t off = static_cast<size_t>(row) * R + nt * 8 + 2 * q;
      if (p.u_out) *reinterpret_cast<float2*>(p.u_out + off) = make_float2(a, b);
      if (p.branch_mode == 1) {
        a = __fdiv_rn(a, gs);
        b = __fdiv_rn(b, gs);
      }
      *reinterpret_cast<uint32_t*>(p.branch + off) = pack2(bf16_bits_rn(a), bf16_bits_rn(b));
    }
  }
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int R, int MODE>
__global__ void __launch_bounds__(128) prologue_kernel(const PrologueParams p) {
  extern __shared__ __align__(16) float smem[];
  constexpr int NT = (R > 0 ? R / 8 : 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g4 = lane >> 2, q = lane & 3;
  const int part = blockIdx.x;
  const int row0 = blockIdx.y * kGroupRows + warp * 16;
  const bool active = row0 < p.rows;
  const int ncols = p.chunks * kChunk;
  const int col_base = part * ncols;
  const int stride = (MODE == 0 ? ncols : kChunk) + kPad;
  float* xt_w = smem + warp * 16 * stride;
  float* upart = smem + kGroupRows * stride;
  float* red = upart + kGroupRows * (R > 0 ? R : 4);

  float u[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.0f;

  float g = 1.0f;
  if constexpr (MODE == 2) {
    g = global_scale_from_amax(__uint_as_float(*p.amax_glob));
    if constexpr (R > 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row0 + g4 + 8 * h;
          if (row < p.rows) {
            const float2 t = *reinterpret_cast<const float2*>(p.u_glob + static_cast<size_t>(row) * R + nt * 8 + 2 * q);
            u[nt][2 * h] = t.x;
            u[nt][2 * h + 1] = t.y;
          }
        }
    }
  }

  // Sweep 1 (Fused / Stats with r > 0): rotate and project every chunk, then
  // sum the partial coordinates across the cluster in rank order.
  if constexpr (MODE != 2 && R > 0) {
    if (active) {
      for (int c = 0; c < p.chunks; ++c) {
        float* xc = xt_w + (MODE == 0 ? c * kChunk : 0);
        rotate_rows(p, row0, col_base + c * kChunk, xc, stride, lane);
        __syncwarp();
        project<R>(p, xc, stride, col_base + c * kChunk, lane, u);
        __syncwarp();
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float* d0 = upart + (warp * 16 + g4) * R + nt * 8 + 2 * q;
      *reinterpret_cast<float2*>(d0) = make_float2(u[nt][0], u[nt][1]);
      *reinterpret_cast<float2*>(d0 + 8 * R) = make_float2(u[nt][2], u[nt][3]);
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nranks = static_cast<int>(cluster.num_blocks());
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.0f;
    for (int rk = 0; rk < nranks; ++rk) {
      const float* rp = cluster.map_shared_rank(upart, rk);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float* s0 = rp + (warp * 16 + g4) * R + nt * 8 + 2 * q;
        const float2 a = *reinterpret_cast<const float2*>(s0);
        const float2 b = *reinterpret_cast<const float2*>(s0 + 8 * R);
        u[nt][0] = __fadd_rn(u[nt][0], a.x);
        u[nt][1] = __fadd_rn(u[nt][1], a.y);
        u[nt][2] = __fadd_rn(u[nt][2], b.x);
        u[nt][3] = __fadd_rn(u[nt][3], b.y);
      }
    }
    if constexpr (MODE == 1) cluster_arrive();  // remote reads of upart are done
  }

  // Sweep 2: deflate (recomputing T~ unless it is still resident), track amax,
  // and in the Quantise launch quantise each chunk straight away.
  float amax = 0.0f;
  if (active) {
    for (int c = 0; c < p.chunks; ++c) {
      float* xc = xt_w + (MODE == 0 ? c * kChunk : 0);
      const int col = col_base + c * kChunk;
      float m;
      if (MODE == 0 && R > 0) {
        m = 0.0f;
      } else {
        m = rotate_rows(p, row0, col, xc, stride, lane);
        __syncwarp();
      }
      if constexpr (R > 0) m = deflate<R>(p, xc, stride, col, lane, u);
      amax = fmaxf(amax, m);
      __syncwarp();
      if constexpr (MODE == 2) {
        quantise_rows(p, xc, stride, row0, col, g, lane);
        __syncwarp();
      }
    }
  }

  if constexpr (MODE == 2) {
    if constexpr (R > 0)
      if (part == 0) write_branch<R>(p, row0, u, g, lane);
    if (part == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.g_out = g;
    return;
  } else {
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (lane == 0) red[warp] = __uint_as_float(wmax);
    __syncthreads();
    if constexpr (MODE == 1) {
      if (threadIdx.x == 0) {
        const float cmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        atomicMax(p.amax_glob, __float_as_uint(cmax));
      }
      if constexpr (R > 0) {
        if (part == 0 && active) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = row0 + g4 + 8 * h;
              if (row < p.rows)
                *reinterpret_cast<float2*>(p.u_glob + static_cast<size_t>(row) * R + nt * 8 + 2 * q) =
                    make_float2(u[nt][2 * h], u[nt][2 * h + 1]);
            }
        }
        cluster_wait();  // no CTA leaves while a peer may still read its upart
      }
    } else {
      // Fused: the cluster holds every row, so its amax is the tensor amax.
      cg::cluster_group cluster = cg::this_cluster();
      if (threadIdx.x == 0) red[4] = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      cluster.sync();
      float A = 0.0f;
      const int nranks = static_cast<int>(cluster.num_blocks());
      for (int rk = 0; rk < nranks; ++rk) A = fmaxf(A, cluster.map_shared_rank(red, rk)[4]);
      cluster_arrive();
      g = global_scale_from_amax(A);
      if (active) {
        for (int c = 0; c < p.chunks; ++c) quantise_rows(p, xt_w + c * kChunk, stride, row0, col_base + c * kChunk, g, lane);
        if constexpr (R > 0)
          if (part == 0) write_branch<R>(p, row0, u, g, lane);
      }
      if (part == 0 && threadIdx.x == 0) *p.g_out = g;
      cluster_wait();
    }
  }
}

// --- standalone quantiser (tests and tools) -------------------------------
__global__ void amax_kernel(const float* __restrict__ T, size_t n, uint32_t* amax) {
  float m = 0.0f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, fabsf(T[i]));
  const uint32_t w = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) atomicMax(amax, w);
}

__global__ void quantize_blocks_kernel(const float* __restrict__ T, int rows, int K, uint8_t* codes, uint8_t* sf,
                                       const uint32_t* amax, float* g_out) {
  const size_t nblk = static_cast<size_t>(rows) * (K / 16);
  const float g = global_scale_from_amax(__uint_as_float(*amax));
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  for (size_t bi = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; bi < nblk;
       bi += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(bi / (K / 16));
    const int kb = static_cast<int>(bi % (K / 16));
    float v[16];
    const float4* src = reinterpret_cast<const float4*>(T + static_cast<size_t>(row) * K + kb * 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 t = src[j];
      v[4 * j] = t.x; v[4 * j + 1] = t.y; v[4 * j + 2] = t.z; v[4 * j + 3] = t.w;
    }
    uint32_t c2[2];
    const uint32_t S = quant_block16(v, g, c2);
    *reinterpret_cast<uint2*>(codes + static_cast<size_t>(row) * (K / 2) + kb * 8) = make_uint2(c2[0], c2[1]);
    sf[sf_offset(row, kb, K)] = static_cast<uint8_t>(S);
  }
}

// --- prepare helpers -------------------------------------------------------
__global__ void recip_kernel(const float* __restrict__ s, float* __restrict__ inv_s, int K, uint32_t* err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K) return;
  const float v = s[i];
  if (!(v > 0.0f) || !isfinite(v)) atomicOr(err, 1u);
  inv_s[i] = __frcp_rn(v);
}

__global__ void split_v_kernel(const float* __restrict__ V, int K, int r, uint16_t* v_hi, uint16_t* v_lo,
                               uint16_t* vt_hi, uint16_t* vt_lo) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K * r) return;
  const int k = i / r, j = i % r;
  uint16_t hi, lo;
  split_bf16(V[i], hi, lo);
  v_hi[i] = hi;
  v_lo[i] = lo;
  vt_hi[static_cast<size_t>(j) * K + k] = hi;
  vt_lo[static_cast<size_t>(j) * K + k] = lo;
}

template <int R, int MODE>
cudaError_t launch_one(const PrologueParams& p, int cluster, cudaStream_t st) {
  const int groups = (p.rows + kGroupRows - 1) / kGroupRows;
  const int parts = p.K / kChunk / p.chunks;
  const size_t smem = prologue_smem_bytes(R, static_cast<PrologueMode>(MODE), p.chunks);
  auto kern = prologue_kernel<R, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(parts, groups, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int nattr = 0;
  if (MODE != 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    nattr = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int MODE>
cudaError_t launch_mode(const PrologueParams& p, int r, int cluster, cudaStream_t st) {
  switch (r) {
    case 0: return launch_one<0, MODE>(p, cluster, st);
    case 16: return launch_one<16, MODE>(p, cluster, st);
    case 32: return launch_one<32, MODE>(p, cluster, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t prologue_smem_bytes(int r, PrologueMode mode, int chunks) {
  const int ncols = (mode == PrologueMode::Fused ? chunks * kChunk : kChunk);
  return static_cast<size_t>(kGroupRows) * (ncols + kPad) * 4 + static_cast<size_t>(kGroupRows) * (r > 0 ? r : 4) * 4 +
         64;
}

cudaError_t launch_prologue(const PrologueParams& p, int r, PrologueMode mode, int cluster, cudaStream_t st) {
  switch (mode) {
    case PrologueMode::Fused: return launch_mode<0>(p, r, cluster, st);
    case PrologueMode::Stats: return launch_mode<1>(p, r, cluster, st);
    case PrologueMode::Quantise: return launch_mode<2>(p, r, cluster, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_recip(const float* s, float* inv_s, int K, uint32_t* err, cudaStream_t st) {
  recip_kernel<<<(K + 255) / 256, 256, 0, st>>>(s, inv_s, K, err);
  return cudaGetLastError();
}

cudaError_t launch_split_v(const float* V, int K, int r, uint16_t* v_hi, uint16_t* v_lo, uint16_t* vt_hi,
                           uint16_t* vt_lo, cudaStream_t st) {
  const int n = K * r;
  split_v_kernel<<<(n + 255) / 256, 256, 0, st>>>(V, K, r, v_hi, v_lo, vt_hi, vt_lo);
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp32(const float* T, int rows, int K, uint8_t* codes, uint8_t* sf, float* g_out,
                                 uint32_t* amax_scratch, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax_scratch, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const size_t n = static_cast<size_t>(rows) * K;
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 148 * 8));
  amax_kernel<<<blocks, 256, 0, st>>>(T, n, amax_scratch);
  const size_t nblk = static_cast<size_t>(rows) * (K / 16);
  const int qblocks = static_cast<int>(std::min<size_t>((nblk + 255) / 256, 148 * 8));
  quantize_blocks_kernel<<<qblocks, 256, 0, st>>>(T, rows, K, codes, sf, amax_scratch, g_out);
  return cudaGetLastError();
}

}  // namespace qwam
