// Kernels outside the per-call hot path: the standalone NVFP4 quantiser (used by
// tests and tools on arbitrary fp32 tensors) and the prepare-time helpers that
// derive 1/s, the bf16 hi/lo split of V and the projection matrix
// P = diag(chan) H V stored in a layer handle.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace qwam {
namespace {

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
    const uint32_t S = quant_block16(v, g, rcp_rn(g), c2);
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

// Row-pipeline channel vector: per 128-column chunk, [chan * hscale | -(chan * hscale)]
// (fp32 products, round to nearest), so the rotation reads a signed, scaled
// factor instead of multiplying by hscale and selecting a sign per element.
__global__ void chan_pm_kernel(const float* __restrict__ chan, float hscale, int K, float* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K) return;
  const float v = __fmul_rn(chan[i], hscale);
  const int chunk = i >> 7, j = i & 127;
  out[chunk * 256 + j] = v;
  out[chunk * 256 + 128 + j] = -v;
}

__global__ void split_v_kernel(const float* __restrict__ V, int K, int r, uint16_t* v_hi, uint16_t* v_lo) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K * r) return;
  uint16_t hi, lo;
  split_bf16(V[i], hi, lo);
  v_hi[i] = hi;
  v_lo[i] = lo;
}

// x~ V = ((x * chan) H) V = x (diag(chan) H V): the rank-r coordinates come
// straight from T with P = diag(chan) H V.  One CTA = 128 consecutive k of one
// column j: Sylvester FWHT of V[:, j] inside each b-block (butterflies
// (lo + hi, lo - hi)), times 1/sqrt(b), times chan[k], split to bf16 hi/lo and
// stored transposed ([r, K], K contiguous: the K-major B operand of the MMA).
__global__ void make_proj_kernel(const float* __restrict__ V, const float* __restrict__ chan, int K, int r, int b,
                                 float hscale, uint16_t* p_hi, uint16_t* p_lo) {
  __shared__ float buf[128];
  const int t = threadIdx.x, j = blockIdx.y;
  const int k = blockIdx.x * 128 + t;
  buf[t] = V[static_cast<size_t>(k) * r + j];
  __syncthreads();
  for (int h = 1; h < b; h <<= 1) {
    const float a = buf[t], c = buf[t ^ h];
    __syncthreads();
    buf[t] = (t & h) ? __fsub_rn(c, a) : __fadd_rn(a, c);
    __syncthreads();
  }
  const float v = __fmul_rn(__fmul_rn(buf[t], hscale), chan[k]);
  uint16_t hi, lo;
  split_bf16(v, hi, lo);
  p_hi[static_cast<size_t>(j) * K + k] = hi;
  p_lo[static_cast<size_t>(j) * K + k] = lo;
}

// Shared-weight arm: the branch weight from the stored FP4 weight,
// L[n, j] = bf16(g * sum_k e2m1(code[n, k]) e4m3(S[n, k / 16]) V[k, j]), fp32
// accumulation in k order (each e2m1 * e4m3 product is exact in fp32).  A CTA
// takes 8 rows; lane j of a row's warp owns column j (r <= 32).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const float v = mag[c & 7u];
  return (c & 8u) ? -v : v;
}

__global__ void dequant_project_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                       const float* __restrict__ g, const float* __restrict__ V, int N, int K, int r,
                                       uint16_t* __restrict__ L) {
  const int j = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (n >= N || j >= r) return;
  const uint8_t* row = codes + static_cast<size_t>(n) * (K / 2);
  float acc = 0.0f;
  for (int kb = 0; kb < K / 16; ++kb) {
    const float sc = e4m3_value(sf[sf_offset(n, kb, K)]);
    for (int t = 0; t < 8; ++t) {
      const uint32_t byte = row[kb * 8 + t];
      const int k = kb * 16 + 2 * t;
      acc = __fmaf_rn(__fmul_rn(e2m1_value(byte & 15u), sc), V[static_cast<size_t>(k) * r + j], acc);
      acc = __fmaf_rn(__fmul_rn(e2m1_value(byte >> 4), sc), V[static_cast<size_t>(k + 1) * r + j], acc);
    }
  }
  L[static_cast<size_t>(n) * r + j] = bf16_bits_rn(__fmul_rn(acc, *g));
}

}  // namespace

cudaError_t launch_dequant_project(const uint8_t* codes, const uint8_t* sf, const float* g, const float* V, int N,
                                   int K, int r, uint16_t* L, cudaStream_t st) {
  if (r < 1 || r > 32) return cudaErrorInvalidValue;
  dequant_project_kernel<<<(N + 7) / 8, 256, 0, st>>>(codes, sf, g, V, N, K, r, L);
  return cudaGetLastError();
}

cudaError_t launch_recip(const float* s, float* inv_s, int K, uint32_t* err, cudaStream_t st) {
  recip_kernel<<<(K + 255) / 256, 256, 0, st>>>(s, inv_s, K, err);
  return cudaGetLastError();
}

// Self-check of the quantiser's FMA-based arithmetic against the fp32 IEEE
// operations: rcp_rn(e) vs __frcp_rn(e) and div6_rn(a) vs __fdiv_rn(a, 6) for
// every positive finite fp32 input; the E4M3 code of u / g vs the code of
// __fdiv_rn(u, g) for every u >= 0 at four divisors spread over the exponent
// range and for n_pairs pseudo-random (u, g) pairs.  counts[0..2] += mismatches.
__global__ void rounding_check_kernel(unsigned long long* counts, unsigned long long n_pairs) {
  const unsigned long long stride = static_cast<unsigned long long>(gridDim.x) * blockDim.x;
  const unsigned long long tid = static_cast<unsigned long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  unsigned long long bad[3] = {0, 0, 0};
  for (unsigned long long i = tid + 1; i < 0x7f800000ull; i += stride) {
    const float a = __uint_as_float(static_cast<uint32_t>(i));
    bad[0] += __float_as_uint(div6_rn(a)) != __float_as_uint(__fdiv_rn(a, 6.0f));
    bad[1] += __float_as_uint(rcp_rn(a)) != __float_as_uint(__frcp_rn(a));
  }
  for (int k = 0; k < 4; ++k) {
    const uint32_t ge = k == 0 ? 27u : (k == 1 ? 97u : (k == 2 ? 157u : 227u));  // 2^-100, 2^-30, 2^30, 2^100
    const float g = __uint_as_float(ge << 23 | (0x2F1A5Bu * (k + 1) & 0x7FFFFFu));
    const float y = rcp_rn(g);
    for (unsigned long long i = tid; i < 0x7f800000ull; i += stride) {
      const float u = __uint_as_float(static_cast<uint32_t>(i));
      bad[2] += e4m3_of_quotient(u, g, y) != e4m3_rn_satfinite(__fdiv_rn(u, g));
    }
  }
  for (unsigned long long j = tid; j < n_pairs; j += stride) {
    // splitmix64 of the pair index: two significands and exponents
    unsigned long long z = j * 0x9E3779B97F4A7C15ull + 0x632BE59BD9B4E019ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const uint32_t ue = 1u + static_cast<uint32_t>((z >> 46) % 253u), ge = 1u + static_cast<uint32_t>((z >> 54) % 253u);
    const float u = __uint_as_float((ue << 23) | static_cast<uint32_t>(z & 0x7FFFFFu));
    const float g = __uint_as_float((ge << 23) | static_cast<uint32_t>((z >> 23) & 0x7FFFFFu));
    bad[2] += e4m3_of_quotient(u, g, rcp_rn(g)) != e4m3_rn_satfinite(__fdiv_rn(u, g));
  }
  for (int k = 0; k < 3; ++k)
    if (bad[k]) atomicAdd(&counts[k], bad[k]);
}

cudaError_t launch_rounding_check(unsigned long long* counts, unsigned long long n_pairs, cudaStream_t st) {
  rounding_check_kernel<<<148 * 8, 256, 0, st>>>(counts, n_pairs);
  return cudaGetLastError();
}

cudaError_t launch_chan_pm(const float* chan, float hscale, int K, float* out, cudaStream_t st) {
  if (K % 128) return cudaErrorInvalidValue;
  chan_pm_kernel<<<(K + 255) / 256, 256, 0, st>>>(chan, hscale, K, out);
  return cudaGetLastError();
}

cudaError_t launch_split_v(const float* V, int K, int r, uint16_t* v_hi, uint16_t* v_lo, cudaStream_t st) {
  const int n = K * r;
  split_v_kernel<<<(n + 255) / 256, 256, 0, st>>>(V, K, r, v_hi, v_lo);
  return cudaGetLastError();
}

cudaError_t launch_make_proj(const float* V, const float* chan, int K, int r, int b, uint16_t* p_hi, uint16_t* p_lo,
                             cudaStream_t st) {
  if (K % 128 || b < 1 || b > 128 || (b & (b - 1)) || r < 1) return cudaErrorInvalidValue;
  const float hscale = 1.0f / std::sqrt(static_cast<float>(b));
  make_proj_kernel<<<dim3(K / 128, r), 128, 0, st>>>(V, chan, K, r, b, hscale, p_hi, p_lo);
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
