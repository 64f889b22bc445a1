// Activation prologue and weight prepare: one row pipeline for both sides of
// the deflated ASP layer ("FastWAM UR3 3-task — 4-bit quantisations", section
// "What ASP is, and what the deflated form means"):
//
//   c  = T P,  P = diag(chan) H V    rank-r coordinates, tcgen05 bf16 MMA on the
//                                    TMA tile of T itself (T is exact bf16; P is
//                                    a bf16 hi/lo pair, two MMAs per K step)
//   T~ = (T * chan) H                per-channel scale and block FWHT in registers
//   Z  = T~ - c V^T                  deflation: c V^T by tcgen05 MMA into TMEM
//                                    (hi/lo split of both operands, three MMAs)
//   amax(Z) -> g, quantise(Z)        NVFP4 codes + 128x4-tiled E4M3 scales
//   branch operand                   bf16(c) (weight side: W~V) or
//                                    bf16(c / (g_x g_w)) (activation side)
//
// T = x and chan = 1/s on the activation side, T = W and chan = s on the weight
// side.  x~ V = ((x * chan) H) V = x (diag(chan) H V), so the projection needs
// no arithmetic on the CUDA cores: it is a pure TMA -> MMA stream.
//
// CTA = 128 rows (one TMEM lane per row) x `chunks` 128-column chunks, 11 warps:
//   warps 0-7   row threads.  Normal layout: warp w serves TMEM lane quarter
//               w % 4 and column half w / 4 of each chunk (one thread = one row x
//               64 columns).  Small layout (tile rows <= 32, Fused only): c is
//               replicated into all four lane quarters and warp q < 4 serves
//               columns [32q, 32q + 32) of rows 0..31, so the four schedulers
//               share the row arithmetic.  The FWHT stages whose butterflies
//               cross the thread's column range read the partner columns from the
//               shared-memory tile of T; the rest run in registers.
//   warps 8, 9  TMA producers, one per ring slot (a TMA instruction holds its
//               warp for a fixed ~600 cycles whatever its size).
//   warp 10     TMEM owner and MMA issuer.
// The CTAs of a row tile form a cluster along K: partial c is summed across it
// through distributed shared memory in rank order (deterministic).
//
// Modes: Fused (rows <= 128: the cluster holds the whole tensor, so amax is a
// cluster reduction and one launch finishes the job; with one chunk per CTA Z
// stays in registers across that reduction, otherwise a second sweep recomputes
// it bit-identically), Stats (c to global, atomic amax) and Quantise (reads c
// and amax, recomputes Z bit-identically from the same code and data,
// quantises).  Every wait on an mbarrier is bounded.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"
#include "quant.cuh"

namespace qwam {
namespace {

constexpr int kRows = 128;
constexpr int kChunk = 128;
constexpr int kRowWarps = 8;
constexpr int kRowThreads = 32 * kRowWarps;
constexpr int kMaxParts = 16;  // 16: a non-portable cluster size (one 128-row tile only)

// What one ring load brings in.
enum : uint32_t { LD_X = 1u, LD_P = 2u, LD_V = 4u, LD_CH = 8u };

// W = columns of a chunk per row thread: 64 (normal) or 32 (small layout).
template <int R, int MODE, int W>
struct PCfg {
  // Stats / Quantise: the rotation runs on the tensor core, Z = (A_hi + A_lo) H -
  // c V^T into TMEM, with A = T * chan * hscale split into bf16 hi/lo by the rows
  static constexpr bool kTC = MODE == 1 || MODE == 2;
  static constexpr bool kMMA = R > 0 || kTC;
  static constexpr bool kProj = R > 0 && MODE != 2;   // this launch computes c
  static constexpr bool kNeedA = kProj;               // cluster exchange of partial c
  static constexpr bool kNeedB = MODE == 0;           // cluster exchange of amax
  static constexpr bool kCluster = kNeedA || kNeedB;  // a cluster launch (peers store into this smem)
  static constexpr bool kSmall = W == 32;
  // Warp roles.  Fused: rows 0-7, producers 8-9, MMA 10.  TC: split warps 0-7
  // (A_hi / A_lo of each chunk), rows 8-15 (exchange, Z from TMEM, amax or the
  // quantiser), producers 16-17, MMA 18, 19 spare (warpgroups of four for the
  // register split below).
  static constexpr int SPLIT_WARPS = kTC ? 8 : 0;
  static constexpr int ROW0 = SPLIT_WARPS;
  static constexpr int PROD0 = ROW0 + kRowWarps;  // one producer per ring slot
  static constexpr int MMA_WARP = PROD0 + 2;
  static constexpr int THREADS = 32 * (kTC ? 20 : 11);
  // TC register split (launch: 640 threads x 96): split warps 56, rows 152,
  // producers / MMA / spare 64; 256 x 56 + 256 x 152 + 128 x 64 = 640 x 96.
  static constexpr int REG_SPLIT = 56, REG_ROWS = 152, REG_OTHER = 64;
  static constexpr int UC = R > 0 ? R / 2 : 1;        // c columns per row thread (two per row)
  static constexpr int X_BYTES = kRows * kChunk * 2;  // two 64-column SW128 boxes (TC: then A_hi)
  static constexpr int ALO_BYTES = kTC ? X_BYTES : 0; // TC: A_lo, same layout as the x tile
  static constexpr int P_BYTES = 512 * R;             // P^T: [kb][hi, lo] boxes of R rows x 128 B
  static constexpr int V_BYTES = 512 * R;             // V hi/lo: 2 boxes of 128 rows x 2R B
  static constexpr int CH_BYTES = kChunk * 8;         // chan * hscale and its negation
  static constexpr int OFF_ALO = X_BYTES;
  static constexpr int OFF_P = X_BYTES + ALO_BYTES;
  static constexpr int OFF_V = kTC ? OFF_P : OFF_P + P_BYTES;  // TC: a load carries P or V, never both
  static constexpr int OFF_CH = OFF_V + V_BYTES;
  static constexpr int SLOT = (OFF_CH + CH_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_H = 2 * SLOT;              // TC: H_b blocks of one chunk, bf16 [128][128]
  static constexpr int H_BYTES = kTC ? kRows * kChunk * 2 : 0;
  static constexpr int OFF_UA = OFF_H + H_BYTES;      // c hi/lo (TC: -c): A operand of the deflation
  static constexpr int UA_BYTES = 512 * R;
  // Cluster sum of c, reduce-scatter then all-gather, both pushed with remote
  // stores: RS[rank][row in slice][R] receives the partials of this CTA's row
  // slice from every rank; UG[row][R + 4] receives the summed rows.
  // TC: RS and UG live in the two A_lo areas, which the rows write only after the
  // exchange (and which no TMA load touches)
  static constexpr int RS_BYTES = kProj ? kRows * R * 4 : 0;
  static constexpr int UG_STRIDE = R + 4;
  static constexpr int UG_BYTES = kProj ? kRows * UG_STRIDE * 4 : 0;
  static constexpr int OFF_RS = kTC ? OFF_ALO : OFF_UA + UA_BYTES;
  static constexpr int OFF_UG = kTC ? SLOT + OFF_ALO : OFF_RS + RS_BYTES;
  static constexpr int OFF_BAR = kTC ? OFF_UA + UA_BYTES : OFF_UG + UG_BYTES;
  static constexpr int OFF_RED = OFF_BAR + 128;       // warp maxima [0, 8), CTA maxima by rank [8, 8 + kMaxParts)
  static constexpr int SMEM = OFF_RED + 128 + 1024;
  // TMEM: D2 [0, 128) (TC: two Z accumulators [0, 256)), then T P^T hi | lo (2R columns)
  static constexpr uint32_t U_COL = kTC ? 256 : 128;
  static constexpr uint32_t TMEM_COLS = (kTC && R > 0) ? 512 : 256;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(!kTC || (RS_BYTES <= ALO_BYTES && UG_BYTES <= ALO_BYTES), "exchange areas fit in A_lo");
  static_assert(!kSmall || MODE == 0, "the small layout is a Fused-only form");
};

__device__ __forceinline__ void unpack8(uint4 w, float* o) {
  o[0] = __uint_as_float(w.x << 16); o[1] = __uint_as_float(w.x & 0xffff0000u);
  o[2] = __uint_as_float(w.y << 16); o[3] = __uint_as_float(w.y & 0xffff0000u);
  o[4] = __uint_as_float(w.z << 16); o[5] = __uint_as_float(w.z & 0xffff0000u);
  o[6] = __uint_as_float(w.w << 16); o[7] = __uint_as_float(w.w & 0xffff0000u);
}

// Row t of a K-major bf16 operand tile with W-byte rows (one swizzle atom wide):
// write 8 consecutive elements (16 bytes) as logical chunk j.
__device__ __forceinline__ void put16(uint8_t* tile, int t, int j, int Wb, uint4 w) {
  *reinterpret_cast<uint4*>(tile + t * Wb + (swz_chunk(t, j, Wb) << 4)) = w;
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

// This thread's W columns [W*s0, W*s0 + W) of tile row `row` of one chunk:
//   out = ((T * chan) H_b) restricted to those columns, times 1/sqrt(b).
// chan (shared memory) holds this chunk's chan * hscale in [0, 128) and its
// negation in [128, 256).  The Hadamard bits above log2(W) combine the chunk's
// column ranges s that lie in the same b-block: each contributes T * (+-chan *
// hscale), the sign (-1)^popcount of the in-block bits of s & s0 (Sylvester
// order) chosen by reading the negated half; the thread's own range first, the
// others added with one packed FMA per pair.  The bits below log2(W) are
// butterflies (lo + hi, lo - hi) in registers.  Identical
// code and op order in every sweep, so recomputed Z is bit-identical.
template <int W>
__device__ __forceinline__ void rotate_cols(const uint8_t* xs, const float* chan, int row, int s0, int b,
                                            float (&v)[W]) {
  constexpr int NSEG = kChunk / W;
  float2* v2 = reinterpret_cast<float2*>(v);  // element pairs (2i, 2i + 1)
  // own range first (d = 0: v = T * c), then the others of the b-block (v += T * c)
#pragma unroll
  for (int d = 0; d < NSEG; ++d) {
    if (d * W >= b) continue;  // range s0 ^ d lies in another b-block
    const int s = s0 ^ d;
    const bool neg = (__popc(s & s0 & ((b - 1) / W)) & 1) != 0;  // in-block segment bits only
    const int col = s * W;                        // first column of range s
    const uint8_t* box = xs + (col >> 6) * 16384 + row * 128;
    const int c16 = (col & 63) >> 3;              // first 16-byte chunk inside the box row
    const float* cs = chan + (neg ? kChunk : 0) + col;
#pragma unroll
    for (int g = 0; g < W / 8; ++g) {
      const uint4 w = *reinterpret_cast<const uint4*>(box + (((c16 + g) ^ (row & 7)) << 4));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      const float4 c0 = *reinterpret_cast<const float4*>(cs + 8 * g);
      const float4 c1 = *reinterpret_cast<const float4*>(cs + 8 * g + 4);
      const float2 cc[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w), make_float2(c1.x, c1.y),
                            make_float2(c1.z, c1.w)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 t = make_float2(__uint_as_float(ws[e] << 16), __uint_as_float(ws[e] & 0xffff0000u));
        v2[4 * g + e] = d == 0 ? f2_mul(t, cc[e]) : f2_fma(t, cc[e], v2[4 * g + e]);
      }
    }
  }
  // stride 1 pairs the two lanes of a float2: scalar
  if (b > 1) {
#pragma unroll
    for (int i = 0; i < W; i += 2) {
      const float a = v[i], c = v[i + 1];
      v[i] = __fadd_rn(a, c);
      v[i + 1] = __fsub_rn(a, c);
    }
  }
#pragma unroll
  for (int hh = 2; hh < W; hh <<= 1) {
    if (hh < b) {
#pragma unroll
      for (int i = 0; i < W; i += 2) {
        if (!(i & hh)) {
          const float2 a = v2[i / 2], c = v2[(i + hh) / 2];
          v2[i / 2] = f2_add(a, c);
          v2[(i + hh) / 2] = f2_sub(a, c);
        }
      }
    }
  }
}

// Tensor-core rotation, row side: this thread's W columns [W*s0, W*s0 + W) of
// tile row `row`: a = T * (chan * hscale) in fp32, split a = hi + lo into bf16
// (round to nearest; lo = bf16(a - hi)), hi written over T in place (the same
// swizzled position, which only this thread reads) and lo at that position of
// the A_lo tile.  The MMA then forms (A_hi + A_lo) H_b.
template <int W>
__device__ __forceinline__ void split_cols(uint8_t* xs, uint8_t* lo_tile, const float* chan, int row, int s0) {
  const int col = s0 * W;
#pragma unroll
  for (int g = 0; g < W / 8; ++g) {
    const int cg = col + 8 * g;  // 64-column box cg / 64, 16-byte chunk (cg % 64) / 8
    const int off = (cg >> 6) * 16384 + row * 128 + ((((cg & 63) >> 3) ^ (row & 7)) << 4);
    const uint4 w = *reinterpret_cast<const uint4*>(xs + off);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    const float4 c0 = *reinterpret_cast<const float4*>(chan + cg);
    const float4 c1 = *reinterpret_cast<const float4*>(chan + cg + 4);
    const float2 cc[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w), make_float2(c1.x, c1.y),
                          make_float2(c1.z, c1.w)};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = f2_mul(make_float2(__uint_as_float(ws[e] << 16), __uint_as_float(ws[e] & 0xffff0000u)), cc[e]);
      hw[e] = bf16x2_rn(a.x, a.y);
      const float2 r = f2_sub(a, make_float2(__uint_as_float(hw[e] << 16), __uint_as_float(hw[e] & 0xffff0000u)));
      lw[e] = bf16x2_rn(r.x, r.y);
    }
    *reinterpret_cast<uint4*>(xs + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Quantise this thread's W values of row `row`, chunk columns starting at `col`.
template <int W>
__device__ __forceinline__ void quantise_cols(const PrologueParams& p, const float (&v)[W], int row, int col,
                                              float g, float y_g) {
  if (p.fmt == FMT_INT4) {
    if constexpr (W == 64)  // the host never runs INT4 in the 32-column layout
      quantise_store_int4<W>(v, row, col, p.K, p.sf_pitch, p.codes, reinterpret_cast<float*>(p.sf), p.z_out);
  } else if (p.fmt == FMT_FP8)
    quantise_store_fp8<W>(v, row, col, p.K, y_g, p.codes, p.z_out);
  else
    quantise_store<W>(v, row, col, p.K, g, y_g, p.codes, p.sf, p.z_out);
}

// Branch operand for this thread's UC columns [c0, c0 + UC) of c.
template <int UC>
__device__ __forceinline__ void write_branch(const PrologueParams& p, const float (&u)[UC], int R, int row, int c0,
                                             float g) {
  const float gs = __fmul_rn(g, p.g_other);
  uint32_t w[UC / 2];
#pragma unroll
  for (int j = 0; j < UC / 2; ++j) {
    float a = u[2 * j], b = u[2 * j + 1];
    if (p.branch_mode == 1) {
      a = __fdiv_rn(a, gs);
      b = __fdiv_rn(b, gs);
    }
    w[j] = pack2(bf16_bits_rn(a), bf16_bits_rn(b));
  }
  uint4* dst = reinterpret_cast<uint4*>(p.branch + static_cast<size_t>(row) * R + c0);
#pragma unroll
  for (int j = 0; j < UC / 8; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  if (p.u_out) {
    float4* o = reinterpret_cast<float4*>(p.u_out + static_cast<size_t>(row) * R + c0);
#pragma unroll
    for (int j = 0; j < UC / 4; ++j) o[j] = make_float4(u[4 * j], u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
  }
}

// Load schedule shared by the producers, the MMA warp and the row threads.
//   merged : one load (T, P, V, chan) serves the projection and the only Z sweep
//   nproj  : projection-only loads (T, P), one per chunk
//   zsweep : sweeps of (T, V, chan) loads over the chunks
//   rev    : the amax sweep after a projection pass takes the chunks in reverse
//            order, so its first loads find the chunks the projection read last
//            still in L2 (a row slab wider than L2 holds is otherwise read twice
//            from DRAM)
//   need_v : the loads of the Z sweeps carry V (not in Local: no deflation)
struct Sched {
  bool merged, rev, need_v;
  int nproj, zsweeps, total;
};

template <int R, int MODE>
__device__ __forceinline__ Sched schedule(int nch) {
  Sched s;
  if constexpr (MODE == 3) {
    // Local: one sweep; each load (T, P, chan) feeds the projection MMA and the
    // quantiser at once, since nothing the rows compute waits for c
    s.merged = R > 0;
    s.rev = false;
    s.need_v = false;
    s.nproj = 0;
    s.zsweeps = 1;
    s.total = nch;
    return s;
  }
  s.need_v = true;
  const bool proj = R > 0 && MODE != 2;
  s.merged = proj && nch == 1 && MODE == 0;  // the tensor-core rotation keeps P and V in one area
  s.nproj = (proj && !s.merged) ? nch : 0;
  s.zsweeps = (MODE == 0 && nch > 1) ? 2 : 1;
  s.total = s.nproj + s.zsweeps * nch;
  s.rev = MODE == 1 && s.nproj > 0;
  return s;
}

template <int R>
__device__ __forceinline__ uint32_t load_kind(const Sched& s, int i) {
  if (i < s.nproj) return LD_X | LD_P;
  uint32_t k = LD_X | LD_CH;
  if (R > 0 && s.need_v) k |= LD_V;
  if (s.merged) k |= LD_P;
  return k;
}

template <int R>
__device__ __forceinline__ uint32_t load_bytes(uint32_t kind) {
  uint32_t n = 0;
  if (kind & LD_X) n += kRows * kChunk * 2;
  if (kind & LD_P) n += 512 * R;
  if (kind & LD_V) n += 512 * R;
  if (kind & LD_CH) n += kChunk * 8;
  return n;
}

// chunk index (within this CTA) of load i
__device__ __forceinline__ int load_chunk(const Sched& s, int i, int nch) {
  if (i < s.nproj) return i;
  const int c = (i - s.nproj) % nch;
  return s.rev ? nch - 1 - c : c;
}

template <int R, int MODE, int W>
__global__ void __launch_bounds__(PCfg<R, MODE, W>::THREADS, 1)
    prologue_kernel(const __grid_constant__ ProMaps maps, const PrologueParams p) {
  using C = PCfg<R, MODE, W>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;         // [2] TMA landed
  uint64_t* empty = bars + 2;    // [2] MMA and row warps done with the slot
  uint64_t* u_full = bars + 4;   // projection MMAs done
  uint64_t* ua_full = bars + 5;  // row warps wrote c hi/lo
  uint64_t* d2_full = bars + 6;  // [2] deflation (TC: Z) MMAs of a chunk done; one buffer unless TC
  uint64_t* d2_free = bars + 8;  // [2] row warps read that result
  uint64_t* a_ready = bars + 10; // [2] TC: row warps wrote A_hi / A_lo of the slot
  uint64_t* h_full = bars + 12;  // TC: H_b landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x;
  const int m0 = blockIdx.y * kRows;
  const int nch = p.chunks;
  const int col0 = part * nch * kChunk;
  const Sched sch = schedule<R, MODE>(nch);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      // TC: the MMA warp is the last reader of a slot (the rows read T before it)
      mbar_init(&empty[i], C::kTC ? 1 : kRowWarps + (C::kMMA ? 1 : 0));
      mbar_init(&d2_full[i], 1);
      mbar_init(&d2_free[i], kRowWarps);
      mbar_init(&a_ready[i], kRowWarps);
    }
    mbar_init(u_full, 1);
    mbar_init(ua_full, kRowWarps);
    mbar_init(h_full, 1);
    fence_barrier_init();
  }
  if constexpr (C::kMMA) {
    if (warp == C::MMA_WARP) {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C::kMMA ? *tmem_slot : 0u;
  // Cluster barriers, in order: A0 (every CTA of the cluster is running, so its
  // shared memory may take remote stores), A1 / A2 (partial c scattered / summed
  // c gathered), B (CTA amax published; Fused).  Every remote store precedes its
  // writer's arrival at the last of these, so once a CTA has passed that
  // barrier no peer touches its shared memory again and it may exit.
  if constexpr (C::kCluster) cluster_arrive();  // A0
  // The next kernel may start its set-up now.  Stats first waits for the kernel
  // before it, so once Quantise (its dependent) runs, T is final and Quantise
  // may load it before its own wait.
  if constexpr (MODE == 1) griddep_wait();
  griddep_launch_dependents();
  const uint32_t d2_tmem = tmem;
  const uint32_t u_tmem = tmem + C::U_COL;

  static_assert(!C::kTC || (C::THREADS == 640 &&
                             256 * C::REG_SPLIT + 256 * C::REG_ROWS + 128 * C::REG_OTHER == 640 * 96),
                "register split of the launch");
  // Each warpgroup changes its register count at one point, at the top of its
  // role branch (the instruction is warpgroup-wide).
  if (warp >= C::PROD0) {
  if constexpr (C::kTC) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_OTHER));
  if (warp < C::MMA_WARP) {
    // ------------------------------------------------------------ producers
    const int my_slot = warp - C::PROD0;
    if (lane == 0 && my_slot == 0) {
      tma_prefetch_desc(&maps.x);
      if constexpr (R > 0) {
        tma_prefetch_desc(&maps.p_hi); tma_prefetch_desc(&maps.p_lo);
        tma_prefetch_desc(&maps.v_hi); tma_prefetch_desc(&maps.v_lo);
      }
    }
    if constexpr (C::kTC) {
      // H_b (a layer constant) once, both 64-column boxes
      if (my_slot == 0) {
        if (lane == 0) mbar_arrive_expect_tx(h_full, C::H_BYTES);
        __syncwarp();
        if (lane < 2) tma_load_2d(smem + C::OFF_H + lane * 16384, &maps.h, h_full, 64 * lane, 0);
      }
    }
    int last = -1;
    bool ok = true;
    bool dep_done = false;  // griddep_wait() done: T may be read
    auto issue = [&](int i) {
      const int slot = i & 1;
      if (slot != my_slot || !ok) return;
      int wok = 1;
      if (lane == 0 && i >= 2) wok = mbar_wait(&empty[slot], ((i >> 1) & 1) ^ 1u, p.err, DEVERR_PRODUCER_WAIT) ? 1 : 0;
      wok = __shfl_sync(0xffffffffu, wok, 0);
      if (!wok) {
        ok = false;
        return;
      }
      const uint32_t kind = load_kind<R>(sch, i);
      uint8_t* s = smem + slot * C::SLOT;
      const int col = col0 + load_chunk(sch, i, nch) * kChunk;
      if (lane == 0) mbar_arrive_expect_tx(&full[slot], load_bytes<R>(kind));
      __syncwarp();
      // one converged instruction: T boxes on lanes 0-1, P^T on 2-5, V on 6-7
      const CUtensorMap* m = nullptr;
      uint8_t* dst = s;
      int x = 0, y = 0;
      if (lane < 2) {
        m = &maps.x; dst = s + lane * 16384; x = col + 64 * lane; y = m0;
      } else if (R > 0 && lane < 6 && (kind & LD_P)) {
        const int pp = (lane - 2) >> 1, kb = (lane - 2) & 1;
        m = pp ? &maps.p_lo : &maps.p_hi; dst = s + C::OFF_P + (kb * 2 + pp) * R * 128; x = col + kb * 64; y = 0;
      } else if (R > 0 && lane >= 6 && lane < 8 && (kind & LD_V)) {
        const int pp = lane - 6;
        m = pp ? &maps.v_lo : &maps.v_hi; dst = s + C::OFF_V + pp * 256 * R; x = 0; y = col;
      }
      // This warp's first load: the layer constants (P, V, chan) go out while the
      // previous kernel in the stream may still run; T only after it finished
      // (Quantise: T was final before it launched).
      if (m && (dep_done || lane >= 2 || MODE == 2)) tma_load_2d(dst, m, &full[slot], x, y);
      if (!dep_done) {
        if constexpr (MODE != 2) griddep_wait();  // Quantise's producers read nothing Stats writes
        dep_done = true;
        if (m && lane < 2 && MODE != 2) tma_load_2d(dst, m, &full[slot], x, y);
      }
      if (lane == 0 && (kind & LD_CH)) bulk_load(s + C::OFF_CH, p.chan + 2 * col, C::CH_BYTES, &full[slot]);
      last = i;
    };
    // The producers pass each cluster barrier before any load whose ring slot
    // the rows free only after that barrier (a slot is reused two loads later),
    // so no wait here depends on a barrier this warp has not reached.
    const int zs1 = sch.nproj, zs2 = sch.nproj + nch;
    bool didA = !C::kNeedA, didB = !C::kNeedB;
    auto pass_a = [&]() {
      if (!didA) {
        __syncwarp();
        cluster_wait();    // A0
        cluster_arrive();  // A1
        cluster_wait();
        cluster_arrive();  // A2
        didA = true;
      }
    };
    auto pass_b = [&]() {
      if (!didB) {
        pass_a();
        __syncwarp();
        cluster_wait();    // A2, or A0 without the exchange of c
        cluster_arrive();  // B
        didB = true;
      }
    };
    for (int i = 0; i < sch.total; ++i) {
      // (Local: the rows free every slot without a barrier, so the producers
      // issue every load first)
      if (MODE != 3 && i == zs1 + 2) pass_a();
      if (sch.zsweeps == 2 && i == zs2 + 2) pass_b();
      issue(i);
    }
    pass_a();
    pass_b();
    __syncwarp();
    if (lane == 0 && last >= 0) mbar_wait(&full[last & 1], (last >> 1) & 1, p.err, DEVERR_DRAIN_WAIT);
    if constexpr (C::kTC)
      if (lane == 0 && my_slot == 0) mbar_wait(h_full, 0, p.err, DEVERR_DRAIN_WAIT);
    __syncwarp();
    if constexpr (C::kCluster) cluster_wait();  // the last barrier arrived at (B, else A2)
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if constexpr (C::kMMA) {
      bool ok = true;
      int i = 0, j = 0;
      if constexpr (C::kProj) {
        if (lane == 0) {
          uint32_t acc = 0;
          for (int c = 0; ok && c < nch; ++c) {
            const int slot = i & 1;
            ok = mbar_wait(&full[slot], (i >> 1) & 1, p.err, DEVERR_MMA_WAIT);
            if (!ok) break;
            tc_fence_after();
            const uint32_t xs = smem_u32(smem + slot * C::SLOT);
            const uint32_t ps = xs + C::OFF_P;
            // B = [P^T hi; P^T lo] (2R rows): columns [0, R) of the result
            // accumulate T P_hi, columns [R, 2R) accumulate T P_lo
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t a = smem_desc(xs + kb * 16384 + k * 32, 16, 1024, 2);
                const uint64_t b = smem_desc(ps + kb * 2 * R * 128 + k * 32, 16, 1024, 2);
                mma_bf16(u_tmem, a, b, idesc_bf16(128, 2 * R), acc);
                acc = 1u;
              }
            if (!sch.merged || MODE == 3) {  // Local: the projection is the slot's only MMA
              tc_commit(&empty[slot]);
              ++i;
            }
          }
          tc_commit(u_full);
        }
        __syncwarp();
      }
      if constexpr (C::kNeedA) {
        cluster_wait();    // A0
        cluster_arrive();  // A1
        cluster_wait();
        cluster_arrive();  // A2
      }
      if constexpr (C::kTC) {
        // Z of chunk c = (A_hi + A_lo) H_b - c V^T into TMEM buffer c % 2, once the
        // rows have written A of the chunk's slot and read the buffer's last Z
        auto zmma = [&](int c) {
          const int li = sch.nproj + c, slot = li & 1, db = c & 1;
          if (!mbar_wait(&full[slot], (li >> 1) & 1, p.err, DEVERR_MMA_WAIT)) return false;
          if (!mbar_wait(&a_ready[slot], (c >> 1) & 1, p.err, DEVERR_MMA_WAIT)) return false;
          if (!mbar_wait(&d2_free[db], ((c >> 1) & 1) ^ 1u, p.err, DEVERR_MMA_WAIT)) return false;
          tc_fence_after();
          const uint32_t d = d2_tmem + 128u * db;
          const uint32_t xs = smem_u32(smem + slot * C::SLOT), hs = smem_u32(smem + C::OFF_H);
#pragma unroll
          for (int part = 0; part < 2; ++part)  // A_hi, then A_lo
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t a = smem_desc(xs + part * C::OFF_ALO + kb * 16384 + k * 32, 16, 1024, 2);
                const uint64_t b = smem_desc(hs + kb * 16384 + k * 32, 16, 1024, 2);
                mma_bf16(d, a, b, idesc_bf16(128, 128), (part | kb | k) ? 1u : 0u);
              }
          if constexpr (R > 0) {
            // + (-c)(V^T): UA holds -c, split hi/lo like V
            const uint32_t sbo_u = 8u * 2u * R;
            const uint32_t swz_u = umma_swizzle_code(2 * R);
            const uint32_t vs = xs + C::OFF_V;
            const uint32_t ua = smem_u32(smem + C::OFF_UA);
#pragma unroll
            for (int k = 0; k < R / 16; ++k) {
              const uint64_t ah = smem_desc(ua + k * 32, 16, sbo_u, swz_u);
              const uint64_t al = smem_desc(ua + 256 * R + k * 32, 16, sbo_u, swz_u);
              const uint64_t bh = smem_desc(vs + k * 32, 16, sbo_u, swz_u);
              const uint64_t bl = smem_desc(vs + 256 * R + k * 32, 16, sbo_u, swz_u);
              mma_bf16(d, al, bh, idesc_bf16(128, 128), 1u);
              mma_bf16(d, ah, bl, idesc_bf16(128, 128), 1u);
              mma_bf16(d, ah, bh, idesc_bf16(128, 128), 1u);
            }
          }
          tc_commit(&d2_full[db]);
          tc_commit(&empty[slot]);
          return true;
        };
        if (lane == 0) {
          if constexpr (R > 0) ok = ok && mbar_wait(ua_full, 0, p.err, DEVERR_MMA_WAIT);
          ok = ok && mbar_wait(h_full, 0, p.err, DEVERR_MMA_WAIT);
          for (int c = 0; ok && c < nch; ++c) ok = zmma(c);
        }
        __syncwarp();
      } else if constexpr (MODE != 3) {
        // deflation of one chunk: D2[128 x 128] = c (hi/lo) . V_chunk^T (hi/lo)
        const uint32_t sbo_u = 8u * 2u * R;
        const uint32_t swz_u = umma_swizzle_code(2 * R);
        auto deflate = [&]() {
          const int slot = i & 1;
          if (!mbar_wait(&full[slot], (i >> 1) & 1, p.err, DEVERR_MMA_WAIT)) return false;
          if (!mbar_wait(d2_free, (j & 1) ^ 1u, p.err, DEVERR_MMA_WAIT)) return false;
          tc_fence_after();
          const uint32_t vs = smem_u32(smem + slot * C::SLOT + C::OFF_V);
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
          tc_commit(&empty[slot]);
          ++i;
          ++j;
          return true;
        };
        if (lane == 0) {
          ok = ok && mbar_wait(ua_full, 0, p.err, DEVERR_MMA_WAIT);
          for (int c = 0; ok && c < nch; ++c) ok = deflate();
        }
        __syncwarp();
        if constexpr (C::kNeedB) {
          cluster_wait();    // A2
          cluster_arrive();  // B
        }
        if (sch.zsweeps == 2) {
          if (lane == 0)
            for (int c = 0; ok && c < nch; ++c) ok = deflate();
          __syncwarp();
        }
      }
    } else {
      if constexpr (C::kNeedB) {
        cluster_wait();    // A0
        cluster_arrive();  // B
      }
    }
    if constexpr (C::kCluster) cluster_wait();  // the last barrier arrived at (B, else A2)
  } else {
    // ------------------------------------------------------------ spare warp (TC)
    if constexpr (C::kNeedA) {
      cluster_wait();    // A0
      cluster_arrive();  // A1
      cluster_wait();
      cluster_arrive();  // A2
    }
    if constexpr (C::kCluster) cluster_wait();
  }
  } else if (C::kTC && warp < C::ROW0) {
    if constexpr (C::kTC) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_SPLIT));
    // ------------------------------------------------------------ split warps (TC)
    // A_hi / A_lo of every chunk, as soon as its load has landed; warp w takes
    // row (w % 4) * 32 + lane, columns [64 (w / 4), 64 (w / 4) + 64).
    const int zrow = (warp & 3) * 32 + lane, s0 = warp >> 2;
    auto prep_a = [&](int c) {
      const int li = sch.nproj + c, slot = li & 1;
      mbar_wait(&full[slot], (li >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      uint8_t* s = smem + slot * C::SLOT;
      split_cols<W>(s, s + C::OFF_ALO, reinterpret_cast<const float*>(s + C::OFF_CH), zrow, s0);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_ready[slot]);
    };
    // Stats: the exchange of c uses the A_lo areas and needs every thread at its
    // cluster barriers, so these warps pass the barriers first and write A only
    // once the rows have read the gathered c (ua_full).
    if constexpr (C::kNeedA) {
      cluster_wait();    // A0
      cluster_arrive();  // A1
      cluster_wait();
      cluster_arrive();  // A2
      mbar_wait(ua_full, 0, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
    }
    for (int c = 0; c < nch; ++c) prep_a(c);
    __syncwarp();
    if constexpr (C::kCluster) cluster_wait();  // A2
  } else {
    if constexpr (C::kTC) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_ROWS));
    // ------------------------------------------------------------ row threads
    // outputs (and the workspace they live in) may still be read by the
    // previous kernel in the stream until it has finished
    griddep_wait();
    const int rw = warp - C::ROW0;  // row warp 0..7
    const int q = warp & 3;         // TMEM lane quarter this warp may access
    const int hf = rw >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // Z work: row zrow (tile-local), columns [W * s0, W * s0 + W) of each chunk
    const bool zact = C::kSmall ? (rw < 4) : true;
    const int zrow = C::kSmall ? lane : q * 32 + lane;
    const int s0 = C::kSmall ? rw : hf;
    const int zrow_g = m0 + zrow;
    const bool zvalid = zact && zrow_g < p.rows;
    // c work: row urow, columns [uc0, uc0 + UC)
    const bool uact = C::kSmall ? (q == 0) : true;
    const int urow = q * 32 + lane;
    const int urow_g = m0 + urow;
    const bool uvalid = uact && urow_g < p.rows;
    const int uc0 = hf * C::UC;

    float u[C::UC];
#pragma unroll
    for (int k = 0; k < C::UC; ++k) u[k] = 0.0f;
    int i = 0, j = 0;

    // projection-only loads: the rows do not read them (TC: the MMA warp alone
    // releases them)
    for (int c = 0; c < sch.nproj && !C::kTC; ++c, ++i) {
      mbar_wait(&full[i & 1], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[i & 1]);
    }

    // Partial c of this CTA's K range (T P_hi + T P_lo, from TMEM), summed
    // over the cluster: reduce-scatter by row slice, then all-gather, both by
    // remote stores (remote loads would cost a round trip each).
    auto gather_c = [&]() {
      if constexpr (C::kProj) {
      mbar_wait(u_full, 0, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
      tc_fence_after();
      const int SL = (C::kSmall ? 32 : kRows) / p.parts;  // rows per owner
      const uint32_t my_rank = cluster_rank();
      float* rs = reinterpret_cast<float*>(smem + C::OFF_RS);
      float* ug = reinterpret_cast<float*>(smem + C::OFF_UG);
      cluster_wait();  // A0
      if (uact) {
        float pu[C::UC];
        if constexpr (C::UC == 16) {
          uint32_t a16[16], b16[16];
          tmem_ld_32x32b_x16(u_tmem + lane_base + uc0, a16);
          tmem_ld_32x32b_x16(u_tmem + lane_base + R + uc0, b16);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) pu[k] = __fadd_rn(__uint_as_float(a16[k]), __uint_as_float(b16[k]));
        } else {
          uint32_t a8[8], b8[8];
          tmem_ld_32x32b_x8(u_tmem + lane_base + uc0, a8);
          tmem_ld_32x32b_x8(u_tmem + lane_base + R + uc0, b8);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) pu[k] = __fadd_rn(__uint_as_float(a8[k]), __uint_as_float(b8[k]));
        }
        const uint32_t dst = dsmem_addr(smem_u32(rs + (static_cast<int>(my_rank) * SL + urow % SL) * R + uc0),
                                        static_cast<uint32_t>(urow / SL));
#pragma unroll
        for (int k = 0; k < C::UC / 4; ++k)
          dsmem_st_f4(dst + 16u * k, make_float4(pu[4 * k], pu[4 * k + 1], pu[4 * k + 2], pu[4 * k + 3]));
      }
      cluster_arrive();  // A1
      cluster_wait();
      for (int it = 32 * rw + lane; it < SL * (R / 4); it += kRowThreads) {
        const int srow = it / (R / 4), c4 = it % (R / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int rk = 0; rk < p.parts; ++rk) {  // rank order: deterministic
          const float4 v = *reinterpret_cast<const float4*>(rs + (rk * SL + srow) * R + 4 * c4);
          acc.x = __fadd_rn(acc.x, v.x);
          acc.y = __fadd_rn(acc.y, v.y);
          acc.z = __fadd_rn(acc.z, v.z);
          acc.w = __fadd_rn(acc.w, v.w);
        }
        const uint32_t src = smem_u32(ug + (static_cast<int>(my_rank) * SL + srow) * C::UG_STRIDE + 4 * c4);
        for (int rk = 0; rk < p.parts; ++rk) dsmem_st_f4(dsmem_addr(src, static_cast<uint32_t>(rk)), acc);
      }
      cluster_arrive();  // A2
      cluster_wait();
      if (uact) {
        const float* g = ug + urow * C::UG_STRIDE + uc0;
#pragma unroll
        for (int k = 0; k < C::UC; k += 4) {
          const float4 v = *reinterpret_cast<const float4*>(g + k);
          u[k] = v.x; u[k + 1] = v.y; u[k + 2] = v.z; u[k + 3] = v.w;
        }
      }
      }
    };
    if constexpr (MODE == 3) {
      // Local: every chunk quantised as it lands (x * chan, no deflation, the
      // group scales local), then the cluster sum of c for the branch bf16(c)
      float z[W];
      for (int c = 0; c < nch; ++c, ++i) {
        const int slot = i & 1;
        mbar_wait(&full[slot], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
        const uint8_t* s = smem + slot * C::SLOT;
        rotate_cols<W>(s, reinterpret_cast<const float*>(s + C::OFF_CH), zrow, s0, p.b, z);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (zvalid) quantise_cols<W>(p, z, zrow_g, col0 + c * kChunk + s0 * W, 1.0f, 1.0f);
      }
      if constexpr (C::kProj) {
        gather_c();
        if (part == 0 && uvalid) write_branch<C::UC>(p, u, R, urow_g, uc0, 1.0f);
      }
    } else {
    if constexpr (C::kProj) {
      gather_c();
      if (MODE == 1 && part == 0 && uvalid) {
        float4* o = reinterpret_cast<float4*>(p.u_glob + static_cast<size_t>(urow_g) * R + uc0);
#pragma unroll
        for (int k = 0; k < C::UC / 4; ++k) o[k] = make_float4(u[4 * k], u[4 * k + 1], u[4 * k + 2], u[4 * k + 3]);
      }
    }
    if constexpr (MODE == 2 && R > 0) {
      if (uvalid) {
        const float4* src = reinterpret_cast<const float4*>(p.u_glob + static_cast<size_t>(urow_g) * R + uc0);
#pragma unroll
        for (int k = 0; k < C::UC / 4; ++k) {
          const float4 a = src[k];
          u[4 * k] = a.x; u[4 * k + 1] = a.y; u[4 * k + 2] = a.z; u[4 * k + 3] = a.w;
        }
        if (part == 0) write_branch<C::UC>(p, u, R, urow_g, uc0, scale_from_amax(__uint_as_float(*p.amax_glob), p.fmt));
      }
    }
    if constexpr (R > 0) {
      // c hi/lo as the A operand of the deflation (replicated in the small layout)
      if (uact) {
        uint8_t* ua = smem + C::OFF_UA;
#pragma unroll
        for (int jj = 0; jj < C::UC / 8; ++jj) {
          uint4 hi, lo;
          float uu[8];  // TC: -c, so the Z accumulation subtracts c V^T
#pragma unroll
          for (int e = 0; e < 8; ++e) uu[e] = C::kTC ? -u[8 * jj + e] : u[8 * jj + e];
          split8(uu, hi, lo);
          const int ch = uc0 / 8 + jj;
#pragma unroll
          for (int rep = 0; rep < (C::kSmall ? 4 : 1); ++rep) {
            const int row = urow + 32 * rep;
            put16(ua, row, ch, 2 * R, hi);
            put16(ua + 256 * R, row, ch, 2 * R, lo);
          }
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(ua_full);
    }

    // Z = T~ - c V^T for chunk c from ring load i
    float z[W];
    auto zchunk = [&]() {
      const int slot = i & 1;
      mbar_wait(&full[slot], (i >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      const uint8_t* s = smem + slot * C::SLOT;
      if (zact) rotate_cols<W>(s, reinterpret_cast<const float*>(s + C::OFF_CH), zrow, s0, p.b, z);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if constexpr (R > 0) {
        mbar_wait(d2_full, j & 1, p.err, DEVERR_EPILOGUE_WAIT);
        __syncwarp();
        tc_fence_after();
        if (zact) {
#pragma unroll
          for (int pc = 0; pc < W / 32; ++pc) {
            uint32_t r32[32];
            tmem_ld_32x32b_x32(d2_tmem + lane_base + s0 * W + pc * 32, r32);
            tmem_ld_wait();
            float2* z2 = reinterpret_cast<float2*>(z + pc * 32);
#pragma unroll
            for (int k = 0; k < 16; ++k)
              z2[k] = f2_sub(z2[k], make_float2(__uint_as_float(r32[2 * k]), __uint_as_float(r32[2 * k + 1])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(d2_free);
        ++j;
      }
      ++i;
    };

    // TC: Z of chunk c, read back from TMEM buffer c % 2
    auto read_z = [&](int c) {
      const int db = c & 1;
      mbar_wait(&d2_full[db], (c >> 1) & 1, p.err, DEVERR_EPILOGUE_WAIT);
      __syncwarp();
      tc_fence_after();
      if (zact) {
#pragma unroll
        for (int pc = 0; pc < W / 32; ++pc) {
          uint32_t r32[32];
          tmem_ld_32x32b_x32(d2_tmem + 128u * db + lane_base + s0 * W + pc * 32, r32);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) z[pc * 32 + k] = __uint_as_float(r32[k]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d2_free[db]);
    };

    float g = 1.0f;
    if constexpr (MODE == 2) g = scale_from_amax(__uint_as_float(*p.amax_glob), p.fmt);
    float y_g = rcp_rn(g);
    float amax = 0.0f;
    for (int c = 0; c < nch; ++c) {
      if constexpr (C::kTC) {
        read_z(c);  // the split warps prepare A
      } else {
        zchunk();
      }
      const int col = col0 + c * kChunk + s0 * W;
      if constexpr (MODE == 2) {
        if (zvalid) quantise_cols<W>(p, z, zrow_g, col, g, y_g);
      } else if (zact) {
#pragma unroll
        for (int k = 0; k < W; ++k) amax = fmaxf(amax, fabsf(z[k]));
      }
    }
    if constexpr (MODE == 0 && !C::kNeedA) cluster_wait();  // A0, before the remote stores below
    if constexpr (MODE != 2) {
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      if (lane == 0) red[rw] = __uint_as_float(wmax);
      named_bar(1, kRowThreads);
      if (rw == 0) {
        float cmax = red[0];
#pragma unroll
        for (int w = 1; w < kRowWarps; ++w) cmax = fmaxf(cmax, red[w]);
        if constexpr (MODE == 1) {
          if (lane == 0) atomicMax(p.amax_glob, __float_as_uint(cmax));
        } else if (lane < p.parts) {
          // push this CTA's maximum into slot [8 + rank] of every rank
          const uint32_t slot = smem_u32(red + kRowWarps + cluster_rank());
          dsmem_st_f32(dsmem_addr(slot, static_cast<uint32_t>(lane)), cmax);
        }
      }
    }
    if constexpr (MODE == 0) {
      cluster_arrive();  // B
      cluster_wait();
      float A = 0.0f;
      for (int rk = 0; rk < p.parts; ++rk) A = fmaxf(A, red[kRowWarps + rk]);
      g = scale_from_amax(A, p.fmt);
      y_g = rcp_rn(g);
      if constexpr (R > 0) {
        if (part == 0 && uvalid) write_branch<C::UC>(p, u, R, urow_g, uc0, g);
      }
      if (part == 0 && blockIdx.y == 0 && rw == 0 && lane == 0) *p.g_out = g;
      if (nch == 1) {
        if (zvalid) quantise_cols<W>(p, z, zrow_g, col0 + s0 * W, g, y_g);
      } else {
        for (int c = 0; c < nch; ++c) {
          zchunk();
          if (zvalid) quantise_cols<W>(p, z, zrow_g, col0 + c * kChunk + s0 * W, g, y_g);
        }
      }
    }
    if constexpr (MODE == 2) {
      if (part == 0 && blockIdx.y == 0 && rw == 0 && lane == 0) *p.g_out = g;
    }
    }  // MODE != 3
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C::kMMA) {
    if (warp == C::MMA_WARP) {
      __syncwarp();
      tmem_dealloc(tmem, C::TMEM_COLS);
    }
  }
}

template <int R, int MODE, int W>
cudaError_t launch_one(const ProMaps& maps, const PrologueParams& p_in, cudaStream_t st) {
  using C = PCfg<R, MODE, W>;
  auto kern = prologue_kernel<R, MODE, W>;
  static const cudaError_t smem_attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (smem_attr != cudaSuccess) return smem_attr;
  PrologueParams p = p_in;
  if (p.parts < 1 || p.parts > kMaxParts || (p.parts & (p.parts - 1))) return cudaErrorInvalidValue;
  static_assert(8 + kMaxParts <= 32, "per-rank maxima fit the reduction area");
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (C::kCluster && p.parts > 8) {
    // 16 CTAs per cluster is beyond the portable size: allowed per kernel, and
    // used only when the device can place such a cluster (else 8 CTAs with
    // twice the chunks each)
    static const bool ok16 = [&]() {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
      }
      cudaLaunchConfig_t q = cfg;
      cudaLaunchAttribute a = {};
      a.id = cudaLaunchAttributeClusterDimension;
      a.val.clusterDim.x = 16;
      a.val.clusterDim.y = 1;
      a.val.clusterDim.z = 1;
      q.attrs = &a;
      q.numAttrs = 1;
      q.gridDim = dim3(16, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
      }
      return n > 0;
    }();
    if (!ok16) {
      p.parts = 8;
      p.chunks *= 2;
    }
  }
  cfg.gridDim = dim3(p.parts, (p.rows + kRows - 1) / kRows, 1);
  if (C::kCluster) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = p.parts;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

template <int R>
cudaError_t launch_r(const ProMaps& maps, const PrologueParams& p, PrologueMode mode, cudaStream_t st) {
  switch (mode) {
    case PrologueMode::Fused:
      // one row tile, since the cluster's amax is the tensor's; INT4 scales are
      // local, so its row tiles may run side by side
      if (p.rows > kRows && p.fmt != FMT_INT4) return cudaErrorInvalidValue;
      // the INT4 quantiser takes one 64-column group per thread
      return p.rows <= 32 && p.fmt != FMT_INT4 ? launch_one<R, 0, 32>(maps, p, st) : launch_one<R, 0, 64>(maps, p, st);
    case PrologueMode::Stats: return launch_one<R, 1, 64>(maps, p, st);
    case PrologueMode::Quantise: return launch_one<R, 2, 64>(maps, p, st);
    case PrologueMode::Local:
      if (p.fmt != FMT_INT4 || p.b != 1) return cudaErrorInvalidValue;
      return launch_one<R, 3, 64>(maps, p, st);
  }
  return cudaErrorInvalidValue;
}

// Stats / Quantise split registers between warpgroups (setmaxnreg); their
// launch gives each of the 640 threads the split's average
template <int R, int MODE>
bool split_ok(char* msg, size_t n) {
  using C = PCfg<R, MODE, 64>;
  constexpr int want = (256 * C::REG_SPLIT + 256 * C::REG_ROWS + 128 * C::REG_OTHER) / C::THREADS;
  cudaFuncAttributes a{};
  const cudaError_t e = cudaFuncGetAttributes(&a, prologue_kernel<R, MODE, 64>);
  if (e != cudaSuccess) {
    snprintf(msg, n, "cudaFuncGetAttributes(prologue_kernel<%d,%d,64>) failed: %s", R, MODE, cudaGetErrorString(e));
    return false;
  }
  if ((a.numRegs + 7) / 8 * 8 != want) {
    snprintf(msg, n,
             "prologue_kernel<%d,%d,64> was compiled to %d registers per thread; its warpgroup register split "
             "assumes %d",
             R, MODE, a.numRegs, want);
    return false;
  }
  return true;
}

}  // namespace

bool prologue_register_split_ok(char* msg, size_t n) {
  return split_ok<0, 1>(msg, n) && split_ok<0, 2>(msg, n) && split_ok<16, 1>(msg, n) && split_ok<16, 2>(msg, n) &&
         split_ok<32, 1>(msg, n) && split_ok<32, 2>(msg, n);
}

cudaError_t launch_prologue(const ProMaps& maps, const PrologueParams& p, int r, PrologueMode mode,
                            cudaStream_t st) {
  switch (r) {
    case 0: return launch_r<0>(maps, p, mode, st);
    case 16: return launch_r<16>(maps, p, mode, st);
    case 32: return launch_r<32>(maps, p, mode, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qwam
