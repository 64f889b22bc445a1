// Internal launch interface between the C-ABI host layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace qwam {

// One "rows" job of the activation prologue / weight prepare:
//   T~ = (T * chan) H,  c = T~ V = T P,  Z = T~ - c V^T,  quantise(Z),
// with T = x, chan = 1/s on the activation side and T = W, chan = s on the
// weight side, and P = diag(chan) H V precomputed once per layer.  T, P and V
// reach the kernel through TMA tensor maps.
struct ProMaps {
  CUtensorMap x;     // T bf16 [rows, K], box 64 x 128 rows, 128B swizzle
  CUtensorMap p_hi;  // P^T bf16 [r, K] (hi/lo split of fp32 P), box 64 x r, 128B swizzle
  CUtensorMap p_lo;
  CUtensorMap v_hi;  // V bf16 [K, r] (hi/lo split), box r x 128 rows, 2r-byte swizzle
  CUtensorMap v_lo;
  CUtensorMap h;     // H_b blocks of one 128-column chunk (+-1, block diagonal) bf16 [128, 128], box 64 x 128, 128B swizzle
};

struct PrologueParams {
  const float* chan;      // fp32 [K / 128][2][128]: chan * hscale, then -(chan * hscale), per chunk
  int rows;
  int K;
  int b;                  // Hadamard block (power of two, <= 128)
  int chunks;             // 128-column chunks per CTA
  int parts;              // CTAs along K per row tile (one cluster when they exchange)
  float hscale;           // fp32(1 / sqrt(b))
  float* u_glob;          // fp32 [rows, r]: written by Stats, read by Quantise
  uint32_t* amax_glob;    // fp32 bits of max|Z|: atomicMax'd by Stats
  uint8_t* codes;         // [rows, K/2]
  uint8_t* sf;            // tiled scales, rows padded to 128
  uint16_t* branch;       // bf16 bits [rows, r]
  int branch_mode;        // 0: bf16(c)   1: bf16(c / (g * g_other))
  float g_other;
  float* g_out;           // fp32 scalar: the per-tensor scale of Z
  float* z_out;           // optional fp32 [rows, K] (debug export of Z)
  float* u_out;           // optional fp32 [rows, r] (debug export of c)
  uint32_t* err;          // device error word for bounded waits
  int fmt;                // element format: 0 NVFP4 (codes [rows, K/2] + tiled
                          // scales), 1 FP8 E4M3 (codes [rows, K], no block scales),
                          // 2 INT4 group 64 (levels as E4M3 bytes [rows, K]; sf
                          // holds fp32 scales [K / 64][sf_pitch])
  int sf_pitch;           // INT4: row pitch of the scale array, in scales
};

// Local: the SVDQuant arm's activation side (b = 1, INT4): x * chan quantised
// group by group as it is read, no deflation and no tensor-wide amax, so every
// row tile is independent; c = x P still summed across the row tile's cluster
// for the branch operand bf16(c).
enum class PrologueMode { Fused = 0, Stats = 1, Quantise = 2, Local = 3 };

// Grid: parts x ceil(rows / 128) CTAs; Fused, Stats and Local (r > 0) launch
// the parts of a row tile as one cluster.  Fused requires rows <= 128 (INT4,
// whose scales are local: any rows); Stats requires *amax_glob == 0; Local
// requires fmt == INT4.
cudaError_t launch_prologue(const ProMaps& maps, const PrologueParams& p, int r, PrologueMode mode,
                            cudaStream_t st);

// Rank 0, more than 128 rows: Stats / Quantise with the rotation as one bf16
// tensor-core product against B = diag(chan / sqrt(b)) H_b (hi / lo) per
// 128-column chunk; grid = (K / 128) x groups CTAs, CTA (c, g) taking the row
// tiles g, g + groups, ...  x: the prologue's x tensor map.  Stats requires
// *amax_glob == 0; p.chan, p.rows, p.K, p.b, p.amax_glob, p.codes, p.sf,
// p.g_out, p.z_out, p.err are read.
int wide_prologue_groups(int rows, int K, int sms);
// One launch of the same rotation for up to six row tiles per CTA and every CTA
// resident (a cooperative launch): x read once, Z kept on chip across one
// bounded grid-wide barrier for the amax.  Requires the 16 bytes at
// p.amax_glob (amax, g_x, barrier count) to be zero at launch.
bool onepass_prologue_fits(int rows, int K, int groups, int sms);
cudaError_t launch_prologue_onepass(const CUtensorMap& x, const PrologueParams& p, int groups, cudaStream_t st);
cudaError_t launch_prologue_wide(const CUtensorMap& x, const PrologueParams& p, PrologueMode mode, int groups,
                                 cudaStream_t st);

cudaError_t launch_recip(const float* s, float* inv_s, int K, uint32_t* err, cudaStream_t st);
// counts[0..2] += mismatches of the quantiser's a / 6 and 1 / a (every positive
// fp32 a) and of the E4M3 code of u / g, against the IEEE fp32 operations.
cudaError_t launch_rounding_check(unsigned long long* counts, unsigned long long n_pairs, cudaStream_t st);
// out [K / 128][2][128] fp32: chunk c holds chan[128c..] * hscale, then its negation.
cudaError_t launch_chan_pm(const float* chan, float hscale, int K, float* out, cudaStream_t st);
cudaError_t launch_split_v(const float* V, int K, int r, uint16_t* v_hi, uint16_t* v_lo, cudaStream_t st);
// P^T = (diag(chan) H V)^T split into bf16 hi/lo, [r, K] each; H block size b.
cudaError_t launch_make_proj(const float* V, const float* chan, int K, int r, int b, uint16_t* p_hi, uint16_t* p_lo,
                             cudaStream_t st);
// L [N, r] bf16 = g * deq(codes, sf) V (V fp32 [K, r], r <= 32): the branch
// weight of the shared-weight arm, from its stored FP4 weight.
cudaError_t launch_dequant_project(const uint8_t* codes, const uint8_t* sf, const float* g, const float* V, int N,
                                   int K, int r, uint16_t* L, cudaStream_t st);
cudaError_t launch_quantize_fp32(const float* T, int rows, int K, uint8_t* codes, uint8_t* sf, float* g_out,
                                 uint32_t* amax_scratch, cudaStream_t st);

// Block-scaled FP4 GEMM.
enum class GemmEpilogue { Bf16 = 0, RawF32 = 1, SplitK = 2 };

struct GemmParams {
  int M, N, K;
  int k_stages;            // ceil(K / ks), ks = K elements per pipeline stage
  int splits;              // 1, or 2 / 4 / 8 (split-K cluster; splits <= k_stages)
  const uint8_t* sfa;      // tiled, rows padded to 128
  const uint8_t* sfb;      // tiled, rows padded to 256
  const float* g_a_ptr;    // device scalar (activation scale) or nullptr
  float g_a;               // used when g_a_ptr == nullptr
  float g_b;
  int has_branch;          // rank-r branch in the accumulator (r = branch_k)
  int branch_k;
  const void* bias;        // bf16 [N] or nullptr
  void* y;                 // bf16 [M, N]
  float* out_f32;          // fp32 [M, N] (raw epilogue)
  uint32_t* err;
  int sms;                 // SMs of the device (0: queried at launch)
  uint64_t wait_ns;        // limit of every bounded wait (0: the default)
  // test only: stage 0 expects this many bytes more than its boxes carry, so
  // its barrier never completes and every wait behind it runs out (0: off)
  uint32_t withheld_bytes;
};

struct GemmMaps {
  CUtensorMap a;    // codes A [M, K/2] u8, box (ks/2) B x 128 rows, 128B (ks 256) / 64B (ks 128) swizzle
  CUtensorMap b;    // codes B [N, K/2] u8, box (ks/2) B x bn rows, same swizzle
  CUtensorMap u;    // branch A [M, r] bf16, box r x 128 rows
  CUtensorMap l;    // branch B [N, r] bf16, box r x bn rows
  CUtensorMap y;    // output y [M, N] bf16 (bf16 epilogue): box 64 x 128 rows, 128B swizzle; on CTA pairs 32 x 128, 64B swizzle
  CUtensorMap sfa;  // A scales viewed as u8 [rows * K / 16 / 256, 256], box 256 x (ks / 32): one stage of 128 rows
  CUtensorMap sfb;  // B scales, same view and box
};

// Tile width, K per pipeline stage and CTA pairing for an M x N output.  With
// pair set, a two-CTA cluster computes 256 x bn tiles (cta_group::2) and each
// CTA reads bn / 2 rows of B: the B (and L) tensor maps must have bn / 2-row
// boxes.  gemm_shape proposes pair for bn == 256; a split-K plan turns it off.
struct GemmShape {
  int bn, ks;   // tile width, K elements per pipeline stage
  bool pair;
  bool fp8;     // FP8 E4M3 operands (the W8A8 arm) instead of NVFP4
};
GemmShape gemm_shape(int M, int N, bool fp8 = false);

// p.k_stages must be ceil(K / shape.ks); split-K (p.splits in {2, 4, 8}) needs
// the SplitK epilogue, shape.pair false, and launches one cluster of p.splits
// CTAs per tile.
cudaError_t launch_gemm(const GemmMaps& maps, const GemmParams& p, GemmShape shape, GemmEpilogue epi,
                        cudaStream_t st);

// INT4 group-64 GEMM of the SVDQuant arm:
//   y = sum_g sa[:, g] sb[:, g]^T * P_g + u' L^T + bias,  P_g the exact group sums
// on E4M3-coded levels.  128 x 128 tiles, K in stages of 128 (two groups).
struct GroupGemmParams {
  int M, N, K;             // K % 128 == 0
  int splits;              // K splits (grid z); the stages are shared out evenly
  int branch_k;            // r of the bf16 branch (0: none); split 0 adds it
  const void* bias;        // bf16 [N] or nullptr (bf16 output only)
  void* y;                 // bf16 [M, N]; nullptr: fp32 partial tiles instead
  float* partial;          // fp32 [splits][M][N] when y == nullptr
  uint32_t* err;
  uint64_t wait_ns;        // limit of every bounded wait (0: the default)
};

struct GroupGemmMaps {
  CUtensorMap a;    // A levels [M, K] u8 (E4M3 bytes) as a 3-D map (bytes, rows, 1), box 128 B x 128 rows x 1, 128B swizzle
  CUtensorMap b;    // B levels [N, K] u8, same form
  CUtensorMap sa;   // A scales fp32 [K / 64][pitch >= M], box 128 rows x 2 groups
  CUtensorMap sb;   // B scales fp32 [K / 64][N], same box
  CUtensorMap u;    // branch A [M, r] bf16, box r x 128 rows (unread when r == 0)
  CUtensorMap l;    // branch B [N, r] bf16, box r x 128 rows
};

cudaError_t launch_group_gemm(const GroupGemmMaps& maps, const GroupGemmParams& p, cudaStream_t st);
// y = bf16(sum over splits of partial + bias), the splits summed in order.
cudaError_t launch_splitk_finalize(const float* partial, int splits, int M, int N, const void* bias, void* y,
                                   cudaStream_t st);

// The warp-specialised kernels move registers between warpgroups with
// setmaxnreg, a split that adds up to the registers the launch gives each
// thread.  A warpgroup that asks for more than the launch holds waits forever,
// so before the first launch the host checks the count every such kernel was
// compiled to.  Each returns false and describes the first mismatch in msg.
bool gemm_register_split_ok(char* msg, size_t n);
bool prologue_register_split_ok(char* msg, size_t n);

}  // namespace qwam
