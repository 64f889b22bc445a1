// C-ABI host layer of libqwam.so: argument checks, handle lifetime, the
// per-device workspace, tensor-map construction and kernel launch order.
// Declarations and the contract of every entry point: include/qwam.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "qwam.h"

using namespace qwam;

namespace {

constexpr uint32_t kMagic = 0x514d5731u;
constexpr int kMaxDevices = 64;
// Scalars at the start of every workspace: [0] activation amax (fp32 bits),
// [4] g_x, [12] the one-pass prologue's grid-barrier count (the first 16 bytes
// are cleared before each such launch), [32] the device error word.
constexpr size_t kHeaderBytes = 256;
constexpr size_t kErrOffset = 32;

thread_local std::string g_err;

qwam_status fail(qwam_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define QW_CUDA(call)                                                                                     \
  do {                                                                                                    \
    cudaError_t e_ = (call);                                                                              \
    if (e_ != cudaSuccess) return fail(QWAM_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));   \
  } while (0)

#define QW_TRY(expr)                    \
  do {                                  \
    qwam_status s_ = (expr);            \
    if (s_ != QWAM_OK) return s_;       \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// SMs per device, looked up once (grids are sized in multiples of it)
int g_sms[kMaxDevices];
inline int sm_count(int dev) { return __atomic_load_n(&g_sms[dev], __ATOMIC_RELAXED); }

// Once per process, before any launch: every warp-specialised kernel was
// compiled to the register count its setmaxnreg split assumes.
qwam_status kernels_ready() {
  static std::once_flag once;
  static bool ok = false;
  static char msg[256];
  std::call_once(once, [] {
    ok = gemm_register_split_ok(msg, sizeof(msg)) && prologue_register_split_ok(msg, sizeof(msg));
    if (!ok) cudaGetLastError();
  });
  if (!ok) return fail(QWAM_ERR_CUDA, "%s", msg);
  return QWAM_OK;
}

qwam_status current_device(int* dev) {
  QW_CUDA(cudaGetDevice(dev));
  int major = 0;
  QW_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev));
  if (major != 10) return fail(QWAM_ERR_ARCH, "device %d is compute capability %d.x; this library is built for sm_100a", *dev, major);
  if (*dev < 0 || *dev >= kMaxDevices) return fail(QWAM_ERR_INVALID_ARG, "device index %d out of range", *dev);
  if (sm_count(*dev) <= 0) {
    int sms = 0;
    QW_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev));
    if (sms <= 0) return fail(QWAM_ERR_CUDA, "device %d reports %d SMs", *dev, sms);
    __atomic_store_n(&g_sms[*dev], sms, __ATOMIC_RELAXED);
  }
  return kernels_ready();
}

// ---- tensor maps -----------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

PFN_cuTensorMapReplaceAddress_v12000 replace_fn() {
  static PFN_cuTensorMapReplaceAddress_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapReplaceAddress", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapReplaceAddress_v12000>(p);
  });
  return fn;
}

// Point an encoded tensor map at another buffer of the same shape.
qwam_status repoint_map(CUtensorMap* m, const void* base) {
  auto fn = replace_fn();
  if (!fn) return fail(QWAM_ERR_CUDA, "cuTensorMapReplaceAddress is not available from the driver");
  CUresult r = fn(m, const_cast<void*>(base));
  if (r != CUDA_SUCCESS) return fail(QWAM_ERR_CUDA, "cuTensorMapReplaceAddress failed with code %d", static_cast<int>(r));
  return QWAM_OK;
}

qwam_status make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail(QWAM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QWAM_ERR_CUDA, "cuTensorMapEncodeTiled failed with code %d", static_cast<int>(r));
  return QWAM_OK;
}

qwam_status make_map3(CUtensorMap* m, const void* base, const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                      const cuuint32_t (&box)[3], CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail(QWAM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QWAM_ERR_CUDA, "cuTensorMapEncodeTiled failed with code %d", static_cast<int>(r));
  return QWAM_OK;
}

// The GEMM's four boxes per stage all come through 3-D maps, so one converged
// TMA instruction issues them (one box per lane).
//
// Scale buffer of `rows_padded` rows (multiple of 128) and K columns in the tiled
// layout, viewed as u8 [rows_padded / 128][K / 32][256]: a 512-byte atom (one K64
// step of 128 rows) is two 256-byte rows, so one stage of ks K elements of
// `blocks` consecutive 128-row blocks is a 256 x (ks / 32) x blocks box.
qwam_status make_sf_map(CUtensorMap* m, const void* base, size_t rows_padded, int K, int ks, int blocks) {
  const cuuint64_t dims[3] = {256, static_cast<cuuint64_t>(K / 32), static_cast<cuuint64_t>(rows_padded / 128)};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(K) * 8};
  const cuuint32_t box[3] = {256, static_cast<cuuint32_t>(ks / 32), static_cast<cuuint32_t>(blocks)};
  return make_map3(m, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// A GEMM operand [rows, row_bytes] u8 (packed E2M1, or FP8 E4M3 one byte per
// element) as the GEMM reads it (a unit third dimension): one box per stage of
// box_bytes per row (one 128B or 64B swizzle atom) by box_rows rows.
qwam_status make_codes_map(CUtensorMap* m, const void* base, int rows, int row_bytes, int box_bytes, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows), 1};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(row_bytes) * rows};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows), 1};
  return make_map3(m, base, dims, strides, box,
                   box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// Bytes of one operand row of K elements, and of one stage of ks elements.
// (FP8 E4M3 and the INT4 arm's levels as E4M3 bytes: one byte per element)
inline int code_bytes(int K, int fmt) { return fmt == 1 || fmt == 2 ? K : K / 2; }

CUtensorMapSwizzle branch_swizzle(int r) { return r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B; }

// ---- GEMM launch plan ------------------------------------------------------
struct Plan {
  int bn, ks, k_stages, splits;
  bool pair;  // 256 x bn tiles on CTA pairs (no split-K)
  bool fp8;   // FP8 operands
  bool wide;  // stages of one 128B swizzle atom per row (large M), else 64B
};

// Split-K when the output tiles leave SMs idle: the largest power of two <= 8
// (one portable cluster per tile) with splits <= k_stages and tiles * splits
// within one wave of the SMs.  Otherwise 256-column tiles run on CTA pairs.
Plan plan_gemm(int M, int N, int K, int sms, int fmt) {
  Plan p{};
  const GemmShape sh = gemm_shape(M, N, fmt == 1);
  p.fp8 = sh.fp8;
  p.wide = code_bytes(sh.ks, fmt) == 128;
  p.bn = sh.bn;
  p.ks = sh.ks;
  p.k_stages = (K + p.ks - 1) / p.ks;
  const int tiles_m = (M + 127) / 128;
  const int tiles = tiles_m * ((N + p.bn - 1) / p.bn);
  p.splits = 1;
  for (int c = 8; c >= 2; c >>= 1)
    if (c <= p.k_stages && tiles * c <= sms) {
      p.splits = c;
      break;
    }
  p.pair = sh.pair && p.splits == 1;
  return p;
}

// INT4 arm: K splits of the group GEMM when its 128 x 128 output tiles leave
// SMs idle: the largest count up to 16 with tiles * splits within one wave and
// at least one stage (K 128) per split.
int group_splits(int M, int N, int K, int sms) {
  const int tiles = ((M + 127) / 128) * ((N + 127) / 128);
  const int k_stages = K / 128;
  int s = 1;
  while (s * 2 <= 16 && s * 2 <= k_stages && tiles * s * 2 <= sms) s *= 2;
  return s;
}

// ---- per-device workspace --------------------------------------------------
struct Arena {
  uint8_t* base = nullptr;
  size_t bytes = 0;
};
std::mutex g_arena_mu;
Arena g_arena[kMaxDevices];

struct Layout {
  size_t codes, sf, u, ub, part, total;
};

// part_bytes: the INT4 arm's split-K partial tiles (0 otherwise).  Its
// activation scales are fp32 [K / 64][round_up(M, 128)], the same bytes as the
// NVFP4 tiles.
Layout layout_for(int M, int K, int r, int fmt, size_t part_bytes = 0) {
  Layout L{};
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + std::max<size_t>(bytes, 16), 256);
    return o;
  };
  const size_t Mp = round_up(static_cast<size_t>(M), 128);
  const size_t rr = static_cast<size_t>(std::max(r, 1));
  L.codes = take(Mp * code_bytes(K, fmt));
  L.sf = take(fmt == 1 ? 16 : Mp * K / 16);  // FP8: no block scales
  L.u = take(static_cast<size_t>(M) * rr * 4);
  L.ub = take(Mp * rr * 2);
  L.part = take(part_bytes);
  L.total = off;
  return L;
}

uint32_t* arena_amax(const Arena& a) { return reinterpret_cast<uint32_t*>(a.base); }
float* arena_gx(const Arena& a) { return reinterpret_cast<float*>(a.base + 4); }
uint32_t* arena_err(const Arena& a) { return reinterpret_cast<uint32_t*>(a.base + kErrOffset); }

qwam_status arena_get(int dev, size_t need, Arena** out) {
  std::lock_guard<std::mutex> lock(g_arena_mu);
  Arena& a = g_arena[dev];
  if (a.bytes < need) {
    if (a.base) {
      QW_CUDA(cudaDeviceSynchronize());
      QW_CUDA(cudaFree(a.base));
      a.base = nullptr;
      a.bytes = 0;
    }
    const size_t bytes = round_up(std::max(need, kHeaderBytes + (size_t(1) << 20)), size_t(1) << 20);
    if (cudaMalloc(&a.base, bytes) != cudaSuccess) {
      cudaGetLastError();
      a.base = nullptr;
      return fail(QWAM_ERR_OOM, "workspace allocation of %zu bytes failed", bytes);
    }
    QW_CUDA(cudaMemset(a.base, 0, bytes));
    QW_CUDA(cudaDeviceSynchronize());
    a.bytes = bytes;
  }
  *out = &a;
  return QWAM_OK;
}

// CTAs along K per 128-row tile of the prologue: the largest power of two
// that divides the chunk count (K / 128), is at most 8 (one portable cluster;
// 16 for a single row tile) and keeps the grid within one wave of the SMs (at
// least one part).
int cluster_parts(int K, int rows, int sms) {
  const int chunks = K / 128;
  const int tiles = (rows + 127) / 128;
  // one row tile (the 32-token layers): up to 16 CTAs (non-portable cluster
  // size; the launch falls back to 8 where the device cannot place 16)
  for (int c = tiles == 1 ? 16 : 8; c > 1; c >>= 1)
    if (chunks % c == 0 && tiles * c <= sms) return c;
  return 1;
}

// Everything the two launches of one layer call need for a given M and scratch
// area: the GEMM plan, the prologue's and the GEMM's tensor maps and
// parameters.  M == -1 marks it empty.
struct CallPlan {
  int M = -1;
  const uint8_t* ws = nullptr;  // scratch the maps and pointers refer to
  const void* x = nullptr;      // buffers the x and y maps point at (nullptr: not encoded yet)
  const void* y = nullptr;
  Plan pl{};
  int pro_form = 0;  // PRO_FUSED, PRO_TWO_PASS or PRO_WIDE
  int pro_groups = 0;
  ProMaps pmaps{};
  PrologueParams prm{};
  GemmMaps gmaps{};
  GemmParams gp{};
  GroupGemmMaps ggmaps{};  // INT4 arm
  GroupGemmParams ggp{};
};

}  // namespace

struct qwam_layer {
  uint32_t magic;
  int N, K, r, b, dev;
  int fmt;      // 0 NVFP4 (W4A4), 1 FP8 E4M3 (W8A8), 2 INT4 group 64 (the SVDQuant arm)
  int variant;  // 0 deflated, 1 shared-weight, 2 SVDQuant
  uint8_t* codes;
  uint8_t* sf;
  uint16_t* L;
  uint16_t *v_hi, *v_lo;    // V [K, r] bf16 hi/lo
  uint16_t *px_hi, *px_lo;  // P^T = (diag(1/s) H V)^T [r, K] bf16 hi/lo
  float* inv_s;
  float* inv_s_pm;  // row-pipeline form of 1/s: [K / 128][2][128], * 1/sqrt(b), then negated
  uint16_t* bias;
  uint16_t* hmat;   // bf16 [128, 128]: the H_b blocks of one 128-column chunk (+-1)
  float g_w;
  size_t sf_bytes;
  CUtensorMap map_b128_k128, map_b128_k256, map_b256_k256, map_l128, map_l256;
  CUtensorMap map_sfb_k128, map_sfb_k256_b1, map_sfb_k256_b2;  // B scales: K per stage, 128-row blocks per box
  CUtensorMap map_sgb;  // INT4: B scales fp32 [K / 64][N], box 128 columns x 2 groups
  ProMaps vmaps;  // P^T and V (hi/lo) tensor maps for the prologue; x is per call
  // Launch arguments of the last call, kept per scratch kind (0: the growable
  // workspace, 1: the static scratch of qwam_linear_noalloc) so that repeated
  // calls with the same M encode no tensor map; a new x or y buffer only
  // re-points its map.  mu orders host access to them.
  std::mutex mu;
  CallPlan call[2];
};

namespace {

void free_layer(qwam_layer* h) {
  if (!h) return;
  void* ptrs[] = {h->codes, h->sf, h->L, h->v_hi, h->v_lo, h->px_hi, h->px_lo, h->inv_s, h->inv_s_pm, h->bias, h->hmat};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  h->magic = 0;
  delete h;
}

qwam_status check_handle(qwam_handle h) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  int dev = -1;
  QW_CUDA(cudaGetDevice(&dev));
  if (dev != h->dev) return fail(QWAM_ERR_INVALID_ARG, "handle belongs to device %d, current device is %d", h->dev, dev);
  return QWAM_OK;
}

qwam_status check_layer_shape(int N, int K, int r, int b) {
  if (K <= 0 || K % 128) return fail(QWAM_ERR_SHAPE, "K=%d must be a positive multiple of 128", K);
  if (b < 1 || b > 128 || (b & (b - 1))) return fail(QWAM_ERR_SHAPE, "hadamard_block=%d must be a power of two <= 128", b);
  if (K % b) return fail(QWAM_ERR_SHAPE, "K=%d is not a multiple of hadamard_block=%d", K, b);
  if (r != 0 && r != 16 && r != 32) return fail(QWAM_ERR_SHAPE, "rank r=%d must be 0, 16 or 32", r);
  if (N < 16 || N % 16) return fail(QWAM_ERR_SHAPE, "N=%d must be a positive multiple of 16", N);
  return QWAM_OK;
}

template <typename T>
qwam_status dmalloc(T** p, size_t bytes) {
  *p = nullptr;
  if (cudaMalloc(reinterpret_cast<void**>(p), std::max<size_t>(bytes, 16)) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(QWAM_ERR_OOM, "device allocation of %zu bytes failed", bytes);
  }
  return QWAM_OK;
}

bool use_fused(int rows) { return rows <= 128; }

// Forms of the activation prologue: one launch for up to 128 rows; above that
// two launches (Stats, Quantise), with the rotation folded into the tensor-core
// operand when there is no subspace (r = 0), else the row pipeline with the
// rank-r projection and deflation.
enum { PRO_FUSED = 0, PRO_TWO_PASS = 1, PRO_WIDE = 2, PRO_ONEPASS = 3, PRO_LOCAL = 4 };
int prologue_form(int rows, int r, int K, int sms) {
  if (use_fused(rows)) return PRO_FUSED;
  if (r != 0) return PRO_TWO_PASS;
  return onepass_prologue_fits(rows, K, wide_prologue_groups(rows, K, sms), sms) ? PRO_ONEPASS : PRO_WIDE;
}

// The launches of the row pipeline: Fused (rows <= 128, when allowed), else
// Stats + Quantise.  prm.amax_glob is the activation / weight amax word.
qwam_status launch_rows(const ProMaps& maps, const PrologueParams& prm, int r, bool fused, cudaStream_t st) {
  if (fused) {
    QW_CUDA(launch_prologue(maps, prm, r, PrologueMode::Fused, st));
    return QWAM_OK;
  }
  QW_CUDA(cudaMemsetAsync(prm.amax_glob, 0, sizeof(uint32_t), st));
  QW_CUDA(launch_prologue(maps, prm, r, PrologueMode::Stats, st));
  QW_CUDA(launch_prologue(maps, prm, r, PrologueMode::Quantise, st));
  return QWAM_OK;
}

// x (or W) bf16 [rows, K] as the prologue's TMA reads it
qwam_status make_rows_map(CUtensorMap* m, const void* T, int rows, int K) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, K, rows, static_cast<uint64_t>(K) * 2, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// One pass of the row pipeline over T (the weight side at prepare).
qwam_status run_rows(const void* T, PrologueParams prm, int r, const ProMaps& vmaps, int sms, uint32_t* amax,
                     cudaStream_t st) {
  ProMaps maps = vmaps;
  QW_TRY(make_rows_map(&maps.x, T, prm.rows, prm.K));
  if (r == 0) maps.p_hi = maps.p_lo = maps.v_hi = maps.v_lo = maps.x;
  prm.amax_glob = amax;
  prm.parts = cluster_parts(prm.K, prm.rows, sms);
  prm.chunks = prm.K / 128 / prm.parts;
  // INT4 (local group scales): the one-launch form at any row count, whose
  // CUDA-core scaling gives W~ = RN(W * s) exactly (b = 1)
  return launch_rows(maps, prm, r, prm.fmt == 2, st);
}

// shared: the shared-weight arm (quantise W~ itself; L = deq(Q(W~)) V) instead
// of the deflated one (quantise W_d = W~ - (W~V)V^T; L = W~V).
// The device arrays a layer owns, sized from its shape (r = 0 keeps
// one-column placeholders for the rank-r arrays, which nothing reads).
size_t layer_code_bytes(const qwam_layer* h) { return static_cast<size_t>(h->N) * code_bytes(h->K, h->fmt); }
size_t layer_branch_bytes(const qwam_layer* h) { return static_cast<size_t>(h->N) * std::max(h->r, 1) * 2; }
size_t layer_v_bytes(const qwam_layer* h) { return static_cast<size_t>(h->K) * std::max(h->r, 1) * 2; }

// Bytes of the weight scales: NVFP4 tiles (rows padded to 256), none for FP8
// (a 16-byte placeholder), fp32 [K / 64][N] for INT4.
size_t layer_sf_bytes(int N, int K, int fmt) {
  if (fmt == 1) return 16;
  if (fmt == 2) return static_cast<size_t>(N) * K / 16;
  return round_up(static_cast<size_t>(N), 256) * K / 16;
}

qwam_status alloc_layer(qwam_layer* h, bool with_bias) {
  h->sf_bytes = layer_sf_bytes(h->N, h->K, h->fmt);
  const size_t K = static_cast<size_t>(h->K);
  QW_TRY(dmalloc(&h->codes, layer_code_bytes(h)));
  QW_TRY(dmalloc(&h->sf, h->sf_bytes));
  QW_TRY(dmalloc(&h->L, layer_branch_bytes(h)));
  QW_TRY(dmalloc(&h->v_hi, layer_v_bytes(h)));
  QW_TRY(dmalloc(&h->v_lo, layer_v_bytes(h)));
  QW_TRY(dmalloc(&h->px_hi, layer_v_bytes(h)));
  QW_TRY(dmalloc(&h->px_lo, layer_v_bytes(h)));
  QW_TRY(dmalloc(&h->inv_s, K * 4));
  QW_TRY(dmalloc(&h->inv_s_pm, K * 8));
  QW_TRY(dmalloc(&h->hmat, 128 * 128 * 2));
  if (with_bias) QW_TRY(dmalloc(&h->bias, static_cast<size_t>(h->N) * 2));
  return QWAM_OK;
}

// Everything of a layer that follows from its shape and its device addresses:
// the bf16 H_b blocks of one 128-column chunk and every tensor map the calls
// read.  A map encodes an address, not data, so this may run before the
// arrays are filled.  The H_b upload is ordered on st (a pageable source is
// staged before the call returns, so the host vector may go).
qwam_status finish_layer(qwam_layer* h, cudaStream_t st) {
  const int N = h->N, K = h->K, r = h->r, b = h->b;
  // H_b restricted to one 128-column chunk, in Sylvester order: +-1 where row and
  // column lie in the same b-block, 0 elsewhere (1/sqrt(b) is in the channel
  // vector); the B operand of the prologue's tensor-core rotation.
  std::vector<uint16_t> hm(128 * 128);
  for (int n = 0; n < 128; ++n)
    for (int k = 0; k < 128; ++k)
      hm[n * 128 + k] = (n ^ k) >= b ? 0 : ((__builtin_popcount(n & k & (b - 1)) & 1) ? 0xBF80u : 0x3F80u);
  QW_CUDA(cudaMemcpyAsync(h->hmat, hm.data(), hm.size() * 2, cudaMemcpyHostToDevice, st));
  QW_TRY(make_map(&h->vmaps.h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->hmat, 128, 128, 256, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B));
  if (r > 0) {
    QW_TRY(make_map(&h->vmaps.p_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->px_hi, K, r, static_cast<uint64_t>(K) * 2, 64,
                    r, CU_TENSOR_MAP_SWIZZLE_128B));
    QW_TRY(make_map(&h->vmaps.p_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->px_lo, K, r, static_cast<uint64_t>(K) * 2, 64,
                    r, CU_TENSOR_MAP_SWIZZLE_128B));
    QW_TRY(make_map(&h->vmaps.v_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->v_hi, r, K, r * 2, r, 128, branch_swizzle(r)));
    QW_TRY(make_map(&h->vmaps.v_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->v_lo, r, K, r * 2, r, 128, branch_swizzle(r)));
  }
  // B boxes: 64-byte rows (small M) or 128-byte rows (large M), 128 or 256 rows
  const int cb = code_bytes(K, h->fmt);
  QW_TRY(make_codes_map(&h->map_b128_k128, h->codes, N, cb, 64, 128));
  QW_TRY(make_codes_map(&h->map_b128_k256, h->codes, N, cb, 128, 128));
  QW_TRY(make_codes_map(&h->map_b256_k256, h->codes, N, cb, 128, 256));
  h->map_sgb = h->map_b128_k128;  // unread unless INT4
  if (h->fmt == 2)
    QW_TRY(make_map(&h->map_sgb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, h->sf, N, K / 64, static_cast<uint64_t>(N) * 4, 128,
                    2, CU_TENSOR_MAP_SWIZZLE_NONE));
  if (h->fmt != 0) {  // no NVFP4 block scales: the unread scale maps alias the codes map
    h->map_sfb_k128 = h->map_sfb_k256_b1 = h->map_sfb_k256_b2 = h->map_b128_k128;
  } else {
    const size_t rows = round_up(static_cast<size_t>(N), 256);
    QW_TRY(make_sf_map(&h->map_sfb_k128, h->sf, rows, K, 128, 1));
    QW_TRY(make_sf_map(&h->map_sfb_k256_b1, h->sf, rows, K, 256, 1));
    QW_TRY(make_sf_map(&h->map_sfb_k256_b2, h->sf, rows, K, 256, 2));
  }
  if (r > 0) {
    QW_TRY(make_map(&h->map_l128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->L, r, N, r * 2, r, 128, branch_swizzle(r)));
    QW_TRY(make_map(&h->map_l256, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h->L, r, N, r * 2, r, 256, branch_swizzle(r)));
  } else {
    h->map_l128 = h->map_b128_k128;
    h->map_l256 = h->map_b256_k256;
  }
  return QWAM_OK;
}

qwam_layer* new_layer(int N, int K, int r, int b, int dev, int fmt, int variant) {
  qwam_layer* h = new qwam_layer();  // value-initialised: every pointer and map zero
  h->magic = kMagic;
  h->N = N; h->K = K; h->r = r; h->b = b; h->dev = dev;
  h->fmt = fmt;
  h->variant = variant;
  return h;
}

qwam_status prepare_impl(const void* W, int N, int K, const float* s, const float* V, int r, const void* bias,
                         int b, float* wd_out, bool shared, int fmt, void* stream, qwam_handle* out) {
  if (!out) return fail(QWAM_ERR_INVALID_ARG, "out handle pointer is NULL");
  *out = nullptr;
  if (!W || !s) return fail(QWAM_ERR_INVALID_ARG, "W and s must be non-NULL");
  QW_TRY(check_layer_shape(N, K, r, b));
  if (r > 0 && !V) return fail(QWAM_ERR_INVALID_ARG, "V must be non-NULL when r > 0");
  if (!aligned16(W) || !aligned16(s) || (V && !aligned16(V)) || (bias && !aligned16(bias)) ||
      (wd_out && !aligned16(wd_out)))
    return fail(QWAM_ERR_ALIGN, "device pointers must be 16-byte aligned");
  int dev = 0;
  QW_TRY(current_device(&dev));
  cudaStream_t st = as_stream(stream);

  qwam_layer* h = new_layer(N, K, r, b, dev, fmt, fmt == 2 ? 2 : (shared ? 1 : 0));
  float* u_tmp = nullptr;
  uint32_t* scratch = nullptr;  // [0] amax, [1] err, [2] g_w (fp32)
  uint16_t *pw_hi = nullptr, *pw_lo = nullptr;  // P^T of the weight side, diag(s) H V
  float* s_pm = nullptr;                         // row-pipeline form of s for the weight pass
  auto cleanup = [&](qwam_status s) {
    if (s_pm) cudaFree(s_pm);
    if (u_tmp) cudaFree(u_tmp);
    if (scratch) cudaFree(scratch);
    if (pw_hi) cudaFree(pw_hi);
    if (pw_lo) cudaFree(pw_lo);
    free_layer(h);
    return s;
  };
  qwam_status s_;
  const size_t rr = static_cast<size_t>(std::max(r, 1));
  if ((s_ = alloc_layer(h, bias != nullptr)) != QWAM_OK || (s_ = dmalloc(&pw_hi, K * rr * 2)) != QWAM_OK ||
      (s_ = dmalloc(&pw_lo, K * rr * 2)) != QWAM_OK || (s_ = dmalloc(&s_pm, static_cast<size_t>(K) * 8)) != QWAM_OK ||
      (s_ = dmalloc(&u_tmp, static_cast<size_t>(N) * rr * 4)) != QWAM_OK || (s_ = dmalloc(&scratch, 64)) != QWAM_OK ||
      (s_ = finish_layer(h, st)) != QWAM_OK)
    return cleanup(s_);

#define QW_CUDA_CLEAN(call)                                                                                      \
  do {                                                                                                           \
    cudaError_t e_ = (call);                                                                                     \
    if (e_ != cudaSuccess) return cleanup(fail(QWAM_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_))); \
  } while (0)

  QW_CUDA_CLEAN(cudaMemsetAsync(h->sf, 0, h->sf_bytes, st));
  QW_CUDA_CLEAN(cudaMemsetAsync(scratch, 0, 64, st));
  if (bias) QW_CUDA_CLEAN(cudaMemcpyAsync(h->bias, bias, static_cast<size_t>(N) * 2, cudaMemcpyDeviceToDevice, st));
  QW_CUDA_CLEAN(launch_recip(s, h->inv_s, K, scratch + 1, st));
  const float hscale = 1.0f / std::sqrt(static_cast<float>(b));
  QW_CUDA_CLEAN(launch_chan_pm(h->inv_s, hscale, K, h->inv_s_pm, st));
  QW_CUDA_CLEAN(launch_chan_pm(s, hscale, K, s_pm, st));
  ProMaps wmaps{};  // the weight pass uses P of the weight side
  wmaps.h = h->vmaps.h;
  if (r > 0) {
    QW_CUDA_CLEAN(launch_split_v(V, K, r, h->v_hi, h->v_lo, st));
    QW_CUDA_CLEAN(launch_make_proj(V, s, K, r, b, pw_hi, pw_lo, st));
    QW_CUDA_CLEAN(launch_make_proj(V, h->inv_s, K, r, b, h->px_hi, h->px_lo, st));
    wmaps = h->vmaps;
    auto pmap = [&](CUtensorMap* m, const uint16_t* base) {
      return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, K, r, static_cast<uint64_t>(K) * 2, 64, r,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    };
    if ((s_ = pmap(&wmaps.p_hi, pw_hi)) != QWAM_OK || (s_ = pmap(&wmaps.p_lo, pw_lo)) != QWAM_OK) return cleanup(s_);
  }
  PrologueParams prm{};
  prm.chan = s_pm;
  prm.rows = N;
  prm.K = K;
  prm.b = b;
  prm.hscale = hscale;
  prm.u_glob = u_tmp;
  prm.codes = h->codes;
  prm.sf = h->sf;
  prm.branch = h->L;
  prm.branch_mode = 0;
  prm.g_other = 1.0f;
  prm.g_out = reinterpret_cast<float*>(scratch + 2);
  prm.z_out = wd_out;
  prm.err = scratch + 3;
  prm.fmt = fmt;
  prm.sf_pitch = N;  // INT4 weight scales [K / 64][N]
  if (shared && r > 0) {
    // W~ itself through the row pipeline (no projection, no deflation), then
    // the branch weight from the stored FP4 weight
    ProMaps w0{};
    w0.h = h->vmaps.h;
    if ((s_ = run_rows(W, prm, 0, w0, sm_count(dev), scratch, st)) != QWAM_OK) return cleanup(s_);
    QW_CUDA_CLEAN(launch_dequant_project(h->codes, h->sf, prm.g_out, V, N, K, r, h->L, st));
  } else {
    if ((s_ = run_rows(W, prm, r, wmaps, sm_count(dev), scratch, st)) != QWAM_OK) return cleanup(s_);
  }
  uint32_t host_scr[4] = {0, 0, 0, 0};
  QW_CUDA_CLEAN(cudaMemcpyAsync(host_scr, scratch, 16, cudaMemcpyDeviceToHost, st));
  QW_CUDA_CLEAN(cudaStreamSynchronize(st));
  if (host_scr[1]) return cleanup(fail(QWAM_ERR_INVALID_ARG, "smoothing vector s has an entry that is <= 0 or not finite"));
  if (host_scr[3]) return cleanup(fail(QWAM_ERR_TIMEOUT, "a bounded device wait expired in prepare (flags 0x%x)", host_scr[3]));
  std::memcpy(&h->g_w, &host_scr[2], 4);
  if (fmt == 2) h->g_w = 1.0f;  // INT4: every scale is a group scale

  cudaFree(s_pm);
  cudaFree(u_tmp);
  cudaFree(scratch);
  cudaFree(pw_hi);
  cudaFree(pw_lo);
#undef QW_CUDA_CLEAN
  *out = h;
  return QWAM_OK;
}

qwam_status check_linear_args(const void* x, int M, qwam_handle h) {
  QW_TRY(check_handle(h));
  if (M < 0) return fail(QWAM_ERR_SHAPE, "M=%d must be >= 0", M);
  if (M > (1 << 24)) return fail(QWAM_ERR_SHAPE, "M=%d exceeds the supported maximum of 2^24", M);
  if (M > 0 && !x) return fail(QWAM_ERR_INVALID_ARG, "x is NULL");
  if (x && !aligned16(x)) return fail(QWAM_ERR_ALIGN, "x must be 16-byte aligned");
  return QWAM_OK;
}

// y [M, N] bf16 for the TMA store of the bf16 epilogue: 128-row boxes of 64
// columns (128B swizzle), or of 32 columns (64B swizzle) on CTA pairs (a
// 16 KB staging area; a fifth operand stage in the room this frees measured
// slower than four).
qwam_status make_y_map(CUtensorMap* m, const void* y, int N, int M, bool pair) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, N, M, static_cast<uint64_t>(N) * 2, pair ? 32 : 64, 128,
                  pair ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// The workspace layout of an M-row call of layer h.
Layout layout_of(const qwam_layer* h, int M) {
  size_t part = 0;
  if (h->fmt == 2) {
    const int sp = group_splits(std::max(M, 1), h->N, h->K, sm_count(h->dev));
    if (sp > 1) part = static_cast<size_t>(sp) * M * h->N * 4;
  }
  return layout_for(M, h->K, h->r, h->fmt, part);
}

// Launch arguments for M rows of layer h with scratch at ws: the workspace
// layout of layout_of (scalars at ws: amax, g_x, error word).
qwam_status build_call(qwam_handle h, int M, uint8_t* ws, CallPlan* c) {
  c->M = -1;
  const int sms = sm_count(h->dev);
  const Plan pl = plan_gemm(M, h->N, h->K, sms, h->fmt);
  const Layout lay = layout_of(h, M);
  PrologueParams prm{};
  prm.chan = h->inv_s_pm;
  prm.rows = M;
  prm.K = h->K;
  prm.b = h->b;
  prm.hscale = 1.0f / std::sqrt(static_cast<float>(h->b));
  prm.u_glob = reinterpret_cast<float*>(ws + lay.u);
  prm.amax_glob = reinterpret_cast<uint32_t*>(ws);
  prm.codes = ws + lay.codes;
  prm.sf = ws + lay.sf;
  prm.branch = reinterpret_cast<uint16_t*>(ws + lay.ub);
  prm.branch_mode = 1;
  prm.g_other = h->g_w;
  prm.g_out = reinterpret_cast<float*>(ws + 4);
  prm.err = reinterpret_cast<uint32_t*>(ws + kErrOffset);
  prm.parts = cluster_parts(h->K, M, sms);
  prm.chunks = h->K / 128 / prm.parts;
  prm.fmt = h->fmt;

  if (h->fmt == 2) {
    // SVDQuant arm: the Local prologue (b = 1, INT4 quantised as read, bf16(c)
    // for the branch) and the group GEMM (+ the split-K sum)
    const int Mp = static_cast<int>(round_up(static_cast<size_t>(M), 128));
    prm.branch_mode = 0;
    prm.sf_pitch = Mp;
    GroupGemmMaps gg{};
    QW_TRY(make_codes_map(&gg.a, ws + lay.codes, M, h->K, 128, 128));
    gg.b = h->map_b128_k256;
    QW_TRY(make_map(&gg.sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, ws + lay.sf, M, h->K / 64, static_cast<uint64_t>(Mp) * 4,
                    128, 2, CU_TENSOR_MAP_SWIZZLE_NONE));
    gg.sb = h->map_sgb;
    if (h->r > 0) {
      QW_TRY(make_map(&gg.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + lay.ub, h->r, M, h->r * 2, h->r, 128,
                      branch_swizzle(h->r)));
      gg.l = h->map_l128;
    } else {
      gg.u = gg.sa;  // unread
      gg.l = gg.sb;
    }
    GroupGemmParams gq{};
    gq.M = M; gq.N = h->N; gq.K = h->K;
    gq.splits = group_splits(M, h->N, h->K, sms);
    gq.branch_k = h->r;
    gq.bias = h->bias;
    gq.partial = gq.splits > 1 ? reinterpret_cast<float*>(ws + lay.part) : nullptr;
    gq.err = prm.err;
    c->pl = pl;
    c->pro_form = PRO_LOCAL;
    c->pro_groups = 0;
    c->pmaps = h->vmaps;
    c->prm = prm;
    c->ggmaps = gg;
    c->ggp = gq;
    c->x = c->y = nullptr;
    c->ws = ws;
    c->M = M;
    return QWAM_OK;
  }

  GemmMaps gm{};
  QW_TRY(make_codes_map(&gm.a, ws + lay.codes, M, code_bytes(h->K, h->fmt), pl.wide ? 128 : 64, 128));
  gm.b = pl.bn == 256 && !pl.pair ? h->map_b256_k256 : (pl.wide ? h->map_b128_k256 : h->map_b128_k128);
  if (h->fmt == 1) {  // FP8: no block scales (the unread maps alias the operands)
    gm.sfa = gm.a;
    gm.sfb = gm.b;
  } else {
    QW_TRY(make_sf_map(&gm.sfa, ws + lay.sf, round_up(static_cast<size_t>(M), 128), h->K, pl.ks, 1));
    gm.sfb = !pl.wide ? h->map_sfb_k128 : (pl.bn == 256 ? h->map_sfb_k256_b2 : h->map_sfb_k256_b1);
  }
  if (h->r > 0) {
    QW_TRY(make_map(&gm.u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ws + lay.ub, h->r, M, h->r * 2, h->r, 128,
                    branch_swizzle(h->r)));
    gm.l = pl.bn == 256 && !pl.pair ? h->map_l256 : h->map_l128;
  } else {
    gm.u = gm.a;
    gm.l = gm.b;
  }
  gm.y = gm.a;  // split-K writes y with plain stores; otherwise encoded by bind_y
  GemmParams gp{};
  gp.M = M; gp.N = h->N; gp.K = h->K;
  gp.k_stages = pl.k_stages;
  gp.splits = pl.splits;
  gp.sfa = ws + lay.sf;
  gp.sfb = h->sf;
  gp.g_a_ptr = prm.g_out;
  gp.g_b = h->g_w;
  gp.has_branch = h->r > 0;
  gp.branch_k = h->r;
  gp.bias = h->bias;
  gp.err = prm.err;
  gp.sms = sms;

  c->pl = pl;
  c->pro_form = prologue_form(M, h->r, h->K, sms);
  c->pro_groups = wide_prologue_groups(M, h->K, sms);
  c->pmaps = h->vmaps;
  c->prm = prm;
  c->gmaps = gm;
  c->gp = gp;
  c->x = c->y = nullptr;
  c->ws = ws;
  c->M = M;
  return QWAM_OK;
}

// The cached arguments for (M, ws), rebuilt when either changed.
qwam_status call_for(qwam_handle h, int M, uint8_t* ws, CallPlan* c) {
  if (c->M == M && c->ws == ws) return QWAM_OK;
  return build_call(h, M, ws, c);
}

qwam_status bind_x(qwam_handle h, CallPlan* c, const void* x) {
  if (x == c->x) return QWAM_OK;
  if (c->x) {
    QW_TRY(repoint_map(&c->pmaps.x, x));
  } else {
    QW_TRY(make_rows_map(&c->pmaps.x, x, c->M, h->K));
    if (h->r == 0) c->pmaps.p_hi = c->pmaps.p_lo = c->pmaps.v_hi = c->pmaps.v_lo = c->pmaps.x;  // unread
  }
  c->x = x;
  return QWAM_OK;
}

qwam_status bind_y(qwam_handle h, CallPlan* c, void* y) {
  if (h->fmt == 2) {  // plain stores; with split K the final sum writes y
    c->ggp.y = c->ggp.splits == 1 ? y : nullptr;
    c->y = y;
    return QWAM_OK;
  }
  c->gp.y = y;
  if (y == c->y || c->pl.splits > 1) {
    c->y = y;
    return QWAM_OK;
  }
  if (c->y) QW_TRY(repoint_map(&c->gmaps.y, y));
  else QW_TRY(make_y_map(&c->gmaps.y, y, h->N, c->M, c->pl.pair));
  c->y = y;
  return QWAM_OK;
}

qwam_status launch_call_prologue(const CallPlan& c, const PrologueParams& prm, int r, cudaStream_t st) {
  if (c.pro_form == PRO_LOCAL) {
    QW_CUDA(launch_prologue(c.pmaps, prm, r, PrologueMode::Local, st));
    return QWAM_OK;
  }
  if (c.pro_form == PRO_ONEPASS) {
    QW_CUDA(cudaMemsetAsync(prm.amax_glob, 0, 16, st));  // amax, g_x, grid-barrier count
    QW_CUDA(launch_prologue_onepass(c.pmaps.x, prm, c.pro_groups, st));
    return QWAM_OK;
  }
  if (c.pro_form == PRO_WIDE) {
    QW_CUDA(cudaMemsetAsync(prm.amax_glob, 0, sizeof(uint32_t), st));
    QW_CUDA(launch_prologue_wide(c.pmaps.x, prm, PrologueMode::Stats, c.pro_groups, st));
    QW_CUDA(launch_prologue_wide(c.pmaps.x, prm, PrologueMode::Quantise, c.pro_groups, st));
    return QWAM_OK;
  }
  return launch_rows(c.pmaps, prm, r, c.pro_form == PRO_FUSED, st);
}

qwam_status launch_call_gemm(const CallPlan& c, cudaStream_t st) {
  if (c.pro_form == PRO_LOCAL) {
    QW_CUDA(launch_group_gemm(c.ggmaps, c.ggp, st));
    if (c.ggp.splits > 1)
      QW_CUDA(launch_splitk_finalize(c.ggp.partial, c.ggp.splits, c.M, c.ggp.N, c.ggp.bias, const_cast<void*>(c.y), st));
    return QWAM_OK;
  }
  QW_CUDA(launch_gemm(c.gmaps, c.gp, GemmShape{c.pl.bn, c.pl.ks, c.pl.pair, c.pl.fp8},
                      c.pl.splits > 1 ? GemmEpilogue::SplitK : GemmEpilogue::Bf16, st));
  return QWAM_OK;
}

// The workspace arena of the handle's device, grown to hold M rows.
qwam_status workspace_for(qwam_handle h, int M, Arena** a) {
  return arena_get(h->dev, layout_of(h, M).total, a);
}

// ---------------------------------------------------------------------------
// Layer images: a prepared layer as one host byte string.  A 64-byte header
// (little-endian), then the arrays the calls read, each padded to 16 bytes:
// codes, block scales (NVFP4 and INT4), L, V hi/lo and P^T hi/lo (r > 0 only),
// 1/s, bias (when present).  INT4 levels are stored 4-bit (two's complement,
// two per byte, the even element in the low nibble) and their scales as
// fp16, as the checkpoint format keeps them; the device holds E4M3 bytes and
// fp32.  What follows from these (the row-pipeline form of
// 1/s, the H_b blocks and every tensor map) is rebuilt on load.  The checksum
// is FNV-1a 64 (Fowler, Noll and Vo) over the whole image with its own field
// taken as zero.
constexpr char kImageMagic[8] = {'Q', 'W', 'A', 'M', 'I', 'M', 'G', '\0'};
constexpr uint32_t kImageVersion = 1;

struct ImageHeader {
  char magic[8];
  uint32_t version, header_bytes;
  int32_t N, K, r, b, fmt, variant;
  uint32_t flags;  // bit 0: bias present
  float g_w;
  uint64_t total_bytes, checksum;
};
static_assert(sizeof(ImageHeader) == 64, "image header is 64 bytes");

struct ImageSection {
  void* dev;
  size_t bytes;  // in the image
  int kind;      // 0 as on the device; 1 INT4 levels (packed 4-bit); 2 INT4 scales (fp16)
};

// E4M3 byte of an INT4 level (-8..7, all exact in E4M3) and back.
uint8_t e4m3_of_level(int v) {
  if (v == 0) return 0;
  const int a = v < 0 ? -v : v;
  int e = 0;
  while ((a >> (e + 1)) != 0) ++e;
  const int m = ((a << 3) >> e) & 7;  // three mantissa bits of a / 2^e
  return static_cast<uint8_t>((v < 0 ? 0x80 : 0) | ((e + 7) << 3) | m);
}
bool level_of_e4m3(uint8_t b, int* v) {
  // byte -> level + 8 (0..15), or -1 for a byte that is no level
  static const std::vector<int8_t> lut = [] {
    std::vector<int8_t> t(256, -1);
    for (int l = -8; l <= 7; ++l) t[e4m3_of_level(l)] = static_cast<int8_t>(l + 8);
    t[0x80] = 8;  // -0
    return t;
  }();
  if (lut[b] < 0) return false;
  *v = lut[b] - 8;
  return true;
}
// fp16 bits of an fp32 value that fp16 holds exactly (false otherwise), and back.
bool half_bits_exact(float f, uint16_t* out) {
  if (!(f >= 0.0f) || f > 65504.0f) return false;
  if (f == 0.0f) {
    *out = 0;
    return true;
  }
  int ex = 0;
  std::frexp(f, &ex);  // f = fr 2^ex, fr in [0.5, 1)
  const int e = ex - 1;
  const double q = e >= -14 ? std::ldexp(static_cast<double>(f), 10 - e) - 1024.0 : std::ldexp(static_cast<double>(f), 24);
  if (q != std::floor(q) || q < 0 || q > 1023) return false;
  *out = static_cast<uint16_t>(e >= -14 ? ((e + 15) << 10) | static_cast<int>(q) : static_cast<int>(q));
  return true;
}
float float_of_half_bits(uint16_t hb) {
  const int e = (hb >> 10) & 31, m = hb & 1023;
  const float v = e == 0 ? std::ldexp(static_cast<float>(m), -24) : std::ldexp(static_cast<float>(1024 + m), e - 25);
  return (hb & 0x8000) ? -v : v;
}

size_t pad16(size_t n) { return (n + 15) & ~static_cast<size_t>(15); }

// The sections of a layer in image order; returns their count (at most 9).
int image_sections(const qwam_layer* h, bool with_bias, ImageSection* out) {
  int n = 0;
  if (h->fmt == 2) {
    out[n++] = {h->codes, layer_code_bytes(h) / 2, 1};
    out[n++] = {h->sf, h->sf_bytes / 2, 2};
  } else {
    out[n++] = {h->codes, layer_code_bytes(h), 0};
    if (h->fmt == 0) out[n++] = {h->sf, h->sf_bytes, 0};
  }
  if (h->r > 0) {
    const size_t vb = static_cast<size_t>(h->K) * h->r * 2;
    out[n++] = {h->L, static_cast<size_t>(h->N) * h->r * 2, 0};
    out[n++] = {h->v_hi, vb, 0};
    out[n++] = {h->v_lo, vb, 0};
    out[n++] = {h->px_hi, vb, 0};
    out[n++] = {h->px_lo, vb, 0};
  }
  out[n++] = {h->inv_s, static_cast<size_t>(h->K) * 4, 0};
  if (with_bias) out[n++] = {h->bias, static_cast<size_t>(h->N) * 2, 0};
  return n;
}

size_t image_bytes(const qwam_layer* h, bool with_bias) {
  ImageSection sec[9];
  const int n = image_sections(h, with_bias, sec);
  size_t total = sizeof(ImageHeader);
  for (int i = 0; i < n; ++i) total += pad16(sec[i].bytes);
  return total;
}

uint64_t fnv1a64(const uint8_t* p, size_t n, uint64_t h = 0xcbf29ce484222325ull) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 0x100000001b3ull;
  }
  return h;
}

uint64_t image_checksum(const uint8_t* img, size_t total) {
  ImageHeader hd;
  std::memcpy(&hd, img, sizeof hd);
  hd.checksum = 0;
  const uint64_t h = fnv1a64(reinterpret_cast<const uint8_t*>(&hd), sizeof hd);
  return fnv1a64(img + sizeof hd, total - sizeof hd, h);
}


}  // namespace

// ---- allocation-free variant of the layer call -----------------------------
// Some callers must not allocate device memory once they are running: a
// fixed-rate control loop (a cudaMalloc can synchronise the whole device and
// stall for milliseconds) and processes whose device memory is budgeted at
// start-up.  qwam_linear_noalloc serves them from this fixed scratch area,
// compiled into the library, instead of the growable per-device workspace.
// It holds the same layout as that workspace (scalars, then activation codes,
// scales, u and u') for up to 128 rows and K <= 16384; for such calls the
// layout needs at most 1.2 MB.
constexpr int kStaticMaxRows = 128;
constexpr int kStaticMaxK = 16384;
constexpr size_t kStaticBytes = size_t(2) << 20;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticBytes];

namespace {

std::mutex g_static_mu;
uint8_t* g_static_base[kMaxDevices];  // this device's address of g_static_scratch, once set up

// Set-up, once per device, with that device current: look up the device
// address of the scratch and clear its header (the device error word must
// start at zero; the other scalars are written before they are read).  The
// clearing runs on the legacy stream and synchronises the device, which a
// stream capture cannot hold: a first call whose stream is being captured is
// refused.
qwam_status static_scratch(int dev, cudaStream_t st, uint8_t** out) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_base[dev]) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    QW_CUDA(cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone)
      return fail(QWAM_ERR_INVALID_ARG,
                  "the first qwam_linear_noalloc call on a device sets up its scratch and must not be stream-captured");
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return fail(QWAM_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    }
    QW_CUDA(cudaMemset(p, 0, kHeaderBytes));
    QW_CUDA(cudaDeviceSynchronize());
    g_static_base[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_static_base[dev];
  return QWAM_OK;
}

// The same two launches as qwam_linear (fused prologue, then the GEMM with
// the same plan), with every workspace pointer inside the static scratch.
qwam_status linear_noalloc_impl(const void* x, int M, qwam_handle h, void* y, cudaStream_t st) {
  if (M > kStaticMaxRows)
    return fail(QWAM_ERR_SHAPE, "qwam_linear_noalloc takes at most %d rows, got M=%d", kStaticMaxRows, M);
  if (h->K > kStaticMaxK)
    return fail(QWAM_ERR_SHAPE, "qwam_linear_noalloc takes K <= %d, this layer has K=%d", kStaticMaxK, h->K);
  const Layout lay = layout_of(h, M);
  if (lay.total > kStaticBytes)
    return fail(QWAM_ERR_SHAPE, "qwam_linear_noalloc needs %zu bytes of scratch, the static scratch holds %zu",
                lay.total, kStaticBytes);
  uint8_t* base = nullptr;
  QW_TRY(static_scratch(h->dev, st, &base));
  std::lock_guard<std::mutex> lock(h->mu);
  CallPlan& c = h->call[1];
  QW_TRY(call_for(h, M, base, &c));
  QW_TRY(bind_x(h, &c, x));
  QW_TRY(bind_y(h, &c, y));
  QW_TRY(launch_call_prologue(c, c.prm, h->r, st));
  return launch_call_gemm(c, st);
}

}  // namespace

extern "C" {

qwam_status qwam_prepare_weight(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                const void* bias_bf16, int hadamard_block, void* stream, qwam_handle* out) {
  return prepare_impl(W_bf16, N, K, s, V, r, bias_bf16, hadamard_block, nullptr, false, 0, stream, out);
}

qwam_status qwam_prepare_weight_shared(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                       const void* bias_bf16, int hadamard_block, float* Wt_f32, void* stream,
                                       qwam_handle* out) {
  return prepare_impl(W_bf16, N, K, s, V, r, bias_bf16, hadamard_block, Wt_f32, true, 0, stream, out);
}

qwam_status qwam_prepare_weight_fp8(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                    const void* bias_bf16, int hadamard_block, float* Wd_f32, void* stream,
                                    qwam_handle* out) {
  return prepare_impl(W_bf16, N, K, s, V, r, bias_bf16, hadamard_block, Wd_f32, false, 1, stream, out);
}

qwam_status qwam_prepare_weight_int4(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                     const void* bias_bf16, float* Wd_f32, void* stream, qwam_handle* out) {
  return prepare_impl(W_bf16, N, K, s, V, r, bias_bf16, 1, Wd_f32, false, 2, stream, out);
}

qwam_status qwam_int4_gemm(const void* a_levels, const float* a_scales, const void* b_levels, const float* b_scales,
                           int M, int N, int K, float* out_f32, void* stream) {
  if (!a_levels || !a_scales || !b_levels || !b_scales || !out_f32) return fail(QWAM_ERR_INVALID_ARG, "NULL argument");
  if (M < 4 || M % 4 || N < 16 || N % 16 || K < 128 || K % 128)
    return fail(QWAM_ERR_SHAPE, "M a positive multiple of 4, N of 16 and K of 128 required (M=%d N=%d K=%d)", M, N, K);
  if (!aligned16(a_levels) || !aligned16(a_scales) || !aligned16(b_levels) || !aligned16(b_scales) || !aligned16(out_f32))
    return fail(QWAM_ERR_ALIGN, "device pointers must be 16-byte aligned");
  int dev = 0;
  QW_TRY(current_device(&dev));
  Arena* ar = nullptr;
  QW_TRY(arena_get(dev, kHeaderBytes, &ar));
  GroupGemmMaps m{};
  QW_TRY(make_codes_map(&m.a, a_levels, M, K, 128, 128));
  QW_TRY(make_codes_map(&m.b, b_levels, N, K, 128, 128));
  QW_TRY(make_map(&m.sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a_scales, M, K / 64, static_cast<uint64_t>(M) * 4, 128, 2,
                  CU_TENSOR_MAP_SWIZZLE_NONE));
  QW_TRY(make_map(&m.sb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, b_scales, N, K / 64, static_cast<uint64_t>(N) * 4, 128, 2,
                  CU_TENSOR_MAP_SWIZZLE_NONE));
  m.u = m.sa;  // no branch: unread
  m.l = m.sb;
  GroupGemmParams p{};
  p.M = M; p.N = N; p.K = K;
  p.splits = 1;
  p.partial = out_f32;
  p.err = arena_err(*ar);
  QW_CUDA(launch_group_gemm(m, p, as_stream(stream)));
  return QWAM_OK;
}

qwam_status qwam_handle_format(qwam_handle h, int* fmt, int* variant) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  if (fmt) *fmt = h->fmt;
  if (variant) *variant = h->variant;
  return QWAM_OK;
}

qwam_status qwam_image_size(qwam_handle h, size_t* bytes) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  if (!bytes) return fail(QWAM_ERR_INVALID_ARG, "bytes pointer is NULL");
  *bytes = image_bytes(h, h->bias != nullptr);
  return QWAM_OK;
}

qwam_status qwam_save_image(qwam_handle h, void* host_buf, size_t buf_bytes, void* stream) {
  QW_TRY(check_handle(h));
  if (!host_buf) return fail(QWAM_ERR_INVALID_ARG, "host buffer is NULL");
  const bool with_bias = h->bias != nullptr;
  const size_t total = image_bytes(h, with_bias);
  if (buf_bytes < total) return fail(QWAM_ERR_INVALID_ARG, "host buffer holds %zu bytes, the image needs %zu", buf_bytes, total);
  uint8_t* img = static_cast<uint8_t*>(host_buf);
  cudaStream_t st = as_stream(stream);
  std::memset(img, 0, total);
  ImageSection sec[9];
  const int n = image_sections(h, with_bias, sec);
  size_t off = sizeof(ImageHeader);
  std::vector<uint8_t> tmp[2];  // INT4 levels and scales as the device holds them
  for (int i = 0; i < n; ++i) {
    if (sec[i].kind == 0) {
      QW_CUDA(cudaMemcpyAsync(img + off, sec[i].dev, sec[i].bytes, cudaMemcpyDeviceToHost, st));
    } else {
      std::vector<uint8_t>& v = tmp[sec[i].kind - 1];
      v.resize(2 * sec[i].bytes);
      QW_CUDA(cudaMemcpyAsync(v.data(), sec[i].dev, v.size(), cudaMemcpyDeviceToHost, st));
    }
    off += pad16(sec[i].bytes);
  }
  QW_CUDA(cudaStreamSynchronize(st));
  off = sizeof(ImageHeader);
  for (int i = 0; i < n; ++i) {
    uint8_t* dst = img + off;
    if (sec[i].kind == 1) {
      const std::vector<uint8_t>& v = tmp[0];
      for (size_t j = 0; j < sec[i].bytes; ++j) {
        int lo = 0, hi = 0;
        if (!level_of_e4m3(v[2 * j], &lo) || !level_of_e4m3(v[2 * j + 1], &hi))
          return fail(QWAM_ERR_FORMAT, "the handle holds a code that is no INT4 level");
        dst[j] = static_cast<uint8_t>((lo & 15) | ((hi & 15) << 4));
      }
    } else if (sec[i].kind == 2) {
      const float* f = reinterpret_cast<const float*>(tmp[1].data());
      for (size_t j = 0; j < sec[i].bytes / 2; ++j) {
        uint16_t hb = 0;
        if (!half_bits_exact(f[j], &hb)) return fail(QWAM_ERR_FORMAT, "the handle holds a scale that is no fp16 value");
        std::memcpy(dst + 2 * j, &hb, 2);
      }
    }
    off += pad16(sec[i].bytes);
  }
  ImageHeader hd{};
  std::memcpy(hd.magic, kImageMagic, 8);
  hd.version = kImageVersion;
  hd.header_bytes = sizeof(ImageHeader);
  hd.N = h->N; hd.K = h->K; hd.r = h->r; hd.b = h->b;
  hd.fmt = h->fmt;
  hd.variant = h->variant;
  hd.flags = with_bias ? 1u : 0u;
  hd.g_w = h->g_w;
  hd.total_bytes = total;
  std::memcpy(img, &hd, sizeof hd);
  hd.checksum = image_checksum(img, total);
  std::memcpy(img, &hd, sizeof hd);
  return QWAM_OK;
}

qwam_status qwam_load_image(const void* host_buf, size_t buf_bytes, void* stream, qwam_handle* out) {
  if (!out) return fail(QWAM_ERR_INVALID_ARG, "out handle pointer is NULL");
  *out = nullptr;
  if (!host_buf) return fail(QWAM_ERR_INVALID_ARG, "host buffer is NULL");
  const uint8_t* img = static_cast<const uint8_t*>(host_buf);
  ImageHeader hd;
  if (buf_bytes < sizeof hd) return fail(QWAM_ERR_FORMAT, "image of %zu bytes is shorter than its header", buf_bytes);
  std::memcpy(&hd, img, sizeof hd);
  if (std::memcmp(hd.magic, kImageMagic, 8) != 0) return fail(QWAM_ERR_FORMAT, "not a layer image (bad magic)");
  if (hd.version != kImageVersion || hd.header_bytes != sizeof hd)
    return fail(QWAM_ERR_FORMAT, "image version %u / header %u bytes is not %u / %zu", hd.version, hd.header_bytes,
                kImageVersion, sizeof hd);
  if (check_layer_shape(hd.N, hd.K, hd.r, hd.b) != QWAM_OK)
    return fail(QWAM_ERR_FORMAT, "image shape N=%d K=%d r=%d b=%d is not a valid layer", hd.N, hd.K, hd.r, hd.b);
  if (hd.fmt < 0 || hd.fmt > 2 || hd.variant < 0 || hd.variant > 2 || (hd.fmt == 1 && hd.variant != 0) ||
      ((hd.fmt == 2) != (hd.variant == 2)) || (hd.fmt == 2 && hd.b != 1) || (hd.flags & ~1u) ||
      !(std::isfinite(hd.g_w) && hd.g_w > 0.0f))
    return fail(QWAM_ERR_FORMAT, "image header fields are out of range (fmt %d, variant %d, flags 0x%x)", hd.fmt,
                hd.variant, hd.flags);
  qwam_layer shape{};
  shape.N = hd.N; shape.K = hd.K; shape.r = hd.r; shape.fmt = hd.fmt;
  shape.sf_bytes = layer_sf_bytes(hd.N, hd.K, hd.fmt);
  const bool with_bias = hd.flags & 1u;
  const size_t total = image_bytes(&shape, with_bias);
  if (hd.total_bytes != total || buf_bytes < total)
    return fail(QWAM_ERR_FORMAT, "image says %llu bytes, its shape needs %zu, the buffer holds %zu",
                static_cast<unsigned long long>(hd.total_bytes), total, buf_bytes);
  if (image_checksum(img, total) != hd.checksum) return fail(QWAM_ERR_FORMAT, "image checksum does not match");

  int dev = 0;
  QW_TRY(current_device(&dev));
  cudaStream_t st = as_stream(stream);
  qwam_layer* h = new_layer(hd.N, hd.K, hd.r, hd.b, dev, hd.fmt, hd.variant);
  h->g_w = hd.g_w;
  auto cleanup = [&](qwam_status s) {
    free_layer(h);
    return s;
  };
  qwam_status s_;
  if ((s_ = alloc_layer(h, with_bias)) != QWAM_OK || (s_ = finish_layer(h, st)) != QWAM_OK) return cleanup(s_);
  ImageSection sec[9];
  const int n = image_sections(h, with_bias, sec);
  size_t off = sizeof(ImageHeader);
  cudaError_t e = cudaSuccess;
  if (hd.fmt == 1) e = cudaMemsetAsync(h->sf, 0, h->sf_bytes, st);
  std::vector<uint8_t> tmp[2];  // INT4 levels and scales in the device's form
  for (int i = 0; i < n && e == cudaSuccess; ++i) {
    const uint8_t* src = img + off;
    if (sec[i].kind == 0) {
      e = cudaMemcpyAsync(sec[i].dev, src, sec[i].bytes, cudaMemcpyHostToDevice, st);
    } else {
      std::vector<uint8_t>& v = tmp[sec[i].kind - 1];
      v.resize(2 * sec[i].bytes);
      if (sec[i].kind == 1) {
        for (size_t j = 0; j < sec[i].bytes; ++j) {
          const int lo = src[j] & 15, hi = src[j] >> 4;
          v[2 * j] = e4m3_of_level(lo >= 8 ? lo - 16 : lo);
          v[2 * j + 1] = e4m3_of_level(hi >= 8 ? hi - 16 : hi);
        }
      } else {
        float* f = reinterpret_cast<float*>(v.data());
        for (size_t j = 0; j < sec[i].bytes / 2; ++j) {
          uint16_t hb;
          std::memcpy(&hb, src + 2 * j, 2);
          f[j] = float_of_half_bits(hb);
        }
      }
      e = cudaMemcpyAsync(sec[i].dev, v.data(), v.size(), cudaMemcpyHostToDevice, st);
    }
    off += pad16(sec[i].bytes);
  }
  if (e == cudaSuccess) e = launch_chan_pm(h->inv_s, 1.0f / std::sqrt(static_cast<float>(hd.b)), hd.K, h->inv_s_pm, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cleanup(fail(QWAM_ERR_CUDA, "loading the image failed: %s", cudaGetErrorString(e)));
  *out = h;
  return QWAM_OK;
}

qwam_status qwam_debug_prepare_weight(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                      const void* bias_bf16, int hadamard_block, float* Wd_f32, void* stream,
                                      qwam_handle* out) {
  return prepare_impl(W_bf16, N, K, s, V, r, bias_bf16, hadamard_block, Wd_f32, false, 0, stream, out);
}

qwam_status qwam_destroy(qwam_handle h) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  int prev = -1;
  QW_CUDA(cudaGetDevice(&prev));
  if (prev != h->dev) QW_CUDA(cudaSetDevice(h->dev));
  QW_CUDA(cudaDeviceSynchronize());
  free_layer(h);
  if (prev != -1) cudaSetDevice(prev);
  return QWAM_OK;
}

qwam_status qwam_prologue(const void* x_bf16, int M, qwam_handle h, void* stream) {
  QW_TRY(check_linear_args(x_bf16, M, h));
  if (M == 0) return QWAM_OK;
  Arena* a = nullptr;
  QW_TRY(workspace_for(h, M, &a));
  std::lock_guard<std::mutex> lock(h->mu);
  CallPlan& c = h->call[0];
  QW_TRY(call_for(h, M, a->base, &c));
  QW_TRY(bind_x(h, &c, x_bf16));
  return launch_call_prologue(c, c.prm, h->r, as_stream(stream));
}

qwam_status qwam_gemm(int M, qwam_handle h, void* y_bf16, void* stream) {
  QW_TRY(check_handle(h));
  if (M < 0) return fail(QWAM_ERR_SHAPE, "M=%d must be >= 0", M);
  if (M == 0) return QWAM_OK;
  if (!y_bf16) return fail(QWAM_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y_bf16)) return fail(QWAM_ERR_ALIGN, "y must be 16-byte aligned");
  Arena* a = nullptr;
  QW_TRY(workspace_for(h, M, &a));
  std::lock_guard<std::mutex> lock(h->mu);
  CallPlan& c = h->call[0];
  QW_TRY(call_for(h, M, a->base, &c));
  QW_TRY(bind_y(h, &c, y_bf16));
  return launch_call_gemm(c, as_stream(stream));
}

qwam_status qwam_linear(const void* x_bf16, int M, qwam_handle h, void* y_bf16, void* stream) {
  QW_TRY(check_linear_args(x_bf16, M, h));
  if (M == 0) return QWAM_OK;
  if (!y_bf16) return fail(QWAM_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y_bf16)) return fail(QWAM_ERR_ALIGN, "y must be 16-byte aligned");
  if (y_bf16 == x_bf16) return fail(QWAM_ERR_INVALID_ARG, "y must not alias x");
  Arena* a = nullptr;
  QW_TRY(workspace_for(h, M, &a));
  const cudaStream_t st = as_stream(stream);
  std::lock_guard<std::mutex> lock(h->mu);
  CallPlan& c = h->call[0];
  QW_TRY(call_for(h, M, a->base, &c));
  QW_TRY(bind_x(h, &c, x_bf16));
  QW_TRY(bind_y(h, &c, y_bf16));
  QW_TRY(launch_call_prologue(c, c.prm, h->r, st));
  return launch_call_gemm(c, st);
}

qwam_status qwam_linear_noalloc(const void* x_bf16, int M, qwam_handle h, void* y_bf16, void* stream) {
  QW_TRY(check_linear_args(x_bf16, M, h));
  if (M == 0) return QWAM_OK;
  if (!y_bf16) return fail(QWAM_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y_bf16)) return fail(QWAM_ERR_ALIGN, "y must be 16-byte aligned");
  if (y_bf16 == x_bf16) return fail(QWAM_ERR_INVALID_ARG, "y must not alias x");
  return linear_noalloc_impl(x_bf16, M, h, y_bf16, as_stream(stream));
}

qwam_status qwam_handle_info(qwam_handle h, int* N, int* K, int* r, int* b, float* g_w) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  if (N) *N = h->N;
  if (K) *K = h->K;
  if (r) *r = h->r;
  if (b) *b = h->b;
  if (g_w) *g_w = h->g_w;
  return QWAM_OK;
}

qwam_status qwam_export_weight(qwam_handle h, void* codes, void* scales, void* L_bf16, void* stream) {
  QW_TRY(check_handle(h));
  cudaStream_t st = as_stream(stream);
  if (codes)
    QW_CUDA(cudaMemcpyAsync(codes, h->codes, static_cast<size_t>(h->N) * code_bytes(h->K, h->fmt),
                            cudaMemcpyDeviceToDevice, st));
  if (scales && h->fmt == 0)
    QW_CUDA(cudaMemcpyAsync(scales, h->sf, round_up(static_cast<size_t>(h->N), 128) * h->K / 16, cudaMemcpyDeviceToDevice, st));
  if (scales && h->fmt == 2) QW_CUDA(cudaMemcpyAsync(scales, h->sf, h->sf_bytes, cudaMemcpyDeviceToDevice, st));
  if (L_bf16 && h->r > 0)
    QW_CUDA(cudaMemcpyAsync(L_bf16, h->L, static_cast<size_t>(h->N) * h->r * 2, cudaMemcpyDeviceToDevice, st));
  return QWAM_OK;
}

qwam_status qwam_debug_prologue(const void* x_bf16, int M, qwam_handle h, float* z_f32, float* u_f32, void* codes,
                                void* scales, void* ubr_bf16, float* g_x, void* stream) {
  QW_TRY(check_linear_args(x_bf16, M, h));
  if (M == 0) return QWAM_OK;
  if ((z_f32 && !aligned16(z_f32)) || (u_f32 && !aligned16(u_f32)))
    return fail(QWAM_ERR_ALIGN, "debug outputs must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  Arena* a = nullptr;
  QW_TRY(workspace_for(h, M, &a));
  const Layout lay = layout_of(h, M);
  {
    std::lock_guard<std::mutex> lock(h->mu);
    CallPlan& c = h->call[0];
    QW_TRY(call_for(h, M, a->base, &c));
    QW_TRY(bind_x(h, &c, x_bf16));
    PrologueParams prm = c.prm;  // with the debug exports of z and u
    prm.z_out = z_f32;
    prm.u_out = u_f32;
    QW_TRY(launch_call_prologue(c, prm, h->r, st));
  }
  if (codes)
    QW_CUDA(cudaMemcpyAsync(codes, a->base + lay.codes, static_cast<size_t>(M) * code_bytes(h->K, h->fmt),
                            cudaMemcpyDeviceToDevice, st));
  if (scales && h->fmt != 1)  // NVFP4 tiles, or INT4 fp32 [K / 64][round_up(M, 128)]: the same bytes
    QW_CUDA(cudaMemcpyAsync(scales, a->base + lay.sf, round_up(static_cast<size_t>(M), 128) * h->K / 16,
                            cudaMemcpyDeviceToDevice, st));
  if (ubr_bf16 && h->r > 0)
    QW_CUDA(cudaMemcpyAsync(ubr_bf16, a->base + lay.ub, static_cast<size_t>(M) * h->r * 2, cudaMemcpyDeviceToDevice, st));
  if (g_x) {
    static const float kOne = 1.0f;  // INT4 has no per-tensor scale
    if (h->fmt == 2) QW_CUDA(cudaMemcpyAsync(g_x, &kOne, 4, cudaMemcpyHostToDevice, st));
    else QW_CUDA(cudaMemcpyAsync(g_x, arena_gx(*a), 4, cudaMemcpyDeviceToDevice, st));
  }
  return QWAM_OK;
}

qwam_status qwam_quantize_fp32(const float* T, int rows, int K, void* codes, void* scales, float* g, void* stream) {
  if (!T || !codes || !scales || !g) return fail(QWAM_ERR_INVALID_ARG, "NULL argument");
  if (rows < 1 || K < 64 || K % 64) return fail(QWAM_ERR_SHAPE, "rows >= 1 and K a positive multiple of 64 required");
  if (!aligned16(T) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(g) & 3))
    return fail(QWAM_ERR_ALIGN, "buffers must be 16-byte aligned");
  int dev = 0;
  QW_TRY(current_device(&dev));
  Arena* a = nullptr;
  QW_TRY(arena_get(dev, kHeaderBytes, &a));
  QW_CUDA(launch_quantize_fp32(T, rows, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), g,
                               arena_amax(*a), as_stream(stream)));
  return QWAM_OK;
}

namespace {

qwam_status fp4_gemm_impl(const void* a_codes, const void* a_scales, const void* b_codes, const void* b_scales, int M,
                          int N, int K, float alpha, float* out_f32, uint64_t wait_ns, uint32_t withheld,
                          cudaStream_t st) {
  if (!a_codes || !a_scales || !b_codes || !b_scales || !out_f32) return fail(QWAM_ERR_INVALID_ARG, "NULL argument");
  if (M < 1 || N < 16 || N % 16 || K < 128 || K % 128) return fail(QWAM_ERR_SHAPE, "bad GEMM shape M=%d N=%d K=%d", M, N, K);
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(out_f32))
    return fail(QWAM_ERR_ALIGN, "buffers must be 16-byte aligned");
  int dev = 0;
  QW_TRY(current_device(&dev));
  Arena* a = nullptr;
  QW_TRY(arena_get(dev, kHeaderBytes, &a));
  const GemmShape sh = gemm_shape(M, N);
  if (withheld && sh.pair)
    return fail(QWAM_ERR_SHAPE, "the wait-expiry check runs on single-CTA tiles (M <= 128 or N < 256)");
  GemmMaps maps{};
  QW_TRY(make_codes_map(&maps.a, a_codes, M, K / 2, sh.ks / 2, 128));
  QW_TRY(make_codes_map(&maps.b, b_codes, N, K / 2, sh.ks / 2, sh.pair ? sh.bn / 2 : sh.bn));
  maps.u = maps.a;
  maps.l = maps.b;
  maps.y = maps.a;
  QW_TRY(make_sf_map(&maps.sfa, a_scales, round_up(static_cast<size_t>(M), 128), K, sh.ks, 1));
  QW_TRY(make_sf_map(&maps.sfb, b_scales, round_up(static_cast<size_t>(N), sh.bn), K, sh.ks, sh.bn / 128));
  GemmParams p{};
  p.M = M; p.N = N; p.K = K;
  p.k_stages = (K + sh.ks - 1) / sh.ks;
  p.splits = 1;
  p.sfa = static_cast<const uint8_t*>(a_scales);
  p.sfb = static_cast<const uint8_t*>(b_scales);
  p.g_a_ptr = nullptr;
  p.g_a = alpha;
  p.g_b = 1.0f;
  p.out_f32 = out_f32;
  p.err = arena_err(*a);
  p.sms = sm_count(dev);
  p.wait_ns = wait_ns;
  p.withheld_bytes = withheld;
  QW_CUDA(launch_gemm(maps, p, sh, GemmEpilogue::RawF32, st));
  return QWAM_OK;
}

}  // namespace

qwam_status qwam_fp4_gemm(const void* a_codes, const void* a_scales, const void* b_codes, const void* b_scales,
                          int M, int N, int K, float alpha, float* out_f32, void* stream) {
  return fp4_gemm_impl(a_codes, a_scales, b_codes, b_scales, M, N, K, alpha, out_f32, 0, 0, as_stream(stream));
}

qwam_status qwam_debug_fp4_gemm_withheld(const void* a_codes, const void* a_scales, const void* b_codes,
                                         const void* b_scales, int M, int N, int K, uint64_t wait_ns, float* out_f32,
                                         void* stream) {
  if (wait_ns < 1000 || wait_ns > 1000000000ull)
    return fail(QWAM_ERR_INVALID_ARG, "wait_ns=%llu must lie in [1 us, 1 s]", static_cast<unsigned long long>(wait_ns));
  return fp4_gemm_impl(a_codes, a_scales, b_codes, b_scales, M, N, K, 1.0f, out_f32, wait_ns, 16u, as_stream(stream));
}

qwam_status qwam_plan_info(int M, qwam_handle h, int* kernels, int* fused, int* splits, int* bn) {
  if (!h || h->magic != kMagic) return fail(QWAM_ERR_INVALID_ARG, "invalid qwam handle");
  if (M < 0) return fail(QWAM_ERR_SHAPE, "M=%d must be >= 0", M);
  if (h->fmt == 2) {  // Local prologue, group GEMM (+ the split-K sum)
    const int sp = group_splits(std::max(M, 1), h->N, h->K, sm_count(h->dev));
    if (kernels) *kernels = M == 0 ? 0 : (sp > 1 ? 3 : 2);
    if (fused) *fused = 0;
    if (splits) *splits = sp;
    if (bn) *bn = 128;
    return QWAM_OK;
  }
  const bool f = use_fused(M);
  const Plan pl = plan_gemm(std::max(M, 1), h->N, h->K, sm_count(h->dev), h->fmt);
  const int form = prologue_form(std::max(M, 1), h->r, h->K, sm_count(h->dev));
  if (kernels) *kernels = M == 0 ? 0 : (form == PRO_FUSED || form == PRO_ONEPASS ? 2 : 3);
  if (fused) *fused = f ? 1 : 0;
  if (splits) *splits = pl.splits;
  if (bn) *bn = pl.bn;
  return QWAM_OK;
}

qwam_status qwam_selfcheck_rounding(uint64_t* mismatches, uint64_t random_pairs, void* stream) {
  if (!mismatches) return fail(QWAM_ERR_INVALID_ARG, "mismatches is NULL");
  unsigned long long* d = nullptr;
  QW_CUDA(cudaMalloc(&d, 3 * sizeof(unsigned long long)));
  const cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemsetAsync(d, 0, 3 * sizeof(unsigned long long), st);
  if (e == cudaSuccess) e = launch_rounding_check(d, random_pairs, st);
  unsigned long long h[3] = {0, 0, 0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(h, d, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(d);
  if (e != cudaSuccess) return fail(QWAM_ERR_CUDA, "rounding self-check failed: %s", cudaGetErrorString(e));
  for (int k = 0; k < 3; ++k) mismatches[k] = h[k];
  return QWAM_OK;
}

qwam_status qwam_device_error(uint32_t* code) {
  if (!code) return fail(QWAM_ERR_INVALID_ARG, "code is NULL");
  *code = 0;
  int dev = 0;
  QW_CUDA(cudaGetDevice(&dev));
  QW_CUDA(cudaDeviceSynchronize());
  if (dev < 0 || dev >= kMaxDevices) return QWAM_OK;
  uint8_t* sbase = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    sbase = g_static_base[dev];
  }
  if (sbase) {  // the error word of qwam_linear_noalloc's static scratch
    uint32_t c = 0;
    QW_CUDA(cudaMemcpy(&c, sbase + kErrOffset, 4, cudaMemcpyDeviceToHost));
    QW_CUDA(cudaMemset(sbase + kErrOffset, 0, 4));
    *code |= c;
  }
  std::lock_guard<std::mutex> lock(g_arena_mu);
  const Arena& a = g_arena[dev];
  if (a.base) {
    uint32_t c = 0;
    QW_CUDA(cudaMemcpy(&c, arena_err(a), 4, cudaMemcpyDeviceToHost));
    QW_CUDA(cudaMemset(arena_err(a), 0, 4));
    *code |= c;
  }
  if (*code) return fail(QWAM_ERR_TIMEOUT, "a bounded device wait expired (flags 0x%x)", *code);
  return QWAM_OK;
}

const char* qwam_last_error(void) { return g_err.c_str(); }

const char* qwam_status_string(qwam_status s) {
  switch (s) {
    case QWAM_OK: return "QWAM_OK";
    case QWAM_ERR_INVALID_ARG: return "QWAM_ERR_INVALID_ARG";
    case QWAM_ERR_SHAPE: return "QWAM_ERR_SHAPE";
    case QWAM_ERR_ALIGN: return "QWAM_ERR_ALIGN";
    case QWAM_ERR_ARCH: return "QWAM_ERR_ARCH";
    case QWAM_ERR_OOM: return "QWAM_ERR_OOM";
    case QWAM_ERR_CUDA: return "QWAM_ERR_CUDA";
    case QWAM_ERR_TIMEOUT: return "QWAM_ERR_TIMEOUT";
    case QWAM_ERR_FORMAT: return "QWAM_ERR_FORMAT";
  }
  return "QWAM_UNKNOWN";
}

int qwam_version(void) { return 100; }

}  // extern "C"
