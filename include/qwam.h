/*
 * qwam — the Action-Subspace-Protected (deflated form) NVFP4 W4A4 linear
 * layer on NVIDIA B200 (sm_100a), as a C-ABI shared library (libqwam.so).
 *
 * The layer ("FastWAM UR3 3-task — 4-bit quantisations", model card, section
 * "What ASP is, and what the deflated form means"):
 *
 *     x~ = (x / s) H
 *     y  = (x~ V)(W~ V)^T + NVFP4GEMM((I - V V^T) x~, W~ (I - V V^T)) + bias
 *
 * s: per-input-channel smoothing vector; H: block Hadamard (blocks of b,
 * Sylvester order, scaled by 1/sqrt(b)); V: K x r basis with orthonormal
 * columns; W~ = W diag(s) H (H on both sides so the branch pairs x~V with W~V
 * in the same coordinates).  NVFP4 ("numeric format" row of the card's top
 * table): E2M1 elements in blocks of 16 along K with E4M3 block scales, plus a
 * fp32 per-tensor scale g = amax / 2688.  The rank-r branch stays bf16 ("The
 * rank-32 branch stays in bf16 by design"; the Q-WAM abstract's "16-bit
 * low-rank branch").
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    "host" pointers are ordinary CPU memory.  Every pointer is BORROWED: the
 *    library never frees caller memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Device work is enqueued on it in order; outputs are valid once the stream
 *    reaches that point.
 *  - Matrices are row-major and contiguous.  Device pointers must be 16-byte
 *    aligned.
 *  - Every call returns a qwam_status.  On any status other than QWAM_OK no
 *    output has been written (argument checks happen before any launch) and
 *    qwam_last_error() returns a message for the calling thread.  Nothing
 *    traps on the device; a bounded device-side wait that runs out sets a
 *    flag read by qwam_device_error().
 *  - Shape limits: K % 128 == 0, K % b == 0, b in {1,2,4,...,128},
 *    r in {0, 16, 32}, N % 16 == 0, N >= 16, M >= 0 (M == 0 is a no-op).
 *  - Requires a compute capability 10.0 device (B200).
 */
#ifndef QWAM_H
#define QWAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct qwam_layer* qwam_handle;

typedef enum {
  QWAM_OK = 0,
  QWAM_ERR_INVALID_ARG = 1, /* null pointer, bad value (e.g. s <= 0), bad handle */
  QWAM_ERR_SHAPE = 2,       /* a shape limit above is violated */
  QWAM_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
  QWAM_ERR_ARCH = 4,        /* current device is not compute capability 10.x */
  QWAM_ERR_OOM = 5,         /* device allocation failed */
  QWAM_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed */
  QWAM_ERR_TIMEOUT = 7,     /* a bounded device wait expired (qwam_device_error) */
  QWAM_ERR_FORMAT = 8       /* a layer image is malformed or fails its checksum */
} qwam_status;

/* ---------------------------------------------------------------------------
 * Weight side (offline).  Card sections "What ASP is..." (deflated form: the
 * branch carries the exact W~V, the FP4 weight holds W~(I - VV^T)) and "Files"
 * (E4M3 scales pre-swizzled to the 128x4 tensor-core tile layout).
 *
 *   W_bf16  device bf16 [N, K]          weight
 *   s       device fp32 [K]             smoothing vector, every entry > 0 and finite
 *   V       device fp32 [K, r]          basis; may be NULL iff r == 0
 *   bias    device bf16 [N] or NULL
 *   out     host   receives the new handle
 *
 * Computes W~ = W diag(s) H, L = W~V (stored bf16 [N, r]), W_d = W~ - L V^T,
 * and quantises W_d (packed E2M1 codes [N, K/2], tiled E4M3 scales, fp32 g_w).
 * The handle owns copies of everything it needs (1/s, V split into bf16
 * hi/lo parts, bias); the caller may free W, s, V and bias when this returns.
 * The call synchronises `stream`.
 * ------------------------------------------------------------------------- */
qwam_status qwam_prepare_weight(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                const void* bias_bf16, int hadamard_block, void* stream, qwam_handle* out);

/* ---------------------------------------------------------------------------
 * The shared-weight arm (card, section "What ASP is...": the cheaper variant
 * that "quantises one weight and stores V alone").  Read here as: the FP4
 * weight is W~ = W diag(s) H itself, not deflated, and the branch weight is
 * formed from that stored weight, L = deq(Q(W~)) V (fp32 accumulation, stored
 * bf16), so a handle carries nothing beyond the FP4 weight, V and the bias.
 * The activation side and every per-call entry point are those of the
 * deflated arm (qwam_linear and the rest take the handle unchanged).
 * Arguments as qwam_prepare_weight; Wt_f32 (device fp32 [N, K] or NULL)
 * receives the exact fp32 W~ the weight quantiser consumed.  With r == 0 the
 * two arms coincide.
 * ------------------------------------------------------------------------- */
qwam_status qwam_prepare_weight_shared(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                       const void* bias_bf16, int hadamard_block, float* Wt_f32, void* stream,
                                       qwam_handle* out);

/* ---------------------------------------------------------------------------
 * The FP8 W8A8 arm ("QuantWAMs: Calibrating at the Right Granularity for World
 * Action Models", section "During inference": FP8 W8A8 for the Linears that
 * calibration upgrades).  The same layer with both quantisers FP8 E4M3 (one
 * byte per element, no block scales) and one fp32 scale per tensor,
 * g = amax / 448: the weight's at prepare, the activation's per call; element
 * code = sign | E4M3_rn_satfinite(|v * (1 / g)|).  The GEMM runs on
 * tcgen05.mma kind::f8f6f4; smoothing, block rotation, the rank-r branch, the
 * epilogue and every per-call entry point are those of the NVFP4 arm.
 * Arguments as qwam_prepare_weight; Wd_f32 (device fp32 [N, K] or NULL)
 * receives the exact fp32 W_d the weight quantiser consumed.  Exports of this
 * handle's codes (qwam_export_weight, qwam_debug_prologue) are [rows, K] bytes
 * and carry no scales.
 * ------------------------------------------------------------------------- */
qwam_status qwam_prepare_weight_fp8(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                    const void* bias_bf16, int hadamard_block, float* Wd_f32, void* stream,
                                    qwam_handle* out);

/* ---------------------------------------------------------------------------
 * The SVDQuant INT4 W4A4 arm ("FastWAM UR3 3-task -- 4-bit quantisations",
 * top table, SVDQuant column: INT4 at group 64 on weights and activations,
 * a low-rank branch, products on integer tensor cores, exact for 4-bit
 * codes; section "Verification -- INT4 SVDQuant").  In this library's terms:
 * smoothing x^ = x / s and W^ = W diag(s) with no rotation (b = 1); the
 * branch from the rank-r basis V, L = W^ V (with V the top right singular
 * vectors of W^, L V^T is its rank-r truncated SVD); the residual
 * R = W^ - L V^T and the activation x^ itself (not deflated) quantised
 * INT4 per group of 64 along K:
 *
 *   y = deq(Q(x^)) deq(Q(R))^T + (x^ V) L^T + bias
 *
 * Q: a = max |v| of the group, s = fp16_rn(a / 7) (saturated to 65504),
 * level = clamp(rint(v * (1 / s)), -8, 7) (fp32, half to even; 0 when
 * s == 0).  The levels reach the tensor core as E4M3 bytes (kind::f8f6f4
 * gives the exact integer group sums); each group's sums are scaled by
 * s_x s_w and added in fp32 in group order.
 *
 * Arguments as qwam_prepare_weight without hadamard_block (b = 1); Wd_f32
 * (device fp32 [N, K] or NULL) receives the exact fp32 R the weight
 * quantiser consumed.  The handle's weight export (qwam_export_weight): codes
 * [N, K] E4M3 bytes of the levels; scales fp32 [K / 64][N] (N * K / 16 bytes).
 * The activation export (qwam_debug_prologue): z = the fp32 x^ quantised,
 * codes [M, K] E4M3 bytes, scales fp32 [K / 64][round_up(M, 128)], u' =
 * bf16(u) (no scale to divide by), g_x = 1.  Every per-call entry point takes
 * the handle; qwam_linear_noalloc within its scratch limit.
 * ------------------------------------------------------------------------- */
qwam_status qwam_prepare_weight_int4(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                     const void* bias_bf16, float* Wd_f32, void* stream, qwam_handle* out);

/* Host outputs (each may be NULL): the element format of the handle (0 NVFP4,
 * 1 FP8 E4M3, 2 INT4 group 64) and its weight arm (0 deflated, 1
 * shared-weight, 2 SVDQuant). */
qwam_status qwam_handle_format(qwam_handle h, int* fmt, int* variant);

/* ---------------------------------------------------------------------------
 * Layer images (card "FastWAM UR3 3-task -- 4-bit quantisations", section
 * "Files": the NVFP4 deflated-ASP checkpoint stores packed E2M1 weights and
 * E4M3 block scales already in the tensor-core tile layout, and is
 * self-contained).  A prepared layer as one host byte string, so that a
 * checkpoint is quantised once and loaded without the bf16 weight.
 *
 * Layout (little-endian): a 64-byte header {char magic[8] = "QWAMIMG\0";
 * uint32 version = 1; uint32 header_bytes = 64; int32 N, K, r, b, fmt,
 * variant; uint32 flags (bit 0: bias present); float g_w; uint64
 * total_bytes; uint64 checksum}, then these arrays, each zero-padded to a
 * multiple of 16 bytes: codes (N * K/2 bytes; FP8: N * K; INT4: the levels
 * as 4-bit two's complement, two per byte, the even element in the low
 * nibble), scales (NVFP4: round_up(N,256) * K/16 bytes, tiled as on the
 * device; INT4: fp16 [K/64][N]; none for FP8), and
 * when r > 0: L bf16 [N, r], V hi and lo bf16 [K, r] each, P^T hi and lo
 * bf16 [r, K] each; then 1/s fp32 [K]; then bias bf16 [N] when flag bit 0
 * is set.  checksum = FNV-1a 64 (offset basis 0xcbf29ce484222325, prime
 * 0x100000001b3) over all total_bytes with the checksum field read as zero.
 *
 * qwam_image_size: *bytes = the image length of h (host call, no device work).
 * qwam_save_image: writes the image of h into host_buf (host memory, pageable
 *   or pinned, at least qwam_image_size bytes; QWAM_ERR_INVALID_ARG if
 *   shorter).  Copies on `stream` and synchronises it.
 * qwam_load_image: checks the image on the host first (magic, version, a
 *   valid shape and format, total_bytes against the shape and buf_bytes, the
 *   checksum: QWAM_ERR_FORMAT on any mismatch, with nothing allocated), then
 *   makes a new handle on the current device whose calls return exactly what
 *   the saved handle's calls return.  The caller keeps host_buf; the call
 *   synchronises `stream`.
 * ------------------------------------------------------------------------- */
qwam_status qwam_image_size(qwam_handle h, size_t* bytes);
qwam_status qwam_save_image(qwam_handle h, void* host_buf, size_t buf_bytes, void* stream);
qwam_status qwam_load_image(const void* host_buf, size_t buf_bytes, void* stream, qwam_handle* out);

/* Release a handle and its device memory (synchronises the device). */
qwam_status qwam_destroy(qwam_handle h);

/* ---------------------------------------------------------------------------
 * Activation side (per call).  y = the layer above for x.
 *
 *   x_bf16  device bf16 [M, K]   (read only)
 *   y_bf16  device bf16 [M, N]   (written; must not alias x)
 *
 * Runs the fused prologue (x/s, block FWHT, u = x~V, z = x~ - uV^T, per-tensor
 * amax, NVFP4 quantisation of z, u' = bf16(u / (g_x g_w))) and the tcgen05
 * block-scaled FP4 GEMM whose epilogue adds u' L^T and the bias and rounds
 * once to bf16.  Scratch comes from a per-device workspace inside the library
 * that grows on first use of a larger shape (that call allocates and
 * synchronises the device, so it must not be stream-captured; a call at the
 * largest M first makes later calls allocation-free).  Calls that share the
 * workspace must be ordered: do not run two qwam_linear calls concurrently on
 * different streams of the same device.  The handle keeps the launch arguments
 * (tensor maps) of its last M, so a repeated call encodes nothing and a new x
 * or y buffer only re-points its map; host calls on one handle are serialised
 * by a lock inside it.
 * ------------------------------------------------------------------------- */
qwam_status qwam_linear(const void* x_bf16, int M, qwam_handle h, void* y_bf16, void* stream);

/* ---------------------------------------------------------------------------
 * qwam_linear without any device allocation.  The model card describes no
 * such call: it exists for callers that must not allocate device memory once
 * running, such as a fixed-rate control loop (a cudaMalloc may synchronise
 * the device and stall it for milliseconds) or a process whose device memory
 * is budgeted at start-up.
 *
 * Same arguments, launches and result as qwam_linear (same kernels and the
 * same GEMM plan), but all scratch lives in one fixed 2 MiB array compiled
 * into the library (one copy per device) instead of the growable workspace.
 * Limits: M <= 128 rows and K <= 16384 (QWAM_ERR_SHAPE beyond them, before
 * anything is launched); within them every N, r and b that qwam_linear takes,
 * except that an INT4 handle's split-K partial tiles (splits x M x N x 4
 * bytes) must fit the array too (QWAM_ERR_SHAPE otherwise).
 * The first call on a device does the set-up (looks up the array's device
 * address and clears its header, whose error word must start at zero,
 * synchronising the device); make that first call before any latency-critical
 * loop and before any stream capture: a first call whose stream is being
 * captured returns QWAM_ERR_INVALID_ARG and does nothing.  All calls share the
 * one array per device, whatever the handle: calls
 * that overlap in time (other streams, other threads) race on it and corrupt
 * each other's results, so order them.
 * Expired bounded waits are reported by qwam_device_error.
 * ------------------------------------------------------------------------- */
qwam_status qwam_linear_noalloc(const void* x_bf16, int M, qwam_handle h, void* y_bf16, void* stream);

/* The two halves of qwam_linear, for measurement: qwam_linear(x, M, h, y, st)
 * == qwam_prologue(x, M, h, st) followed by qwam_gemm(M, h, y, st) on the same
 * stream with nothing else using the workspace in between. */
qwam_status qwam_prologue(const void* x_bf16, int M, qwam_handle h, void* stream);
qwam_status qwam_gemm(int M, qwam_handle h, void* y_bf16, void* stream);

/* ---------------------------------------------------------------------------
 * Inspection and test exports (not on the hot path).
 * ------------------------------------------------------------------------- */

/* Host outputs (each may be NULL): N, K, r, b and the weight scale g_w. */
qwam_status qwam_handle_info(qwam_handle h, int* N, int* K, int* r, int* b, float* g_w);

/* Copy the handle's weight operands into caller device buffers (each may be
 * NULL): codes [N, K/2] bytes (FP8 handles: [N, K]); scales: the tiled layout,
 * round_up(N,128)*K/16 bytes (not written for FP8 handles); L: bf16 [N, r]. */
qwam_status qwam_export_weight(qwam_handle h, void* codes, void* scales, void* L_bf16, void* stream);

/* Same as qwam_prepare_weight, and also writes W_d (the exact fp32 tensor the
 * weight quantiser consumed) to Wd_f32 (device fp32 [N, K]). */
qwam_status qwam_debug_prepare_weight(const void* W_bf16, int N, int K, const float* s, const float* V, int r,
                                      const void* bias_bf16, int hadamard_block, float* Wd_f32, void* stream,
                                      qwam_handle* out);

/* Run the activation prologue and copy its products to caller device buffers
 * (each may be NULL): z fp32 [M, K] (the exact quantiser input), u fp32 [M, r],
 * codes [M, K/2] (FP8 handles: [M, K]), scales (tiled, round_up(M,128)*K/16
 * bytes; not written for FP8 handles), u' bf16 [M, r], g_x fp32 scalar. */
qwam_status qwam_debug_prologue(const void* x_bf16, int M, qwam_handle h, float* z_f32, float* u_f32,
                                void* codes, void* scales, void* ubr_bf16, float* g_x, void* stream);

/* The bare NVFP4 quantiser on a device fp32 tensor T [rows, K] (K % 64 == 0):
 * codes [rows, K/2], scales in the tiled layout (round_up(rows,128)*K/16 bytes;
 * padding rows are not written), g (device fp32 scalar). */
qwam_status qwam_quantize_fp32(const float* T, int rows, int K, void* codes, void* scales, float* g, void* stream);

/* The bare block-scaled FP4 GEMM: out[m,n] = alpha * sum_k deq(A)[m,k] deq(B)[n,k]
 * with deq = e2m1(code) * e4m3(scale) (no per-tensor scales).  a_codes [M, K/2],
 * b_codes [N, K/2]; a_scales / b_scales in the tiled layout with rows padded to
 * 128 (A) and 256 (B), padding bytes zero; out fp32 [M, N] device.  K % 128 == 0. */
qwam_status qwam_fp4_gemm(const void* a_codes, const void* a_scales, const void* b_codes, const void* b_scales,
                          int M, int N, int K, float alpha, float* out_f32, void* stream);

/* Check of the bounded device waits (failure detection without a fault): the
 * bare GEMM above (alpha = 1) on single-CTA tiles (M <= 128, or N < 256),
 * with every wait limited to wait_ns (1 us .. 1 s) and the first pipeline
 * stage's barrier told to expect 16 bytes more than its TMA boxes carry, so
 * it never completes.  Every role's wait behind it runs out, sets its bit in
 * the device error word and the kernel returns; qwam_device_error() then
 * reports QWAM_ERR_TIMEOUT and the context stays usable.  out_f32 is not
 * written.  The card has no counterpart: this exercises the library's own
 * wind-down paths. */
qwam_status qwam_debug_fp4_gemm_withheld(const void* a_codes, const void* a_scales, const void* b_codes,
                                         const void* b_scales, int M, int N, int K, uint64_t wait_ns, float* out_f32,
                                         void* stream);

/* How qwam_linear runs for M rows of this layer (host outputs, each may be
 * NULL): kernels = kernel launches per call (2 when the prologue is one launch:
 * up to 128 rows, or rank 0 with at most six 128-row tiles per CTA; else 3),
 * fused = 1 when the prologue is the single-launch cluster form for up to 128
 * rows, splits = K splits of the GEMM, bn = GEMM tile width. */
qwam_status qwam_plan_info(int M, qwam_handle h, int* kernels, int* fused, int* splits, int* bn);

/* The bare INT4 group GEMM of the SVDQuant arm, for tests: out_f32 [M, N] =
 * sum over the K / 64 groups g of P_g (sa[g][m] sb[g][n]), with P_g the exact
 * group sums of the levels, accumulated in fp32 in group order (no branch, no
 * bias).  a_levels [M, K] and b_levels [N, K]: E4M3 bytes of INT4 levels;
 * a_scales fp32 [K / 64][M], b_scales fp32 [K / 64][N].  M % 4 == 0,
 * N % 16 == 0, K % 128 == 0 (QWAM_ERR_SHAPE otherwise); 16-byte aligned device
 * buffers.  Expired waits are reported by qwam_device_error. */
qwam_status qwam_int4_gemm(const void* a_levels, const float* a_scales, const void* b_levels, const float* b_scales,
                           int M, int N, int K, float* out_f32, void* stream);

/* Synchronise the current device, then return (and clear) the device error
 * word set by bounded waits: *code == 0 means none expired.  Returns
 * QWAM_ERR_TIMEOUT when *code != 0. */
qwam_status qwam_device_error(uint32_t* code);

/* Self-check of the quantiser's arithmetic on the current device.  The block
 * scale's two divisions and the reciprocal of the scale are computed with fp32
 * FMAs (an estimate, an exact residual, one correction) instead of the IEEE
 * division / reciprocal sequences, with results required to be identical:
 * mismatches[0] counts inputs where a / 6 differs from the IEEE division and
 * mismatches[1] where 1 / e differs from the IEEE reciprocal, over every
 * positive finite fp32 input; mismatches[2] counts (u, g) pairs whose E4M3 code
 * of u / g differs from the code of the IEEE quotient, over every u >= 0 at four
 * divisors and `random_pairs` pseudo-random pairs.  All zero means identical.
 * `mismatches` is host memory with three entries.  Allocates 24 bytes of device
 * memory and synchronises the stream.  The card (section "What ASP is...") has
 * no counterpart; the op order it checks is the quantiser's (NVFP4 format). */
qwam_status qwam_selfcheck_rounding(uint64_t* mismatches, uint64_t random_pairs, void* stream);

/* Message for the last failing call on this thread ("" if none). */
const char* qwam_last_error(void);

/* Static name of a status code. */
const char* qwam_status_string(qwam_status s);

/* Library version (major * 10000 + minor * 100 + patch). */
int qwam_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QWAM_H */
