/*
 * w4a4.h -- C ABI of the B200 (sm_100a) ConvRot W4A4 linear layer.
 *
 * The method (page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with
 * fused CUDA kernels", section "Description"):
 *   - activations x[M,K] are rotated with a blockwise Walsh-Hadamard
 *     transform (ConvRot; contiguous groups of g columns, natural order,
 *     normalised by 1/sqrt(g)), then quantised per row to signed int4 with
 *     one fp32 scale per row (scale = amax/7, round half to even, clamp to
 *     [-7, 7]) and packed two per byte, low nibble first, into an [M, K/2]
 *     int8 container;
 *   - weights W[N,K] are rotated and quantised the same way once, offline,
 *     giving packed [N, K/2] int8 plus fp32 [N] scales;
 *   - an s4 x s4 GEMM accumulates in int32 (|acc| <= 49*K), and a rank-one
 *     epilogue writes y[m,n] = bf16(acc * sx[m] * sw[n] + bias[n]).
 *
 * Conventions for every entry point:
 *   - Every tensor pointer is DEVICE memory owned by the caller; the library
 *     never allocates or frees memory.  Matrices are row-major with the
 *     inner dimension contiguous; ld* arguments are row strides in elements.
 *   - bf16 tensors are passed as raw 16-bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued asynchronously on it; the return value reports argument
 *     checks and launch errors only.  Kernels that give up waiting record
 *     W4A4_ERR_TIMEOUT in a device status word read by w4a4_last_device_error.
 *   - Errors are returned as w4a4_status codes, never printed or thrown.
 *   - Only sm_100 devices are supported (W4A4_ERR_DEVICE otherwise).
 *   - Calls are thread-safe as long as different host threads use different
 *     outputs and workspaces.
 *
 * Environment (read once per process, at the first call that needs it; they
 * choose between kernels that compute the same result):
 *   - W4A4_SMALLM_MAX=<0..64>: w4a4_linear and w4a4_linear_fused use the
 *     weight-streaming kernels for M up to this value (default 64); the
 *     CUDA-core one serves M = 1 and M <= 4 with M*K <= 12288 of those.
 *   - W4A4_ROTATE_TC_MIN_ROWS=<n>: activations without GELU, g in {64, 128}
 *     and K/g <= 128 are rotated on the tensor cores from n rows up (default
 *     8192); W4A4_ROTATE_TC=0 keeps the register-butterfly kernel for every
 *     shape.  The two differ only in the order of the fp32 additions of the
 *     rotation.
 */
#ifndef W4A4_H_
#define W4A4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4A4_OK = 0,
  W4A4_ERR_NULL = 1,      /* a required pointer is NULL                         */
  W4A4_ERR_SHAPE = 2,     /* a size is out of range or breaks a multiple rule   */
  W4A4_ERR_GROUP = 3,     /* g not in {64,128,256} or does not divide K          */
  W4A4_ERR_ALIGN = 4,     /* a pointer or leading dimension is misaligned        */
  W4A4_ERR_WORKSPACE = 5, /* workspace missing or smaller than required          */
  W4A4_ERR_DEVICE = 6,    /* the current device is not an sm_100 GPU             */
  W4A4_ERR_CUDA = 7,      /* a CUDA runtime/driver call or a launch failed       */
  W4A4_ERR_TIMEOUT = 8,   /* a kernel gave up waiting (bounded spin expired)     */
  W4A4_ERR_ARG = 9        /* another argument is invalid (e.g. an unknown act)   */
} w4a4_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* w4a4_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int w4a4_version(void);

/*
 * Offline weight preparation: rotate (ConvRot) and quantise the rows of an
 * fp32 weight.  Page "[PR #63] ...", Description: the weight is stored as
 * two signed 4-bit codes per byte, the even element in the low nibble, in an
 * int8 array of N rows by K/2 bytes, with one fp32 scale per output row.
 *   W   [N, K] fp32, row stride ldw >= K (elements), 16-byte aligned, ldw % 4 == 0
 *   N >= 1;  K % 128 == 0, K % g == 0, 128 <= K <= 24576;  g in {64,128,256}
 *   Wq  [N, K/2] int8 output, contiguous rows, 16-byte aligned
 *   sw  [N] fp32 output
 */
int w4a4_quantize_weight(const float* W, int64_t N, int64_t K, int64_t ldw, int g,
                         int8_t* Wq, float* sw, void* stream);

/*
 * Run-time activation preparation: the page's Description fuses the
 * Hadamard rotation, the per-row int4 quantisation and the packing into one
 * kernel, and so does this call.
 *   x   [M, K] bf16 bits, row stride ldx >= K, 16-byte aligned, ldx % 8 == 0
 *   act 0: none; 1: exact-erf GELU applied to x before the rotation (used to
 *       feed an MLP down projection from the up projection's output).  The
 *       first act = 1 call on a device uploads a table of the normal CDF
 *       (15 KB, synchronously); make that first call before any stream
 *       capture.
 *   Xq  [M, K/2] int8 output (contiguous rows, 16-byte aligned); sx [M] fp32
 *   M >= 0 (M == 0 is a no-op); K % 128 == 0, K % g == 0, 128 <= K <= 32768.
 * A row that is all zero gets sx = 0 and all-zero codes.
 */
int w4a4_quantize_activation(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g,
                             int act, int8_t* Xq, float* sx, void* stream);

/*
 * w4a4_quantize_activation with the kernel chosen by the caller, for tests
 * and measurements (both kernels compute the same page's rotation,
 * quantisation and packing; they differ only in the order of the fp32
 * additions of the rotation).
 *   path 0: the routing of w4a4_quantize_activation (see
 *           w4a4_quantize_activation_kernel);
 *   path 1: the register-butterfly kernel (every shape);
 *   path 2: the tensor-core kernel, for act = 0, g in {64, 128} and
 *           K / g <= 128 (W4A4_ERR_SHAPE otherwise).
 * Any other path gives W4A4_ERR_ARG.  Other arguments as above.
 */
int w4a4_quantize_activation_path(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g,
                                  int act, int8_t* Xq, float* sx, int path, void* stream);

/* The kernel w4a4_quantize_activation (and the fused entries) run for this
 * shape, as a path number of w4a4_quantize_activation_path (1 or 2); 0 for
 * an invalid shape.  Pure host function; it reads the environment switches
 * above. */
int w4a4_quantize_activation_kernel(int64_t M, int64_t K, int g, int act);

/*
 * W4A4 linear on already-quantised operands: the s4 x s4 GEMM with int32
 * accumulation and the rank-one epilogue of the page's Description (the row
 * and column scales are applied once per output, after the K loop).
 *   Xq [M, K/2] int8, sx [M] fp32 (from w4a4_quantize_activation)
 *   Wq [N, K/2] int8, sw [N] fp32 (from w4a4_quantize_weight)
 *   bias [N] bf16 bits or NULL
 *   y  [M, N] bf16 bits output, row stride ldy >= N, ldy % 8 == 0, 16-byte aligned
 *   M >= 0, N >= 1, N % 8 == 0, 32 <= K <= 131072, K % 32 == 0; Xq/Wq 16-byte aligned
 *   workspace, workspace_bytes: reserved; no kernel needs scratch memory
 *       (w4a4_workspace_bytes returns 0), so both may be NULL / 0.
 * M = 1, or M <= 4 with M*K <= 12288, takes a weight-streaming kernel on
 * the CUDA cores (dp4a on widened nibbles), M <= 64 the weight-streaming split-K
 * tensor-core kernel (K slices reduced on chip within a CTA cluster), larger
 * M the tcgen05 tensor-core kernel; all give bit-identical int32
 * accumulators.
 */
int w4a4_linear(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw,
                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K,
                int64_t ldy, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Fused layer: w4a4_quantize_activation followed by w4a4_linear, with the
 * packed activation and its scales kept in the workspace.
 *   x [M, K] bf16 bits with row stride ldx; other arguments as above.
 *   workspace: at least w4a4_fused_workspace_bytes(M, N, K) bytes, 256-byte
 *       aligned, laid out as [packed x][sx]; its contents need no
 *       initialisation.  Calls that share one workspace must be ordered on the
 *       same stream.
 */
int w4a4_linear_fused(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw,
                      const uint16_t* bias, uint16_t* y, int64_t ldy, int64_t M, int64_t N,
                      int64_t K, int g, int act, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Which GEMM kernel w4a4_linear and w4a4_linear_fused run for this shape,
 * numbered as w4a4_gemm_s32's path: 0 = tcgen05 tensor-core kernel, 1 =
 * small-M split-K kernel, 3 = tiny-M CUDA-core kernel.  Pure host function;
 * it reads the environment switches above. */
int w4a4_linear_kernel(int64_t M, int64_t N, int64_t K);

/* Workspace sizes in bytes (0 when none is needed: w4a4_workspace_bytes is
 * always 0).  Pure host functions. */
size_t w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K);
size_t w4a4_fused_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Raw int32 accumulators acc[m, n] = sum_k qx[m,k] * qw[n,k] (no epilogue),
 * for bit-exact checks of the GEMM.  path: 0 = tcgen05 tensor-core kernel,
 * 1 = small-M weight-streaming kernel (M <= 64 only), 2 = a comparison
 * kernel in the pages' own design (warp-level mma.m16n8k64.s4 fed from
 * shared memory), kept to measure the tcgen05 kernel against, 3 = tiny-M
 * CUDA-core weight-streaming kernel (M <= 4, M*K <= 96 KiB; W4A4_ERR_SHAPE
 * otherwise).
 *   acc [M, N] int32 output with row stride ldc >= N, ldc % 4 == 0.
 * Other rules as for w4a4_linear.
 */
int w4a4_gemm_s32(const int8_t* Xq, const int8_t* Wq, int32_t* acc, int64_t M, int64_t N,
                  int64_t K, int64_t ldc, int path, void* workspace, size_t workspace_bytes,
                  void* stream);

/*
 * The fused layer of w4a4_linear_fused for callers that cannot allocate
 * device memory.  The pages have no counterpart to this entry point.  The
 * fused layer needs scratch memory between its two kernels (the packed
 * activation and its row scales); w4a4_linear_fused takes it from the
 * caller as a workspace, but some callers cannot provide one: a plug-in
 * whose host framework owns every byte of device memory and hands a custom
 * op only its inputs and outputs, or a serving loop that must not call
 * cudaMalloc once it runs (an allocation can synchronise the device and
 * fragment a pool sized in advance).  This entry point keeps that scratch in
 * a fixed 8 MiB array inside the library instead, and neither allocates nor
 * frees anything.
 *   Arguments, layouts and results are those of w4a4_linear_fused without
 *   the workspace; the output is bit-identical to it.
 *   Size limit: the scratch must hold round256(M * K / 2) + round256(4 * M)
 *   bytes (w4a4_fused_workspace_bytes), at most 8 MiB -- e.g. M = 4608 at
 *   K = 3072, or any M <= 64 at K <= 32768.  Larger shapes return
 *   W4A4_ERR_SHAPE before anything is launched.
 *   The array exists once per GPU on which the library is loaded and holds
 *   its 8 MiB until the process exits.  The first call on a device looks up
 *   the array's device address (a CUDA runtime query, no allocation); make
 *   that first call before any stream capture.
 *   Every call on a device shares the one array, and it keeps the last
 *   call's contents (nothing needs to start at zero: the activation kernel
 *   writes all of it before the GEMM reads it).  Calls that overlap on the
 *   GPU -- on different streams, or from different host threads -- race on
 *   the array and give wrong results: order them on one stream.
 */
int w4a4_linear_fused_noalloc(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw,
                              const uint16_t* bias, uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                              int g, int act, void* stream);

/*
 * Layer chains: the fused layer (w4a4_linear_fused) together with the
 * quantised input of the layer after it, taken from GELU of this layer's
 * output -- what w4a4_quantize_activation(y, M, N, ldy, g_next, act = 1, ...)
 * returns (page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused
 * CUDA kernels", Description: the activation pass -- rotate, one int4 scale
 * per row, pack -- here applied to the layer's own output).  The row scale
 * needs the amax of a whole output row, which many output tiles produce, so
 * it runs in two passes: the GEMM's epilogue applies GELU and the rotation to
 * every output tile it has just written and records, per row, the largest
 * rotated magnitude over the tile's columns (atomic maxima in the
 * workspace); a streaming kernel then rotates and quantises y with the row
 * amax already known (no row reduction).  This entry has no counterpart in
 * the pages, whose layers quantise their input in a pass of their own.
 *   Arguments as for w4a4_linear_fused, plus:
 *   g_next   rotation group of the next layer, in {64, 128, 256}; N is the
 *            next layer's K: N % 128 == 0, N % g_next == 0, N <= 32768
 *   Xq_next  [M, N / 2] packed int4 codes (16-byte aligned), written
 *   sx_next  [M] fp32 row scales, written
 *   workspace: w4a4_fused_requant_workspace_bytes(M, N, K) bytes, 256-byte
 *       aligned (the activation codes of x, their scales and the row amax
 *       slots; the call sets the slots to zero itself).
 *   The first call on a device uploads the GELU table as w4a4_quantize_
 *   activation with act = 1 does: make it before any stream capture.
 * y is bit-identical to w4a4_linear_fused's.  Xq_next and sx_next match the
 * one-pass activation kernel up to the rounding of the rotated values (both
 * passes form GELU with its table; the rotation is summed in another order).
 * Batches that w4a4_linear_kernel routes to the
 * weight-streaming kernels (M <= 64) run the layer and then the one-pass
 * activation kernel on y.
 */
size_t w4a4_fused_requant_workspace_bytes(int64_t M, int64_t N, int64_t K);
int w4a4_linear_fused_requant(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw,
                              const uint16_t* bias, uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                              int g, int act, int g_next, int8_t* Xq_next, float* sx_next, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Dynamic LoRA (page "Comfy-INT4-HIPtest README", section "LoRA modes":
 * Dynamic keeps the LoRA matrices separate and applies their deltas at
 * inference time; page "ComfyUI-INT4-Fast", "Dynamic LoRA Patching": the
 * down projection is rotated into the layer's Hadamard basis).  Adds
 *     y[m, n] += scale * sum_j t[m, j] B[n, j],   t = x_rot A_rot^T = x A^T
 * to an existing bf16 output: the rotation is orthogonal, so the rotated
 * activation against the rotated down projection equals the plain product,
 * which the kernels form from the bf16 activation and the unrotated A.
 *   x [M, K] bf16 bits, row stride ldx >= K, ldx % 8 == 0 (the layer's input)
 *   A [r, K] bf16 bits (the down projection, contiguous rows)
 *   B [N, r] bf16 bits (the up projection, contiguous rows)
 *   r in {16, 32, 48, 64};  scale finite (e.g. alpha / r)
 *   y [M, N] bf16 bits, row stride ldy >= N, ldy % 8 == 0; updated in place:
 *       y = bf16(fma(scale, delta, y)) with delta accumulated in fp32 from
 *       bf16 t (t itself accumulated in fp32 from bf16 products)
 *   M >= 0, N % 8 == 0, K % 8 == 0;  every pointer 16-byte aligned
 *   workspace: at least w4a4_lora_workspace_bytes(M, K) bytes, 256-byte
 *       aligned: t as [M, 64] bf16, then the fp32 partial sums of the down
 *       projection's K slices; no initialisation needed.
 */
size_t w4a4_lora_workspace_bytes(int64_t M, int64_t K);
int w4a4_lora_add(const uint16_t* x, int64_t ldx, const uint16_t* A, const uint16_t* B, int r, float scale,
                  uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * The fused layer (w4a4_linear_fused, act = 0) followed by the Dynamic LoRA
 * update of w4a4_lora_add on its output.  Arguments as for those two calls;
 * the workspace holds both (w4a4_fused_lora_workspace_bytes(M, N, K) bytes,
 * 256-byte aligned).  GELU inputs (act = 1) are not supported here.
 */
size_t w4a4_fused_lora_workspace_bytes(int64_t M, int64_t N, int64_t K);
int w4a4_linear_fused_lora(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw,
                           const uint16_t* bias, const uint16_t* A, const uint16_t* B, int r, float scale,
                           uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, int g,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the device status word that
 * kernels set when a bounded wait expires.  Returns W4A4_OK,
 * W4A4_ERR_TIMEOUT, or W4A4_ERR_CUDA if the synchronisation failed.
 */
int w4a4_last_device_error(void* stream);

/*
 * Test hook for the bounded waits of the product kernels: every kernel
 * launched after this call (in this process, on any device) gives up a wait
 * that has not ended after `limit_ns` nanoseconds, records W4A4_ERR_TIMEOUT
 * in the device status word, stops every role, drains its copies and MMAs,
 * frees its tensor memory and exits; its outputs are then undefined.  A
 * limit of a few nanoseconds makes most waits expire at once.  0 restores
 * the default of 2 s; values above 2 s or below 0 give W4A4_ERR_ARG.  Not
 * for production use: it is process-wide and not synchronised with launches
 * on other host threads.
 */
int w4a4_debug_set_wait_limit(int64_t limit_ns);

/*
 * Test hook for the bounded-wait machinery: launches one CTA whose only
 * thread waits on an mbarrier that nothing ever arrives on, with a wait
 * limit of `timeout_us` microseconds (1..1000000).  The kernel must record
 * W4A4_ERR_TIMEOUT and return; it never traps or hangs.
 */
int w4a4_debug_wait_timeout(int64_t timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A4_H_ */
