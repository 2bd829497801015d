// Internal launch interfaces shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace w4a4 {

// ---- shared host helpers (api.cu)
struct DeviceInfo {
  int checked = 0;     // 0 unknown, 1 supported, -1 unsupported
  int num_sms = 0;
  unsigned int* status = nullptr;   // device address of the status word
};
// The current device (must be sm_100); W4A4_OK or an error status.
int current_device(DeviceInfo** out);
// How long the kernels' bounded waits spin before they give up: kWaitLimitNs
// (2 s), or the value set by w4a4_debug_set_wait_limit.
unsigned long long wait_limit_ns();
// TMA map over a packed int4 matrix [rows, K/2] bytes with box {64, box_rows}
// (64-byte swizzle in shared memory when swizzle64).
int packed_map(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows, bool swizzle64 = false);
// TMA map over bf16 rows [M, K] (row stride ldx) viewed as [M][K/g][g], box
// {64, K/g, rows_per_tile}, 128-byte swizzle (the tensor-core rotation's A tiles).
int group_rows_map(CUtensorMap* map, const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g, int rows_per_tile);
// Argument checks of w4a4_linear (out_s32 = 0) / w4a4_gemm_s32 (out_s32 = 1).
int validate_linear(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                    const void* y, int64_t M, int64_t N, int64_t K, int64_t ldy, int out_s32);
// Argument checks of w4a4_linear_fused (no CUDA call).
int validate_fused(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                   const uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, int g, int act);

// ---- activation / weight rotate + quantise + pack (quant.cu)
// path: 0 = the routing of w4a4_quantize_activation, 1 = the register-butterfly
// kernel, 2 = the tensor-core kernel (cudaErrorNotSupported where it does not apply).
cudaError_t rotate_quant_bf16(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                              float* scale, int num_sms, unsigned int* status, cudaStream_t stream, int path = 0);
// Which kernel path 0 picks: 1 (register butterflies) or 2 (tensor cores).
int rotate_quant_bf16_route(int64_t M, int K, int g, int act);
// Codes and row scales of GELU(y) for the next layer, rotation group g, from
// a bf16 y [M, K] (row stride ldy, 16-byte aligned rows) and the row amax of
// the rotated values as fp32 bits (amax [M], from the GEMM's requantising
// epilogue).  K % g == 0, K % 128 == 0.
// Device address of the GELU table (gelu_table.cuh), filled on first use;
// the first call on a device must not be inside a stream capture.
cudaError_t gelu_table_device(const float** table);
cudaError_t requant_bf16(const uint16_t* y, int64_t M, int K, int64_t ldy, int g, const unsigned int* amax,
                         int8_t* out, float* scale, int num_sms, cudaStream_t stream);
cudaError_t rotate_quant_f32(const float* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                             int num_sms, unsigned int* status, cudaStream_t stream);
// Tensor-core form of rotate_quant_bf16 for act = 0, g in {64, 128} and
// K / g <= 128 (quant_tc.cu); returns cudaErrorNotSupported for other shapes.
cudaError_t rotate_quant_bf16_tc(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                                 int num_sms, unsigned int* status, cudaStream_t stream);
// Largest K the in-register rotate kernel supports: 512 threads x 64 codes
// per row for bf16 rows; fp32 rows (weights) are limited by two ring stages
// of one row in shared memory (2 x 96 KB).
constexpr int kQuantMaxK = 512 * 64;
constexpr int kQuantMaxKF32 = 384 * 64;

// ---- tcgen05 GEMM (gemm.cu)
struct GemmArgs {
  int64_t M, N, K;        // K in int4 elements
  const float* sx;        // [M]
  const float* sw;        // [N]
  const uint16_t* bias;   // [N] bf16 bits or nullptr
  void* out;              // bf16 bits [M, ldo] or int32 [M, ldo]
  int64_t ldo;
  int out_s32;            // 1: raw int32 accumulators
  unsigned int* status;   // device status word (bounded-wait timeouts)
  unsigned long long wait_ns;   // bounded-wait limit (wait_limit_ns())
  // Requantising epilogue for a following layer (0: off; else its rotation
  // group 64, 128 or 256): per row, atomicMax of fp32 bits of the amax of
  // rotate(GELU(y)) over each tile's columns into chain_amax [M] (zeroed
  // before the launch).
  int chain_g;
  unsigned int* chain_amax;
  const float* gelu_tab;   // the GELU table in device memory (gelu_table_device)
};
// tmA: packed activations [M, K/2] bytes, tmB: packed weights [N, K/2] bytes,
// both with box {64 bytes, kGemmBM/2 rows}; tmY: bf16 output [M, N] (row
// stride ldo) with box {32, 32} and 64-byte swizzle (unused for int32 output).
// Launched as clusters of 2 CTAs.
cudaError_t gemm_tc_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY, const GemmArgs& a,
                           int num_sms, cudaStream_t stream);
// Comparison kernel in the pages' warp-level mma.m16n8k64.s4 design (raw int32
// accumulators only); tmA / tmB: packed operands, box {64 bytes, 128 rows},
// 64-byte swizzle.
cudaError_t gemm_legacy_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, int32_t* out, int64_t M, int64_t N,
                               int64_t K, int64_t ldo, unsigned int* status, cudaStream_t stream);
constexpr int kGemmBM = 256;
constexpr int kGemmBN = 256;

// ---- small-M weight-streaming GEMM (smallm.cu)
struct SmallMArgs {
  const int8_t* xq;       // [M, K/2]
  const int8_t* wq;       // [N, K/2]
  int64_t M, N, K;
  const float* sx;
  const float* sw;
  const uint16_t* bias;
  void* out;
  int64_t ldo;
  int out_s32;
  unsigned int* status;   // device status word
  unsigned long long wait_ns;   // bounded-wait limit (wait_limit_ns())
  int num_sms;            // SMs of the device (the split plan keeps every cluster resident)
  // 1: the packed weights (and their scales) were complete before this
  // kernel started, so it may read them before its grid-dependency wait (set
  // by the fused entry, whose previous kernel is its own activation
  // quantiser, which lets its dependents start only after its own wait); 0:
  // read nothing before the wait
  int early_w;
};
// tmW: packed weights [N, K/2] bytes, box {64, 128}, 64-byte swizzle; tmX:
// packed activations [M, K/2] bytes, box {64, smallm_rows_padded(M)}.
// Launched as clusters of up to 8 CTAs (one cluster per 128-row weight tile,
// one CTA per K slice); needs no workspace.
cudaError_t smallm_launch_tm(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a,
                             cudaStream_t stream);
int smallm_rows_padded(int64_t M);
constexpr int kSmallMMax = 64;

// ---- Dynamic LoRA (lora.cu)
// Largest LoRA rank; t is stored as [M, 64] bf16 (row stride 64, zero beyond r).
constexpr int kLoraMaxRank = 64;
// t[M, r] = x[M, K] A[r, K]^T (bf16 in, fp32 accumulation, bf16 out); the K
// slices' fp32 partial sums go through `partial` (lora_slices(M, K) x M x 64
// floats).
int lora_slices(int64_t M, int64_t K);
cudaError_t lora_down_launch(const uint16_t* x, int64_t ldx, const uint16_t* A, float* partial, uint16_t* t,
                             int64_t M, int64_t K, int r, unsigned int* status, cudaStream_t stream);
// y[M, N] = bf16(y + scale * t B^T), B [N, r] bf16.
cudaError_t lora_up_launch(const uint16_t* t, const uint16_t* B, uint16_t* y, int64_t ldy, int64_t M, int64_t N,
                           int r, float scale, int num_sms, unsigned int* status, cudaStream_t stream);
// Generic 2-D TMA map: [rows, cols] elements, row stride in bytes, box
// {box_cols, box_rows}; out-of-range elements read as zero.
int tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t rows, int64_t cols,
                  int64_t row_stride_bytes, int box_cols, int box_rows, CUtensorMapSwizzle swizzle);

// ---- tiny-M weight streaming on the CUDA cores (gemv.cu)
struct GemvArgs {
  const int8_t* xq;       // [M, K/2]
  const float* sx;        // [M]
  const int8_t* wq;       // [N, K/2]
  const float* sw;        // [N]
  const uint16_t* bias;   // [N] bf16 bits or NULL
  void* out;              // y [M, ldo] bf16, or acc [M, ldo] int32 when out_s32
  int64_t M, N, K, ldo;
  int out_s32;
  int early_w;            // as SmallMArgs::early_w
};
constexpr int kGemvMaxM = 4;
// widened activations (M * K bytes) live in one CTA's shared memory
constexpr size_t kGemvMaxSmem = 96 * 1024;
inline bool gemv_fits(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvMaxM && static_cast<size_t>(M) * static_cast<size_t>(K) <= kGemvMaxSmem;
}
// The shapes the linear entries route to it: measured against the split-K
// tensor-core kernel (CUDA-graph replay, N x K in {12288 x 3072, 3072 x 12288,
// 5120^2, 3072^2}) it is faster for every M = 1 shape (6.2 vs 10.7 us at
// 12288 x 3072) and whenever M * K <= 12288; above that each weight byte
// costs too many shared-memory reads of the activations.
inline bool gemv_preferred(int64_t M, int64_t K) { return gemv_fits(M, K) && (M == 1 || M * K <= 12288); }
cudaError_t gemv_launch(const GemvArgs& a, int num_sms, cudaStream_t stream);

}  // namespace w4a4
