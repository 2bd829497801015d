// C ABI of the W4A4 library: argument validation, device checks, TMA tensor
// maps and dispatch to the kernels.  Every check that needs no GPU runs before
// the first CUDA call, so invalid arguments are reported even on a machine
// without a device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "w4a4.h"
#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {

// Device status word (bounded-wait timeouts); one copy per device context.
__device__ unsigned int g_device_status = 0;

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
std::atomic<unsigned long long> g_wait_limit_ns{kWaitLimitNs};
}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

// Resolve the current device; fills its SM count and the device address of
// the status word on first use.
int current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return W4A4_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return W4A4_ERR_CUDA;
    if (major != 10 || minor != 0) {
      d.checked = -1;
    } else {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return W4A4_ERR_CUDA;
      d.status = static_cast<unsigned int*>(p);
      d.num_sms = sms;
      d.checked = 1;
    }
  }
  if (d.checked < 0) return W4A4_ERR_DEVICE;
  *out = &d;
  return W4A4_OK;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// 2-D map over a packed int4 matrix [rows, K/2] bytes, box {64 bytes, box_rows};
// out-of-range rows and columns read as zero.  swizzle64: the box lands in
// shared memory with the 64-byte swizzle (16-byte chunk j of row r at
// j ^ ((r >> 1) & 3)), for readers that take one row per thread.
int packed_map(CUtensorMap* map, const int8_t* base, int64_t rows, int64_t K, int box_rows, bool swizzle64) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return W4A4_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

// 3-D map over bf16 rows x [M, K] (row stride ldx elements) viewed as
// [M][K/g][g]: box {64 elements, K/g groups, rows_per_tile rows}, 128-byte
// swizzle, so one box lands as rows_per_tile * K/g consecutive 128-byte
// rows (group j of row p at row p * K/g + j); rows past M read as zero.
int group_rows_map(CUtensorMap* map, const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g, int rows_per_tile) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return W4A4_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(g), static_cast<cuuint64_t>(K / g), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(g) * 2, static_cast<cuuint64_t>(ldx) * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(K / g), static_cast<cuuint32_t>(rows_per_tile)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

int tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t rows, int64_t cols,
                  int64_t row_stride_bytes, int box_cols, int box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return W4A4_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

namespace {

// 2-D map over a bf16 output [rows, cols] with row stride ld (elements), box
// {32, 32}, 64-byte swizzle (the epilogue's staging layout).
int output_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, int64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return W4A4_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  const cuuint32_t box[2] = {32u, 32u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline size_t round256(size_t b) { return (b + 255) / 256 * 256; }

int smallm_threshold() {
  static int v = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    v = kSmallMMax;
    const char* e = std::getenv("W4A4_SMALLM_MAX");
    if (e != nullptr) {
      const long x = std::strtol(e, nullptr, 10);
      if (x >= 0 && x <= kSmallMMax) v = static_cast<int>(x);
    }
  });
  return v;
}

// The weight-streaming kernels by batch size: the CUDA-core one for a few
// rows, the split-K tensor-core one up to smallm_threshold(), else the
// tcgen05 GEMM.
int linear_path(int64_t M, int64_t K) {
  const int64_t small = smallm_threshold();
  if (M <= small && gemv_preferred(M, K)) return 3;
  return M <= small ? 1 : 0;
}

int check_quant_shape(int64_t K, int g) {
  if (g != 64 && g != 128 && g != 256) return W4A4_ERR_GROUP;
  if (K < 128 || K > kQuantMaxK || K % 128 != 0) return W4A4_ERR_SHAPE;
  if (K % g != 0) return W4A4_ERR_GROUP;
  return W4A4_OK;
}

int check_gemm_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || M > (int64_t(1) << 26)) return W4A4_ERR_SHAPE;
  if (N < 1 || N % 8 != 0 || N > (int64_t(1) << 24)) return W4A4_ERR_SHAPE;
  // K <= 2^17 keeps the widened accumulator 256*acc (|.| <= 12544*K) in int32
  if (K < 32 || K % 32 != 0 || K > (int64_t(1) << 17)) return W4A4_ERR_SHAPE;
  return W4A4_OK;
}


// Shared body of w4a4_linear / w4a4_gemm_s32 after validation.  path 0: the
// tcgen05 tensor-core kernel; 1: the small-M weight-streaming kernel; 2: the
// warp-level mma.sync comparison kernel (int32 output only); 3: the tiny-M
// weight-streaming kernel on the CUDA cores.
int run_linear(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw, const uint16_t* bias, void* out,
               int64_t M, int64_t N, int64_t K, int64_t ldo, int out_s32, int path, cudaStream_t stream,
               int early_w = 0, int chain_g = 0, unsigned int* chain_amax = nullptr) {
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  if (path == 3) {
    GemvArgs a{};
    a.xq = Xq;
    a.sx = sx;
    a.wq = Wq;
    a.sw = sw;
    a.bias = bias;
    a.out = out;
    a.M = M;
    a.N = N;
    a.K = K;
    a.ldo = ldo;
    a.out_s32 = out_s32;
    a.early_w = early_w;
    return gemv_launch(a, dev->num_sms, stream) == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
  }
  if (path == 2) {
    CUtensorMap tmA, tmB;
    if ((st = packed_map(&tmA, Xq, M, K, 128, true)) != W4A4_OK) return st;
    if ((st = packed_map(&tmB, Wq, N, K, 128, true)) != W4A4_OK) return st;
    return gemm_legacy_launch(tmA, tmB, static_cast<int32_t*>(out), M, N, K, ldo, dev->status, stream) == cudaSuccess
               ? W4A4_OK
               : W4A4_ERR_CUDA;
  }
  if (path == 1) {
    CUtensorMap tmW, tmX;
    if ((st = packed_map(&tmW, Wq, N, K, 128, true)) != W4A4_OK) return st;
    if ((st = packed_map(&tmX, Xq, M, K, smallm_rows_padded(M))) != W4A4_OK) return st;
    SmallMArgs a{};
    a.xq = Xq;
    a.wq = Wq;
    a.M = M;
    a.N = N;
    a.K = K;
    a.sx = sx;
    a.sw = sw;
    a.bias = bias;
    a.out = out;
    a.ldo = ldo;
    a.out_s32 = out_s32;
    a.status = dev->status;
    a.wait_ns = wait_limit_ns();
    a.num_sms = dev->num_sms;
    a.early_w = early_w;
    return smallm_launch_tm(tmW, tmX, a, stream) == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
  }
  CUtensorMap tmA, tmB, tmY;
  if ((st = packed_map(&tmA, Xq, M, K, kGemmBM / 2)) != W4A4_OK) return st;
  if ((st = packed_map(&tmB, Wq, N, K, kGemmBN / 2)) != W4A4_OK) return st;
  if (out_s32) {
    tmY = tmA;   // not read by the int32 epilogue
  } else if ((st = output_map(&tmY, out, M, N, ldo)) != W4A4_OK) {
    return st;
  }
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.sx = sx;
  a.sw = sw;
  a.bias = bias;
  a.out = out;
  a.ldo = ldo;
  a.out_s32 = out_s32;
  a.status = dev->status;
  a.wait_ns = wait_limit_ns();
  a.chain_g = chain_g;
  a.chain_amax = chain_amax;
  a.gelu_tab = nullptr;
  if (chain_g != 0 && gelu_table_device(&a.gelu_tab) != cudaSuccess) return W4A4_ERR_CUDA;
  return gemm_tc_launch(tmA, tmB, tmY, a, dev->num_sms, stream) == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

__global__ void wait_forever_bounded_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    // nothing ever arrives: the wait must expire and record a timeout
    (void)mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  }
}

}  // namespace

int validate_linear(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw,
                           const uint16_t* bias, const void* y, int64_t M, int64_t N, int64_t K, int64_t ldy,
                           int out_s32) {
  if (Wq == nullptr || (!out_s32 && sw == nullptr)) return W4A4_ERR_NULL;
  // an empty batch (M == 0) may pass NULL for its zero-size tensors
  if (M != 0 && (Xq == nullptr || y == nullptr || (!out_s32 && sx == nullptr))) return W4A4_ERR_NULL;
  int st = check_gemm_shape(M, N, K);
  if (st != W4A4_OK) return st;
  if (ldy < N) return W4A4_ERR_SHAPE;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(y, 16)) return W4A4_ERR_ALIGN;
  if (out_s32) {
    if (ldy % 4 != 0) return W4A4_ERR_ALIGN;
  } else {
    if (ldy % 8 != 0 || !aligned(sw, 16) || !aligned(sx, 4)) return W4A4_ERR_ALIGN;
    if (bias != nullptr && !aligned(bias, 16)) return W4A4_ERR_ALIGN;
  }
  return W4A4_OK;
}

int validate_fused(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                   const uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, int g, int act) {
  if (Wq == nullptr || sw == nullptr) return W4A4_ERR_NULL;
  // an empty batch (M == 0) may pass NULL for its zero-size tensors
  if (M != 0 && (x == nullptr || y == nullptr)) return W4A4_ERR_NULL;
  int st = check_quant_shape(K, g);
  if (st != W4A4_OK) return st;
  if (act != 0 && act != 1) return W4A4_ERR_ARG;
  if ((st = check_gemm_shape(M, N, K)) != W4A4_OK) return st;
  if (ldx < K || ldy < N) return W4A4_ERR_SHAPE;
  if (ldx % 8 != 0 || !aligned(x, 16)) return W4A4_ERR_ALIGN;
  if (ldy % 8 != 0 || !aligned(y, 16) || !aligned(Wq, 16) || !aligned(sw, 16)) return W4A4_ERR_ALIGN;
  if (bias != nullptr && !aligned(bias, 16)) return W4A4_ERR_ALIGN;
  return W4A4_OK;
}

}  // namespace w4a4

using namespace w4a4;

extern "C" {

const char* w4a4_status_string(int status) {
  switch (status) {
    case W4A4_OK: return "W4A4_OK";
    case W4A4_ERR_NULL: return "W4A4_ERR_NULL: a required pointer is NULL";
    case W4A4_ERR_SHAPE: return "W4A4_ERR_SHAPE: a size is out of range or breaks a multiple rule";
    case W4A4_ERR_GROUP: return "W4A4_ERR_GROUP: group size not in {64,128,256} or does not divide K";
    case W4A4_ERR_ALIGN: return "W4A4_ERR_ALIGN: pointer or leading dimension misaligned";
    case W4A4_ERR_WORKSPACE: return "W4A4_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case W4A4_ERR_DEVICE: return "W4A4_ERR_DEVICE: the current device is not an sm_100 GPU";
    case W4A4_ERR_CUDA: return "W4A4_ERR_CUDA: a CUDA call or kernel launch failed";
    case W4A4_ERR_TIMEOUT: return "W4A4_ERR_TIMEOUT: a kernel gave up waiting";
    case W4A4_ERR_ARG: return "W4A4_ERR_ARG: invalid argument";
    default: return "W4A4: unknown status";
  }
}

int w4a4_version(void) { return 100; }

int w4a4_quantize_weight(const float* W, int64_t N, int64_t K, int64_t ldw, int g, int8_t* Wq, float* sw,
                         void* stream) {
  if (W == nullptr || Wq == nullptr || sw == nullptr) return W4A4_ERR_NULL;
  int st = check_quant_shape(K, g);
  if (st != W4A4_OK) return st;
  if (K > kQuantMaxKF32) return W4A4_ERR_SHAPE;
  if (N < 1 || N > (int64_t(1) << 26)) return W4A4_ERR_SHAPE;
  if (ldw < K) return W4A4_ERR_SHAPE;
  if (ldw % 4 != 0 || !aligned(W, 16) || !aligned(Wq, 16) || !aligned(sw, 4)) return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  return rotate_quant_f32(W, N, static_cast<int>(K), ldw, g, Wq, sw, dev->num_sms, dev->status,
                          static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? W4A4_OK
             : W4A4_ERR_CUDA;
}

int w4a4_quantize_activation(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g, int act, int8_t* Xq,
                             float* sx, void* stream) {
  return w4a4_quantize_activation_path(x, M, K, ldx, g, act, Xq, sx, 0, stream);
}

int w4a4_quantize_activation_kernel(int64_t M, int64_t K, int g, int act) {
  if (check_quant_shape(K, g) != W4A4_OK || (act != 0 && act != 1) || M < 0) return 0;
  return rotate_quant_bf16_route(M, static_cast<int>(K), g, act);
}

int w4a4_quantize_activation_path(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int g, int act, int8_t* Xq,
                                  float* sx, int path, void* stream) {
  // an empty batch (M == 0) may pass NULL for its zero-size tensors
  if (M != 0 && (x == nullptr || Xq == nullptr || sx == nullptr)) return W4A4_ERR_NULL;
  int st = check_quant_shape(K, g);
  if (st != W4A4_OK) return st;
  if (act != 0 && act != 1) return W4A4_ERR_ARG;
  if (path < 0 || path > 2) return W4A4_ERR_ARG;
  // the tensor-core rotation: bf16 rows without GELU, g in {64, 128}, K/g <= 128
  if (path == 2 && (act != 0 || g == 256 || K / g > 128)) return W4A4_ERR_SHAPE;
  if (M < 0 || M > (int64_t(1) << 26)) return W4A4_ERR_SHAPE;
  if (ldx < K) return W4A4_ERR_SHAPE;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(Xq, 16) || !aligned(sx, 4)) return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  return rotate_quant_bf16(x, M, static_cast<int>(K), ldx, g, act, Xq, sx, dev->num_sms, dev->status,
                           static_cast<cudaStream_t>(stream), path) == cudaSuccess
             ? W4A4_OK
             : W4A4_ERR_CUDA;
}

// No kernel of the linear needs a workspace any more (the small-M kernel
// reduces its K slices on chip); the workspace arguments of w4a4_linear and
// w4a4_gemm_s32 are kept for ABI stability and may be NULL.
int w4a4_linear_kernel(int64_t M, int64_t N, int64_t K) {
  (void)N;
  return linear_path(M, K);
}

size_t w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;
}

// The fused workspace holds the packed activation and its scales.
static size_t fused_codes_bytes(int64_t M, int64_t K) {
  return round256(static_cast<size_t>(M) * static_cast<size_t>(K / 2));
}

size_t w4a4_fused_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return fused_codes_bytes(M, K) + round256(static_cast<size_t>(M) * 4);
}

int w4a4_linear(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t ldy, void* workspace, size_t workspace_bytes,
                void* stream) {
  int st = validate_linear(Xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0);
  if (st != W4A4_OK) return st;
  const int path = linear_path(M, K);
  (void)workspace;
  (void)workspace_bytes;
  return run_linear(Xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0, path, static_cast<cudaStream_t>(stream));
}

int w4a4_gemm_s32(const int8_t* Xq, const int8_t* Wq, int32_t* acc, int64_t M, int64_t N, int64_t K, int64_t ldc,
                  int path, void* workspace, size_t workspace_bytes, void* stream) {
  int st = validate_linear(Xq, nullptr, Wq, nullptr, nullptr, acc, M, N, K, ldc, 1);
  if (st != W4A4_OK) return st;
  if (path < 0 || path > 3) return W4A4_ERR_ARG;
  if (path == 1 && M > kSmallMMax) return W4A4_ERR_SHAPE;
  if (path == 3 && M != 0 && !gemv_fits(M, K)) return W4A4_ERR_SHAPE;
  (void)workspace;
  (void)workspace_bytes;
  return run_linear(Xq, nullptr, Wq, nullptr, nullptr, acc, M, N, K, ldc, 1, path, static_cast<cudaStream_t>(stream));
}

int w4a4_linear_fused(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                      uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, int g, int act, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int st = validate_fused(x, ldx, Wq, sw, bias, y, ldy, M, N, K, g, act);
  if (st != W4A4_OK) return st;
  if (M == 0) {
    DeviceInfo* dev = nullptr;
    return current_device(&dev);
  }
  const size_t need = w4a4_fused_workspace_bytes(M, N, K);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return W4A4_ERR_WORKSPACE;
  // Layout: [packed x][sx]
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* sx = reinterpret_cast<float*>(ws + fused_codes_bytes(M, K));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = w4a4_quantize_activation(x, M, K, ldx, g, act, xq, sx, stream)) != W4A4_OK) return st;
  const int path = linear_path(M, K);
  // The quantiser above lets the next kernel start only after its own
  // grid-dependency wait, i.e. once everything before it has finished, so
  // whatever wrote the weights is complete when the GEMM kernel starts: the
  // weight-streaming kernels may begin reading them before their own wait.
  return run_linear(xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0, path, s, 1);
}

// [packed x][sx][the next layer's row amax (fp32 bits)]
size_t w4a4_fused_requant_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return w4a4_fused_workspace_bytes(M, N, K) + round256(static_cast<size_t>(M) * 4);
}

int w4a4_linear_fused_requant(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                              uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, int g, int act, int g_next,
                              int8_t* Xq_next, float* sx_next, void* workspace, size_t workspace_bytes, void* stream) {
  int st = validate_fused(x, ldx, Wq, sw, bias, y, ldy, M, N, K, g, act);
  if (st != W4A4_OK) return st;
  if ((st = check_quant_shape(N, g_next)) != W4A4_OK) return st;   // N is the next layer's K
  if (Xq_next == nullptr || sx_next == nullptr) return W4A4_ERR_NULL;
  if (!aligned(Xq_next, 16) || !aligned(sx_next, 4)) return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  const size_t need = w4a4_fused_requant_workspace_bytes(M, N, K);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return W4A4_ERR_WORKSPACE;
  // Layout: [packed x][sx][amax]
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* sx = reinterpret_cast<float*>(ws + fused_codes_bytes(M, K));
  unsigned int* amax = reinterpret_cast<unsigned int*>(ws + w4a4_fused_workspace_bytes(M, N, K));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int path = linear_path(M, K);
  if (path != 0) {
    // the weight-streaming kernels of small batches have no requantising
    // epilogue: the layer, then the one-pass activation kernel on its output
    if ((st = w4a4_quantize_activation(x, M, K, ldx, g, act, xq, sx, stream)) != W4A4_OK) return st;
    if ((st = run_linear(xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0, path, s, 1)) != W4A4_OK) return st;
    return w4a4_quantize_activation(y, M, N, ldy, g_next, 1, Xq_next, sx_next, stream);
  }
  // the amax slots start at zero (atomic maxima of non-negative values); set
  // before the activation kernel so that it and the GEMM stay back to back
  if (cudaMemsetAsync(amax, 0, static_cast<size_t>(M) * 4, s) != cudaSuccess) return W4A4_ERR_CUDA;
  if ((st = w4a4_quantize_activation(x, M, K, ldx, g, act, xq, sx, stream)) != W4A4_OK) return st;
  if ((st = run_linear(xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0, 0, s, 1, g_next, amax)) != W4A4_OK) return st;
  return requant_bf16(y, M, static_cast<int>(N), ldy, g_next, amax, Xq_next, sx_next, dev->num_sms, s) == cudaSuccess
             ? W4A4_OK
             : W4A4_ERR_CUDA;
}

// [t: M x 64 bf16][the K slices' partial sums: slices x M x 64 fp32]
static size_t lora_t_bytes(int64_t M) { return round256(static_cast<size_t>(M) * kLoraMaxRank * 2); }

size_t w4a4_lora_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K <= 0) return 0;
  return lora_t_bytes(M) + static_cast<size_t>(lora_slices(M, K)) * static_cast<size_t>(M) * kLoraMaxRank * 4;
}

int w4a4_lora_add(const uint16_t* x, int64_t ldx, const uint16_t* A, const uint16_t* B, int r, float scale,
                  uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                  void* stream) {
  if (A == nullptr || B == nullptr) return W4A4_ERR_NULL;
  if (M != 0 && (x == nullptr || y == nullptr)) return W4A4_ERR_NULL;
  if (r < 16 || r > kLoraMaxRank || r % 16 != 0) return W4A4_ERR_SHAPE;
  if (M < 0 || M > (int64_t(1) << 26)) return W4A4_ERR_SHAPE;
  if (N < 1 || N % 8 != 0 || N > (int64_t(1) << 24)) return W4A4_ERR_SHAPE;
  if (K < 8 || K % 8 != 0 || K > (int64_t(1) << 20)) return W4A4_ERR_SHAPE;
  if (ldx < K || ldy < N) return W4A4_ERR_SHAPE;
  if (ldx % 8 != 0 || ldy % 8 != 0 || !aligned(x, 16) || !aligned(y, 16) || !aligned(A, 16) || !aligned(B, 16))
    return W4A4_ERR_ALIGN;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return W4A4_ERR_ARG;   // finite
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  if (workspace == nullptr || workspace_bytes < w4a4_lora_workspace_bytes(M, K) || !aligned(workspace, 256))
    return W4A4_ERR_WORKSPACE;
  uint16_t* t = static_cast<uint16_t*>(workspace);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lora_t_bytes(M));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (lora_down_launch(x, ldx, A, partial, t, M, K, r, dev->status, s) != cudaSuccess) return W4A4_ERR_CUDA;
  return lora_up_launch(t, B, y, ldy, M, N, r, scale, dev->num_sms, dev->status, s) == cudaSuccess ? W4A4_OK
                                                                                                   : W4A4_ERR_CUDA;
}

size_t w4a4_fused_lora_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return w4a4_fused_workspace_bytes(M, N, K) + w4a4_lora_workspace_bytes(M, K);
}

int w4a4_linear_fused_lora(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw, const uint16_t* bias,
                           const uint16_t* A, const uint16_t* B, int r, float scale, uint16_t* y, int64_t ldy,
                           int64_t M, int64_t N, int64_t K, int g, void* workspace, size_t workspace_bytes,
                           void* stream) {
  int st = validate_fused(x, ldx, Wq, sw, bias, y, ldy, M, N, K, g, 0);
  if (st != W4A4_OK) return st;
  if (A == nullptr || B == nullptr) return W4A4_ERR_NULL;
  if (r < 16 || r > kLoraMaxRank || r % 16 != 0) return W4A4_ERR_SHAPE;
  if (!aligned(A, 16) || !aligned(B, 16)) return W4A4_ERR_ALIGN;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return W4A4_ERR_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  const size_t base = w4a4_fused_workspace_bytes(M, N, K);
  if (workspace == nullptr || workspace_bytes < base + w4a4_lora_workspace_bytes(M, K) || !aligned(workspace, 256))
    return W4A4_ERR_WORKSPACE;
  uint16_t* t = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + base);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + base + lora_t_bytes(M));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The activation kernel reads x first; the down projection follows while
  // x is still in L2; then the GEMM (its packed activation and scales from the
  // workspace, as in w4a4_linear_fused) and the up projection, which adds to
  // the layer's output.
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* sx = reinterpret_cast<float*>(ws + fused_codes_bytes(M, K));
  if ((st = w4a4_quantize_activation(x, M, K, ldx, g, 0, xq, sx, stream)) != W4A4_OK) return st;
  if (lora_down_launch(x, ldx, A, partial, t, M, K, r, dev->status, s) != cudaSuccess) return W4A4_ERR_CUDA;
  // every kernel before the GEMM has finished when it starts (the reduction
  // kernel ahead of it completes before its dependents launch), so the
  // weight-streaming kernels may read the weights before their own wait
  if ((st = run_linear(xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0, linear_path(M, K), s, 1)) != W4A4_OK) return st;
  return lora_up_launch(t, B, y, ldy, M, N, r, scale, dev->num_sms, dev->status, s) == cudaSuccess ? W4A4_OK
                                                                                                   : W4A4_ERR_CUDA;
}

int w4a4_last_device_error(void* stream) {
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != W4A4_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return W4A4_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, dev->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return W4A4_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpy(dev->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return W4A4_ERR_CUDA;
    return W4A4_ERR_TIMEOUT;
  }
  return W4A4_OK;
}

int w4a4_debug_set_wait_limit(int64_t limit_ns) {
  if (limit_ns < 0 || limit_ns > static_cast<int64_t>(kWaitLimitNs)) return W4A4_ERR_ARG;
  g_wait_limit_ns.store(limit_ns == 0 ? kWaitLimitNs : static_cast<unsigned long long>(limit_ns),
                        std::memory_order_relaxed);
  return W4A4_OK;
}

int w4a4_debug_wait_timeout(int64_t timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return W4A4_ERR_ARG;
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != W4A4_OK) return st;
  wait_forever_bounded_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(timeout_us) * 1000ull, dev->status);
  return cudaGetLastError() == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}

}  // extern "C"
