// The fused W4A4 layer for callers that cannot allocate device memory
// (w4a4_linear_fused_noalloc in w4a4.h).
//
// The fused layer needs scratch memory between its two kernels: the packed
// int4 activation and its per-row scales, which the activation kernel writes
// and the GEMM kernel reads.  w4a4_linear_fused takes that scratch from the
// caller as a workspace.  Some callers have no way to provide one -- a plug-in
// inside a host framework that owns every byte of device memory and hands a
// custom op only its inputs and outputs, or a serving loop that must not call
// cudaMalloc once it runs (an allocation can synchronise the device and
// fragment a pool that was sized in advance).  This entry point keeps the
// scratch in a fixed array of the library itself instead.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

// 8 MiB: [packed x][sx] of up to M * K / 2 + 4 * M bytes (each part rounded
// up to 256 bytes) -- the 4608-row square layer (K = 3072) needs 7.1 MB.
// Every GPU on which the library is loaded holds this array until the
// process exits.
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev] = {};
std::mutex g_scratch_mu;

// The device address of the scratch array on the current device.  In host
// code the array's name is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A4_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return W4A4_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W4A4_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return W4A4_OK;
}

}  // namespace
}  // namespace w4a4

extern "C" int w4a4_linear_fused_noalloc(const uint16_t* x, int64_t ldx, const int8_t* Wq, const float* sw,
                                         const uint16_t* bias, uint16_t* y, int64_t ldy, int64_t M, int64_t N,
                                         int64_t K, int g, int act, void* stream) {
  using namespace w4a4;
  // the checks of w4a4_linear_fused, before any CUDA call
  int st = validate_fused(x, ldx, Wq, sw, bias, y, ldy, M, N, K, g, act);
  if (st != W4A4_OK) return st;
  // the scratch holds what the caller's workspace would: [packed x][sx]
  if (w4a4_fused_workspace_bytes(M, N, K) > kScratchBytes) return W4A4_ERR_SHAPE;
  // the device must be an sm_100 GPU before the scratch address is looked up
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  if (M == 0) return W4A4_OK;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != W4A4_OK) return st;
  // The activation kernel writes every byte of the packed activation and
  // every scale before the GEMM reads them, so the scratch needs no clearing.
  return w4a4_linear_fused(x, ldx, Wq, sw, bias, y, ldy, M, N, K, g, act, scratch, kScratchBytes, stream);
}
