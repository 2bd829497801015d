// Small-M (M <= 64) W4A4 linear: weight-streaming split-K kernel.
//
// With a handful of activation rows the layer is bound by reading the packed
// weight from HBM (N*K/2 bytes), not by the tensor cores.  The pages' own
// answer for this regime (page "[PR #97] ... grouped W4A8 over the INT8 GEMM",
// section "Chunk sizing": a separate path for M <= 64 that keeps the weight
// stream close to the GEMM) motivates a dedicated kernel; the arithmetic is the
// same s4 x s4 -> s32 product and rank-one epilogue as the large-M kernel.
//
// Design (swap-AB + split-K):
//   * The MMA M side is 128 weight rows, the N side the activation rows padded
//     to NP in {16, 32, 64}; tcgen05.mma.kind::i8 accumulates int32 in TMEM.
//   * Work units are (128-row weight tile, K slice) pairs, sized so that about
//     two CTAs run on every SM; each streams its weight slice through a TMA
//     ring, widens nibbles to bytes in shared memory and issues the MMAs.
//   * K slices are reduced exactly: each CTA stores its int32 partial tile in
//     its own workspace slot, then increments a per-tile arrival counter with
//     a wrapping atomicInc; the CTA that arrives last sums the slots in split
//     order (integer addition, so the result is exact and deterministic),
//     applies the epilogue and writes y.  The wrap leaves every counter at 0,
//     so only the counter block has to be zero before the first call.  With a
//     single K slice the epilogue runs directly from the accumulator.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int WM = 128;        // weight rows per tile (MMA M)
constexpr int BK = 128;        // codes per k-block
constexpr int BKP = BK / 2;    // packed bytes per k-block row
constexpr int SP = 3;          // packed ring depth
constexpr int SWD = 2;         // widened ring depth
constexpr int kWorkWarps = 4;  // widen + epilogue warps
constexpr int kThreads = (2 + kWorkWarps) * 32;

template <int NP>
struct Layout {
  static constexpr uint32_t kWideW = WM * BK;     // 16 KB
  static constexpr uint32_t kWideX = NP * BK;     // <= 8 KB
  static constexpr uint32_t kPackW = WM * BKP;    // 8 KB
  static constexpr uint32_t kPackX = NP * BKP;    // <= 4 KB
  static constexpr uint32_t kOffWideW = 0;
  static constexpr uint32_t kOffWideX = kOffWideW + SWD * kWideW;
  static constexpr uint32_t kOffPackW = kOffWideX + SWD * kWideX;
  static constexpr uint32_t kOffPackX = kOffPackW + SP * kPackW;
  static constexpr uint32_t kBytes = kOffPackX + SP * kPackX;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = NP < 32 ? 32 : NP;
};

struct Bars {
  uint64_t packed_full[SP];
  uint64_t packed_empty[SP];
  uint64_t wide_full[SWD];
  uint64_t wide_empty[SWD];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
  unsigned int last;
};

// Same widening as the large-M kernel: each nibble q lands in the high half of
// a byte (the signed byte 16*q); both operands share the byte order, the MMA
// accumulates 256*acc exactly and the epilogue shifts the factor out.
__device__ __forceinline__ void widen_word16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  o0 = w & 0xF0F0F0F0u;
  o1 = (w << 4) & 0xF0F0F0F0u;
}

template <int kUnits>
__device__ __forceinline__ void widen_tile(const uint8_t* __restrict__ packed, uint8_t* __restrict__ wide, int wt) {
  constexpr int kPer = (kUnits + kWorkWarps * 32 - 1) / (kWorkWarps * 32);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int u = wt + i * kWorkWarps * 32;
    if (kUnits % (kWorkWarps * 32) != 0 && u >= kUnits) break;
    const int r = u >> 2;
    const int part = u & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(packed + u * 16);
    uint4 c0, c1;
    widen_word16(w.x, c0.x, c0.y);
    widen_word16(w.y, c0.z, c0.w);
    widen_word16(w.z, c1.x, c1.y);
    widen_word16(w.w, c1.z, c1.w);
    uint8_t* rowp = wide + (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    *reinterpret_cast<uint4*>(rowp + (((2 * part) ^ sw) << 4)) = c0;
    *reinterpret_cast<uint4*>(rowp + (((2 * part + 1) ^ sw) << 4)) = c1;
  }
}

template <int NP>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NP]);
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_32x32b_x32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, uint32_t (&r)[64]) {
  uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
  uint32_t (&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
  tmem_ld_32x32b_x32(taddr, a);
  tmem_ld_32x32b_x32(taddr + 32, b);
}

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

template <int NP, int OUT_S32>
__global__ void __launch_bounds__(kThreads, 1)
    smallm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, SmallMArgs args,
                  int kb_per_split, int splits) {
  using Lay = Layout<NP>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = args.M, N = args.N;
  const int num_kb = static_cast<int>((args.K + BK - 1) / BK);
  const int ntile = blockIdx.x / splits;
  const int split = blockIdx.x - ntile * splits;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(num_kb, kb0 + kb_per_split);
  const int nkb = kb1 - kb0;   // >= 1 by construction

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP; ++s) {
      mbar_init(&bars.packed_full[s], 1);
      mbar_init(&bars.packed_empty[s], kWorkWarps);
    }
    for (int s = 0; s < SWD; ++s) {
      mbar_init(&bars.wide_full[s], kWorkWarps);
      mbar_init(&bars.wide_empty[s], 1);
    }
    mbar_init(&bars.acc_full, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t ps = 0, ph = 0;
      int issued = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&bars.packed_empty[ps], ph ^ 1, abort_flag, args.status)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars.packed_full[ps], Lay::kPackW + Lay::kPackX);
        tma_load_2d(smem + Lay::kOffPackW + ps * Lay::kPackW, &tmW, &bars.packed_full[ps], kb * BKP, ntile * WM);
        tma_load_2d(smem + Lay::kOffPackX + ps * Lay::kPackX, &tmX, &bars.packed_full[ps], kb * BKP, 0);
        ++issued;
        if (++ps == SP) { ps = 0; ph ^= 1; }
      }
      if (!ok) {
        for (int s = 0; s < SP && s < issued; ++s) {
          const int n_s = issued / SP + (s < issued % SP ? 1 : 0);
          (void)mbar_wait(&bars.packed_full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(WM, NP);
      uint32_t ws = 0, wph = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&bars.wide_full[ws], wph, abort_flag, args.status)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + Lay::kOffWideW + ws * Lay::kWideW));
        const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + Lay::kOffWideX + ws * Lay::kWideX));
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          mma_i8(tmem_base, ad + 2 * kk, bd + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        mma_commit(&bars.wide_empty[ws]);
        if (++ws == SWD) { ws = 0; wph ^= 1; }
      }
      (void)ok;
      mma_commit(&bars.acc_full);   // also the drain point on an abort
    }
  } else {
    const int wt = threadIdx.x - 64;
    uint32_t ps = 0, ph = 0, ws = 0, wph = 0;
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      if (!warp_wait(&bars.packed_full[ps], ph, abort_flag, args.status) ||
          !warp_wait(&bars.wide_empty[ws], wph ^ 1, abort_flag, args.status)) { ok = false; break; }
      widen_tile<WM * BKP / 16>(smem + Lay::kOffPackW + ps * Lay::kPackW, smem + Lay::kOffWideW + ws * Lay::kWideW, wt);
      widen_tile<NP * BKP / 16>(smem + Lay::kOffPackX + ps * Lay::kPackX, smem + Lay::kOffWideX + ws * Lay::kWideX, wt);
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.wide_full[ws]);
        mbar_arrive(&bars.packed_empty[ps]);
      }
      if (++ps == SP) { ps = 0; ph ^= 1; }
      if (++ws == SWD) { ws = 0; wph ^= 1; }
    }
    // ------------------------------------------------------------- epilogue
    if (ok) (void)warp_wait(&bars.acc_full, 0, abort_flag, args.status);
    // the four work warps agree before any of them takes the named barriers below
    asm volatile("bar.sync 1, %0;" ::"r"(kWorkWarps * 32) : "memory");
    const bool all_ok = *abort_flag == 0;
    __syncwarp();
    const int q = warp & 3;
    const int64_t n = static_cast<int64_t>(ntile) * WM + q * 32 + lane;   // weight row = output column
    const bool ncol = n < N;
    uint32_t acc[NP];
    if (all_ok) {
      tc_fence_after();
      tmem_ld_cols<NP>(tmem_base + (static_cast<uint32_t>(q * 32) << 16), acc);
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < NP; ++m) acc[m] = static_cast<uint32_t>(static_cast<int32_t>(acc[m]) >> 8);
    }
    const int mrows = static_cast<int>(M);
    bool do_epi = all_ok && splits == 1;
    if (all_ok && splits > 1) {
      // this split's partial tile goes to its own slot: no zeroed memory needed
      if (ncol) {
        int32_t* slot = args.partial + static_cast<int64_t>(split) * M * N;
#pragma unroll
        for (int m = 0; m < NP; ++m)
          if (m < mrows) __stcg(slot + static_cast<int64_t>(m) * N + n, static_cast<int>(acc[m]));
      }
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"r"(kWorkWarps * 32) : "memory");
      if (wt == 0) {
        // wraps back to 0 on the last arrival, leaving the counter ready for the next call
        const unsigned int old = atomicInc(args.counters + ntile, static_cast<unsigned int>(splits - 1));
        bars.last = (old == static_cast<unsigned int>(splits - 1)) ? 1u : 0u;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kWorkWarps * 32) : "memory");
      if (bars.last) {
        __threadfence();
        if (ncol) {
          // sum the slots in split order (integer addition: exact)
#pragma unroll
          for (int m = 0; m < NP; ++m) {
            if (m < mrows) {
              int sum = 0;
              for (int sp = 0; sp < splits; ++sp)
                sum += __ldcg(args.partial + (static_cast<int64_t>(sp) * M + m) * N + n);
              acc[m] = static_cast<uint32_t>(sum);
            }
          }
        }
        do_epi = true;
      }
    }
    if (do_epi && ncol) {
      if (OUT_S32) {
        int32_t* out = reinterpret_cast<int32_t*>(args.out);
#pragma unroll
        for (int m = 0; m < NP; ++m)
          if (m < mrows) out[static_cast<int64_t>(m) * args.ldo + n] = static_cast<int32_t>(acc[m]);
      } else {
        uint16_t* out = reinterpret_cast<uint16_t*>(args.out);
        const float swn = args.sw[n];
        const float bn = args.bias != nullptr ? bf16_to_f(args.bias[n]) : 0.0f;
#pragma unroll
        for (int m = 0; m < NP; ++m) {
          if (m < mrows) {
            float y = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(acc[m])), args.sx[m]), swn);
            if (args.bias != nullptr) y = __fadd_rn(y, bn);
            out[static_cast<int64_t>(m) * args.ldo + n] = f_to_bf16(y);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // the MMA thread's final commit arrives when every MMA has completed
    if (lane == 0) (void)mbar_wait(&bars.acc_full, 0, nullptr, nullptr, 100000000ull);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

template <int NP>
cudaError_t launch_np(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a, int kb_per, int splits,
                      int ntiles, cudaStream_t stream) {
  using Lay = Layout<NP>;
  const int grid = ntiles * splits;
  cudaError_t e;
  if (a.out_s32) {
    e = cudaFuncSetAttribute(smallm_kernel<NP, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    smallm_kernel<NP, 1><<<grid, kThreads, Lay::kAlloc, stream>>>(tmW, tmX, a, kb_per, splits);
  } else {
    e = cudaFuncSetAttribute(smallm_kernel<NP, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess) return e;
    smallm_kernel<NP, 0><<<grid, kThreads, Lay::kAlloc, stream>>>(tmW, tmX, a, kb_per, splits);
  }
  return cudaGetLastError();
}

}  // namespace

// Split plan shared by the launcher and the workspace query.  It is sized for
// the 148 SMs of a B200 (about two CTAs per SM) rather than the device's own
// count, so that the workspace size stays a pure function of the shape.
constexpr int kPlanSms = 148;
static void smallm_plan(int64_t N, int64_t K, int num_sms, int* ntiles, int* kb_per, int* splits) {
  const int nt = static_cast<int>((N + WM - 1) / WM);
  const int num_kb = static_cast<int>((K + BK - 1) / BK);
  int s = static_cast<int>((2.0 * num_sms) / nt + 0.5);
  if (s < 1) s = 1;
  if (s > num_kb) s = num_kb;
  const int per = (num_kb + s - 1) / s;
  *ntiles = nt;
  *kb_per = per;
  *splits = (num_kb + per - 1) / per;
}

size_t smallm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  int nt, per, splits;
  smallm_plan(N, K, kPlanSms, &nt, &per, &splits);
  size_t part = splits > 1 ? static_cast<size_t>(splits) * M * N * 4 : 0;
  return kSmallMCounterBytes + (part + 255) / 256 * 256;
}

cudaError_t smallm_launch_tm(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a, int num_sms,
                             cudaStream_t stream) {
  (void)num_sms;
  int nt, per, splits;
  smallm_plan(a.N, a.K, kPlanSms, &nt, &per, &splits);
  if (a.M <= 16) return launch_np<16>(tmW, tmX, a, per, splits, nt, stream);
  if (a.M <= 32) return launch_np<32>(tmW, tmX, a, per, splits, nt, stream);
  return launch_np<64>(tmW, tmX, a, per, splits, nt, stream);
}

int smallm_rows_padded(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

}  // namespace w4a4

// ---------------------------------------------------------------------------
// Small-M linear that allocates nothing (w4a4_linear_noalloc in w4a4.h).
//
// Same kernel and launch as the workspace-taking path; only the scratch is
// different: the arrival counters and split-K slots live in a fixed array of
// this library's own device memory instead of a caller workspace.
// ---------------------------------------------------------------------------
#include <mutex>

#include "w4a4.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB: counter block + split-K slots
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};   // device address of the array, per device
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device.  The host-side
// name g_noalloc_scratch is only a stand-in for the symbol, never a device
// pointer, so its address is resolved once per device with
// cudaGetSymbolAddress (with that device current) and cached; the same first
// call clears the counter block on `stream` (the counters must start at zero;
// every completed call leaves them at zero again).
int noalloc_scratch(uint8_t** out, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A4_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return W4A4_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W4A4_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, w4a4::kSmallMCounterBytes, stream) != cudaSuccess) return W4A4_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_noalloc_ptr[dev]);
  return W4A4_OK;
}

}  // namespace

extern "C" int w4a4_linear_noalloc(const int8_t* Xq, const float* sx, const int8_t* Wq, const float* sw,
                                   const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t ldy,
                                   void* stream) {
  using namespace w4a4;
  int st = validate_linear(Xq, sx, Wq, sw, bias, y, M, N, K, ldy, 0);
  if (st != W4A4_OK) return st;
  if (M < 1 || M > kSmallMMax || N > kSmallMMaxN) return W4A4_ERR_SHAPE;
  if (smallm_workspace_bytes(M, N, K) > kNoAllocScratchBytes) return W4A4_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != W4A4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch, s)) != W4A4_OK) return st;
  CUtensorMap tmW, tmX;
  if ((st = packed_map(&tmW, Wq, N, K, WM)) != W4A4_OK) return st;
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
  a.out = y;
  a.ldo = ldy;
  a.out_s32 = 0;
  a.counters = reinterpret_cast<unsigned int*>(scratch);
  a.partial = reinterpret_cast<int32_t*>(scratch + kSmallMCounterBytes);
  a.status = dev->status;
  return smallm_launch_tm(tmW, tmX, a, dev->num_sms, s) == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA;
}
