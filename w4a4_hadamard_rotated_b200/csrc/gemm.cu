// s4 x s4 -> s32 GEMM with the rank-one epilogue, on the sm_100a tensor cores.
//
// The page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels" (Description) keeps the per-row and per-column scales out of the K
// loop, so the main loop is a pure integer product with int32 accumulators
// (|acc| <= 49*K) and y = acc * sx[m] * sw[n] (+ bias) is applied once per
// output.  Its kernel is an Ampere/Ada mma.sync s4 design; on sm_100a there is
// no 4-bit integer tcgen05 kind, so this kernel:
//   1. TMA-loads packed nibble tiles of both operands (no swizzle, 64 bytes =
//      128 codes per row per k-block) into a 4-deep shared-memory ring,
//   2. widens them in shared memory to signed bytes written directly in the
//      128-byte-swizzle K-major layout the MMA reads (4 "widen" warps,
//      128-bit loads/stores, a LOP3/IADD/PRMT nibble-to-byte sign extension),
//   3. issues tcgen05.mma.kind::i8 (M=128, N=256, K=32 per instruction) from one
//      thread into a double-buffered int32 accumulator in tensor memory,
//   4. drains the accumulator with tcgen05.ld in 4 epilogue warps, applying
//      y = bf16(((float)acc * sx[m]) * sw[n] + bias[n]) with explicitly
//      rounded fp32 steps (no contraction), while the MMA warp already works on
//      the next tile.
// The kernel is persistent (one CTA per SM, static round-robin tiles).  Every
// wait is bounded: an expired wait records W4A4_ERR_TIMEOUT in the device
// status word, all roles stop, in-flight copies and MMAs are drained and the
// tensor memory is freed before the CTA exits.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int BM = kGemmBM;     // rows of A (activations) per tile
constexpr int BN = kGemmBN;     // rows of B (weights) per tile
constexpr int BK = 128;         // int4 codes per k-block (= bytes per widened row)
constexpr int BKP = BK / 2;     // packed bytes per row per k-block
constexpr int SP = 4;           // packed ring depth
constexpr int SWD = 2;          // widened ring depth
constexpr int kWidenWarps = 4;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (2 + kWidenWarps + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * BN;   // two int32 accumulators of BN columns

constexpr uint32_t kWideA = BM * BK;     // 16 KB
constexpr uint32_t kWideB = BN * BK;     // 32 KB
constexpr uint32_t kPackA = BM * BKP;    // 8 KB
constexpr uint32_t kPackB = BN * BKP;    // 16 KB
constexpr uint32_t kOffWideA = 0;
constexpr uint32_t kOffWideB = kOffWideA + SWD * kWideA;
constexpr uint32_t kOffPackA = kOffWideB + SWD * kWideB;
constexpr uint32_t kOffPackB = kOffPackA + SP * kPackA;
constexpr uint32_t kSmemBytes = kOffPackB + SP * kPackB;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // slack for 1024-byte alignment

struct Bars {
  uint64_t packed_full[SP];
  uint64_t packed_empty[SP];
  uint64_t wide_full[SWD];
  uint64_t wide_empty[SWD];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Two signed-nibble words -> sign-extended bytes, element order preserved.
__device__ __forceinline__ void widen_word(uint32_t w, uint32_t& o0, uint32_t& o1) {
  uint32_t lo = w & 0x0F0F0F0Fu;          // nibbles 0,2,4,6
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // nibbles 1,3,5,7
  // per byte: u in [0,15] -> u for u < 8, u - 16 otherwise (no inter-byte carry)
  lo = (lo + 0x78787878u) ^ 0x78787878u;
  hi = (hi + 0x78787878u) ^ 0x78787878u;
  o0 = __byte_perm(lo, hi, 0x5140);
  o1 = __byte_perm(lo, hi, 0x7362);
}

// Widen `units` 16-byte packed units (32 codes each) of a [rows x 64 B] packed
// tile into the [rows x 128 B] 128B-swizzled K-major tile.
template <int kUnits>
__device__ __forceinline__ void widen_tile(const uint8_t* __restrict__ packed, uint8_t* __restrict__ wide, int wt) {
#pragma unroll
  for (int i = 0; i < kUnits / (kWidenWarps * 32); ++i) {
    const int u = wt + i * kWidenWarps * 32;
    const int r = u >> 2;
    const int part = u & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(packed + u * 16);
    uint4 c0, c1;
    widen_word(w.x, c0.x, c0.y);
    widen_word(w.y, c0.z, c0.w);
    widen_word(w.z, c1.x, c1.y);
    widen_word(w.w, c1.z, c1.w);
    uint8_t* rowp = wide + (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    *reinterpret_cast<uint4*>(rowp + (((2 * part) ^ sw) << 4)) = c0;
    *reinterpret_cast<uint4*>(rowp + (((2 * part + 1) ^ sw) << 4)) = c1;
  }
}

template <int OUT_S32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs args) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Bars bars;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = args.M, N = args.N;
  const int num_m = static_cast<int>((M + BM - 1) / BM);
  const int num_n = static_cast<int>((N + BN - 1) / BN);
  const int tiles = num_m * num_n;
  const int num_kb = static_cast<int>((args.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP; ++s) {
      mbar_init(&bars.packed_full[s], 1);
      mbar_init(&bars.packed_empty[s], kWidenWarps);
    }
    for (int s = 0; s < SWD; ++s) {
      mbar_init(&bars.wide_full[s], kWidenWarps);
      mbar_init(&bars.wide_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.acc_full[s], 1);
      mbar_init(&bars.acc_empty[s], kEpiWarps);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int64_t issued = 0;
      uint32_t ps = 0, ph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mb = t % num_m, nb = t / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars.packed_empty[ps], ph ^ 1, abort_flag, args.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.packed_full[ps], kPackA + kPackB);
          tma_load_2d(smem + kOffPackA + ps * kPackA, &tmA, &bars.packed_full[ps], kb * BKP, mb * BM);
          tma_load_2d(smem + kOffPackB + ps * kPackB, &tmB, &bars.packed_full[ps], kb * BKP, nb * BN);
          ++issued;
          if (++ps == SP) { ps = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // let every copy this thread issued land before the CTA goes away
        for (int s = 0; s < SP && s < issued; ++s) {
          const int64_t n_s = issued / SP + (s < issued % SP ? 1 : 0);
          (void)mbar_wait(&bars.packed_full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      uint32_t ws = 0, wph = 0;
      uint32_t acc_ph[2] = {0, 0};
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        if (!mbar_wait(&bars.acc_empty[ab], acc_ph[ab] ^ 1, abort_flag, args.status)) { ok = false; break; }
        acc_ph[ab] ^= 1;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars.wide_full[ws], wph, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + kOffWideA + ws * kWideA));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + kOffWideB + ws * kWideB));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_i8(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(&bars.wide_empty[ws]);
          if (++ws == SWD) { ws = 0; wph ^= 1; }
        }
        if (ok) mma_commit(&bars.acc_full[ab]);
      }
      // all issued MMAs complete before the tensor memory can be released
      mma_commit(&bars.drain);
      (void)mbar_wait(&bars.drain, 0, nullptr, nullptr, 100000000ull);
    }
  } else if (warp < 2 + kWidenWarps) {
    // ------------------------------------------------------------ widen warps
    const int wt = threadIdx.x - 64;
    uint32_t ps = 0, ph = 0, ws = 0, wph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb) {
        // every lane waits (bounded); the warp then agrees, so that no lane
        // leaves the loop while the others sit in __syncwarp
        bool got = mbar_wait(&bars.packed_full[ps], ph, abort_flag, args.status);
        got = got && mbar_wait(&bars.wide_empty[ws], wph ^ 1, abort_flag, args.status);
        if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
        widen_tile<BM * BKP / 16>(smem + kOffPackA + ps * kPackA, smem + kOffWideA + ws * kWideA, wt);
        widen_tile<BN * BKP / 16>(smem + kOffPackB + ps * kPackB, smem + kOffWideB + ws * kWideB, wt);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.wide_full[ws]);
          mbar_arrive(&bars.packed_empty[ps]);
        }
        if (++ps == SP) { ps = 0; ph ^= 1; }
        if (++ws == SWD) { ws = 0; wph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    uint32_t acc_ph[2] = {0, 0};
    int lt = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
      const int ab = lt & 1;
      const int mb = t % num_m, nb = t / num_m;
      const bool got = mbar_wait(&bars.acc_full[ab], acc_ph[ab], abort_flag, args.status);
      __syncwarp();
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      acc_ph[ab] ^= 1;
      tc_fence_after();
      const int64_t m = static_cast<int64_t>(mb) * BM + q * 32 + lane;
      const bool mrow = m < M;
      float sxm = 0.0f;
      if (!OUT_S32 && mrow) sxm = args.sx[m];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * BN + c * 32, r);
        tmem_wait_ld();
        const int64_t n0 = static_cast<int64_t>(nb) * BN + c * 32;
        if (!mrow || n0 >= N) continue;   // the loads above stay warp-uniform
        const bool full = n0 + 32 <= N;
        if (OUT_S32) {
          int32_t* dst = reinterpret_cast<int32_t*>(args.out) + m * args.ldo + n0;
          if (full) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              reinterpret_cast<uint4*>(dst)[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
          } else {
            for (int i = 0; i < 32 && n0 + i < N; ++i) dst[i] = static_cast<int32_t>(r[i]);
          }
        } else {
          uint16_t* dst = reinterpret_cast<uint16_t*>(args.out) + m * args.ldo + n0;
          float swv[32], bv[32];
          if (full) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 s4 = __ldg(reinterpret_cast<const float4*>(args.sw + n0) + i);
              swv[4 * i] = s4.x; swv[4 * i + 1] = s4.y; swv[4 * i + 2] = s4.z; swv[4 * i + 3] = s4.w;
            }
            if (args.bias != nullptr) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint4 b4 = __ldg(reinterpret_cast<const uint4*>(args.bias + n0) + i);
                const uint32_t bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  bv[8 * i + 2 * j] = __uint_as_float(bw[j] << 16);
                  bv[8 * i + 2 * j + 1] = __uint_as_float(bw[j] & 0xFFFF0000u);
                }
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const bool in = n0 + i < N;
              swv[i] = in ? args.sw[n0 + i] : 0.0f;
              bv[i] = (in && args.bias != nullptr) ? __uint_as_float(static_cast<uint32_t>(args.bias[n0 + i]) << 16) : 0.0f;
            }
          }
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float y0 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[2 * i])), sxm), swv[2 * i]);
            float y1 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[2 * i + 1])), sxm), swv[2 * i + 1]);
            if (args.bias != nullptr) {
              y0 = __fadd_rn(y0, bv[2 * i]);
              y1 = __fadd_rn(y1, bv[2 * i + 1]);
            }
            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
            packed[i] = *reinterpret_cast<const uint32_t*>(&h);
          }
          if (full) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4*>(dst)[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          } else {
            for (int i = 0; i < 32 && n0 + i < N; ++i)
              dst[i] = static_cast<uint16_t>((packed[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t gemm_tc_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int num_sms,
                           cudaStream_t stream) {
  const int64_t tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  if (tiles == 0) return cudaSuccess;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  cudaError_t e;
  if (a.out_s32) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<1><<<grid, kThreads, kSmemAlloc, stream>>>(tmA, tmB, a);
  } else {
    e = cudaFuncSetAttribute(gemm_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<0><<<grid, kThreads, kSmemAlloc, stream>>>(tmA, tmB, a);
  }
  return cudaGetLastError();
}

}  // namespace w4a4
