// s4 x s4 -> s32 GEMM with the rank-one epilogue, on the sm_100a tensor cores.
//
// The page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels" (Description) keeps the per-row and per-column scales out of the K
// loop, so the main loop is a pure integer product with int32 accumulators
// (|acc| <= 49*K) and y = acc * sx[m] * sw[n] (+ bias) is applied once per
// output.  Its kernel is an Ampere/Ada mma.sync s4 design; on sm_100a there is
// no 4-bit integer tcgen05 kind, so this kernel widens the packed nibbles to
// bytes in shared memory and runs tcgen05.mma.kind::i8.
//
// B200 design
//   * CTA pairs (clusters of 2) share one 256 x 256 output tile: CTA r holds
//     rows [128 r, 128 r + 128) of the A tile and of the B tile, and the even
//     CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32), which
//     reads A and B from both CTAs' shared memory and accumulates int32 in
//     both CTAs' tensor memory.  Each SM thus widens and feeds only half of
//     the B tile, which keeps its shared-memory traffic per k-block (32 KB of
//     widened bytes written, 32 KB read by the tensor core) under the time of
//     the MMA itself.
//   * A producer warp per CTA TMA-loads the packed nibbles of its half-tiles
//     (64-byte rows, 128 rows of A and of B per k-block) into a 4-deep ring.
//     Eight "widen" warps read them back with 128-bit shared loads, place
//     every nibble q in the high half of a byte -- the signed byte 16*q, so no
//     sign extension is needed -- and store the bytes in the 128-byte-swizzle
//     K-major layout the MMA reads, into a second 4-deep ring.  Both operands
//     get the same treatment (and the same byte order inside each word), so
//     the MMA accumulates 256 * acc exactly (|256 acc| <= 12544 K < 2^31 for
//     K <= 131072) and the epilogue shifts the factor back out.
//   * One thread of the even CTA issues the MMAs; tcgen05.commit with a
//     cluster multicast frees a ring slot in both CTAs at once.  The
//     accumulator is double-buffered in tensor memory (2 x 256 columns), so
//     four epilogue warps per CTA drain tile i (tcgen05.ld, y = bf16(((float)acc
//     * sx[m]) * sw[n] + bias[n]) with explicitly rounded fp32 steps) while the
//     MMAs of tile i+1 run.
//   * The kernel is persistent: the clusters walk the tiles with a static
//     stride.  Every wait is bounded: an expired wait records W4A4_ERR_TIMEOUT
//     in the device status word, every role stops, the MMAs are drained and
//     the tensor memory is freed before the CTAs exit.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int BM = kGemmBM;     // output rows per cluster tile (256)
constexpr int BN = kGemmBN;     // output columns per cluster tile (256)
constexpr int HM = BM / 2;      // A rows per CTA
constexpr int HN = BN / 2;      // B rows per CTA
constexpr int BK = 128;         // int4 codes per k-block (= bytes per widened row)
constexpr int BKP = BK / 2;     // packed bytes per row per k-block
constexpr int SP = 4;           // packed ring depth
constexpr int SWD = 4;          // widened ring depth
constexpr int kWidenWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kWarpMma = 0;
constexpr int kWarpTma = 1;
constexpr int kWarpWiden0 = 2;
constexpr int kWarpEpi0 = kWarpWiden0 + kWidenWarps;
constexpr int kThreads = (kWarpEpi0 + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * BN;   // two int32 accumulators of BN columns

constexpr uint32_t kWideA = HM * BK;     // 16 KB
constexpr uint32_t kWideB = HN * BK;     // 16 KB
constexpr uint32_t kStage = kWideA + kWideB;
constexpr uint32_t kPackA = HM * BKP;    // 8 KB
constexpr uint32_t kPackB = HN * BKP;    // 8 KB
constexpr uint32_t kPStage = kPackA + kPackB;
constexpr uint32_t kOffPack = SWD * kStage;
constexpr uint32_t kSmemBytes = kOffPack + SP * kPStage;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // slack for 1024-byte alignment

// packed 16-byte units per CTA and k-block: (HM + HN) rows x 4 units
constexpr int kUnits = (HM + HN) * (BKP / 16);
constexpr int kUnitsPerThread = kUnits / (kWidenWarps * 32);   // 4

struct Bars {
  uint64_t packed_full[SP];   // TMA transaction barrier
  uint64_t packed_empty[SP];  // kWidenWarps local arrivals
  // even CTA: its kWidenWarps local arrivals plus one forwarded by the odd
  // CTA; odd CTA: its kWidenWarps local arrivals (consumed by the forwarder)
  uint64_t wide_full[SWD];
  uint64_t wide_empty[SWD];   // both CTAs: one multicast commit per phase
  uint64_t acc_full[2];       // both CTAs: one multicast commit per phase
  uint64_t acc_empty[2];      // even CTA: 2 x kEpiWarps arrivals per phase (local and remote)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Widening without sign extension: a signed nibble q placed in the high half
// of a byte IS the signed byte 16*q.  The nibbles of a 32-bit word go to bytes
// in the order (1,3,5,7, 0,2,4,6); that K permutation is the same for both
// operands, so the dot product is unchanged.  Three integer ops per 8 codes.
__device__ __forceinline__ void widen_word16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  o0 = w & 0xF0F0F0F0u;
  o1 = (w << 4) & 0xF0F0F0F0u;
}

// Widen this thread's packed units of one k-block (read from the packed
// stage; A units first, then B) into the widened stage.
__device__ __forceinline__ void widen_units(const uint8_t* __restrict__ pstage, uint8_t* __restrict__ stage, int wt) {
  uint4 buf[kUnitsPerThread];
#pragma unroll
  for (int i = 0; i < kUnitsPerThread; ++i)
    buf[i] = *reinterpret_cast<const uint4*>(pstage + (wt + i * kWidenWarps * 32) * 16);
#pragma unroll
  for (int i = 0; i < kUnitsPerThread; ++i) {
    const int u = wt + i * kWidenWarps * 32;
    const bool isA = u < HM * 4;
    const int uu = isA ? u : u - HM * 4;
    const int r = uu >> 2;
    const int part = uu & 3;
    uint4 c0, c1;
    widen_word16(buf[i].x, c0.x, c0.y);
    widen_word16(buf[i].y, c0.z, c0.w);
    widen_word16(buf[i].z, c1.x, c1.y);
    widen_word16(buf[i].w, c1.z, c1.w);
    uint8_t* rowp = stage + (isA ? 0 : kWideA) + (r >> 3) * 1024 + (r & 7) * 128;
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
  const uint32_t rank = cluster_rank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
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
      mbar_init(&bars.wide_full[s], rank == 0 ? kWidenWarps + 1 : kWidenWarps);
      mbar_init(&bars.wide_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.acc_full[s], 1);
      mbar_init(&bars.acc_empty[s], 2 * kEpiWarps);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(&bars.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers and tensor memory of both CTAs are ready
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      uint32_t ws = 0, wph = 0, acc_ph = 0;
      int lt = 0;
      bool ok = true;
      for (int t = cluster; t < tiles && ok; t += nclusters, ++lt) {
        const int ab = lt & 1;
        if (!mbar_wait_cluster(&bars.acc_empty[ab], ((acc_ph >> ab) & 1) ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        acc_ph ^= 1u << ab;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&bars.wide_full[ws], wph, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + ws * kStage));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + ws * kStage + kWideA));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_i8_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_pair_mc(&bars.wide_empty[ws], 0x3);
          if (++ws == SWD) { ws = 0; wph ^= 1; }
        }
        if (ok) mma_commit_pair_mc(&bars.acc_full[ab], 0x3);
      }
      // every issued MMA completes before the tensor memory can be released
      mma_commit_pair_mc(&bars.drain, 0x1);
      (void)mbar_wait_cluster(&bars.drain, 0, nullptr, nullptr, 100000000ull);
    } else if (rank == 1 && lane == 0) {
      // Forwarder: a completed ring slot of this (odd) CTA becomes one arrival
      // on the even CTA's barrier.  The widen warps only release locally (a
      // cluster-scope release would wait for their prefetch loads in flight);
      // this thread has no memory traffic of its own, and it forwards in the
      // order the MMA consumes the slots.
      uint32_t ws = 0, wph = 0;
      for (int t = cluster; t < tiles; t += nclusters) {
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars.wide_full[ws], wph, abort_flag, args.status)) { ok = false; break; }
          mbar_arrive_remote(&bars.wide_full[ws], 0);
          if (++ws == SWD) { ws = 0; wph ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t ps = 0, ph = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int t = cluster; t < tiles && ok; t += nclusters) {
        const int mb = t % num_m, nb = t / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars.packed_empty[ps], ph ^ 1, abort_flag, args.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.packed_full[ps], kPStage);
          uint8_t* dst = smem + kOffPack + ps * kPStage;
          tma_load_2d(dst, &tmA, &bars.packed_full[ps], kb * BKP, mb * BM + static_cast<int>(rank) * HM);
          tma_load_2d(dst + kPackA, &tmB, &bars.packed_full[ps], kb * BKP, nb * BN + static_cast<int>(rank) * HN);
          ++issued;
          if (++ps == SP) { ps = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // let every copy this thread issued land before the CTA goes away
        for (int s2 = 0; s2 < SP && s2 < issued; ++s2) {
          const int64_t n_s = issued / SP + (s2 < issued % SP ? 1 : 0);
          (void)mbar_wait(&bars.packed_full[s2], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (warp < kWarpEpi0) {
    // ------------------------------------------------------------ widen warps
    const int wt = threadIdx.x - kWarpWiden0 * 32;
    uint32_t ps = 0, ph = 0, ws = 0, wph = 0;
    bool ok = true;
    for (int t = cluster; t < tiles && ok; t += nclusters) {
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!warp_wait(&bars.packed_full[ps], ph, abort_flag, args.status) ||
            !warp_wait_cluster(&bars.wide_empty[ws], wph ^ 1, abort_flag, args.status)) { ok = false; break; }
        widen_units(smem + kOffPack + ps * kPStage, smem + ws * kStage, wt);
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
    uint32_t acc_ph = 0;
    int lt = 0;
    for (int t = cluster; t < tiles; t += nclusters, ++lt) {
      const int ab = lt & 1;
      const int mb = t % num_m, nb = t / num_m;
      if (!warp_wait_cluster(&bars.acc_full[ab], (acc_ph >> ab) & 1, abort_flag, args.status)) break;
      acc_ph ^= 1u << ab;
      tc_fence_after();
      const int64_t m = static_cast<int64_t>(mb) * BM + rank * HM + q * 32 + lane;
      const bool mrow = m < M;
      float sxm = 0.0f;
      if (!OUT_S32 && mrow) sxm = args.sx[m];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * BN + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = static_cast<uint32_t>(static_cast<int32_t>(r[i]) >> 8);
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
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (n0 + i < N) dst[i] = static_cast<int32_t>(r[i]);
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
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (n0 + i < N) dst[i] = static_cast<uint16_t>((packed[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(&bars.acc_empty[ab], 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs are done with the pair's MMAs and tensor memory
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Largest number of 2-CTA clusters of this kernel that can be resident at
// once (queried once per device; the persistent grid never exceeds it).
template <int OUT_S32>
int max_clusters(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
  if (cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<OUT_S32>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  if (n > num_sms / 2) n = num_sms / 2;
  cached[dev] = n;
  return n;
}

template <int OUT_S32>
cudaError_t launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int64_t tiles, int num_sms,
                   cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<OUT_S32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemAlloc));
  if (e != cudaSuccess) return e;
  const int64_t cmax = max_clusters<OUT_S32>(num_sms);
  const int grid = static_cast<int>(2 * (tiles < cmax ? tiles : cmax));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<OUT_S32>, tmA, tmB, a);
}

}  // namespace

cudaError_t gemm_tc_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int num_sms,
                           cudaStream_t stream) {
  const int64_t tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  if (tiles == 0) return cudaSuccess;
  cudaError_t e =
      a.out_s32 ? launch<1>(tmA, tmB, a, tiles, num_sms, stream) : launch<0>(tmA, tmB, a, tiles, num_sms, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a4
