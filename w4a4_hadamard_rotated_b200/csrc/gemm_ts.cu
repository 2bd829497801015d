// W4A4 GEMM + rank-one epilogue on the sm_100a tensor cores, with the packed
// weights widened into tensor memory and the activation codes read straight
// from shared memory.
//
// Arithmetic (page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with
// fused CUDA kernels", Description): acc[m, n] = sum_k qx[m, k] * qw[n, k] in
// int32, then y = bf16(acc * sx[m] * sw[n] + bias[n]) with the scales kept out
// of the K loop.  tcgen05 has no 4-bit integer kind, so the int4 codes are fed
// to tcgen05.mma.kind::i8 as bytes.
//
// B200 design
//   * The activation operand arrives as one int8 code per byte (written by the
//     rotate + quantise kernel for the fused layer, or unpacked once from the
//     packed layout), so the TMA places it directly in the 128-byte-swizzle
//     K-major layout the MMA reads: no shared-memory pass over it.
//   * The weights stay packed in HBM ([N, K/2], two codes per byte).  Each CTA
//     TMA-loads the packed rows of its half tile into a shared-memory ring
//     (64-byte swizzle), and eight widen warps turn every row into 128 bytes
//     -- each nibble q becomes the byte 16*q, in natural K order -- and write
//     them to TENSOR memory with tcgen05.st.  The MMA takes its A operand from
//     there (tcgen05.mma ... [d], [a_tmem], b_desc): the widened weights never
//     touch shared memory, which halves the shared-memory traffic per k-block
//     against widening both operands into shared memory.
//   * Swap-AB on CTA pairs: the MMA M side is 256 weight rows (128 per CTA,
//     A from each CTA's tensor memory), the N side 192 activation rows (96 per
//     CTA, B from each CTA's shared memory); tcgen05.mma.cta_group::2 is issued
//     by one thread of the even CTA.  Both CTAs' activation loads signal the
//     even CTA's barrier, which expects the bytes of both.  The accumulator
//     holds 16*acc exactly (|16 acc| <= 784 K < 2^31 for K <= 2^21).
//   * Tensor memory (512 columns per CTA): two 192-column int32 accumulators
//     (the epilogue of tile i overlaps the MMAs of tile i+1) and four 32-column
//     stages of widened weights.
//   * Epilogue: four warps per CTA, one per tensor-memory lane quarter; lane l
//     owns weight row n (an output column), so sw[n] and bias[n] are scalars
//     per thread and the tile's 192 activation scales are staged in shared
//     memory.  y = ((float)acc * sx[m]) * sw[n] (+ bias[n]), each step rounded
//     in fp32, then bf16; each 32 x 32 block is staged in shared memory and
//     written with one TMA store, which clips the M and N tails.
//   * Persistent: the clusters walk the tiles with a static stride, activation
//     tiles fastest.  Every wait is bounded (W4A4_ERR_TIMEOUT in the device
//     status word; all roles stop, MMAs drain, tensor memory is freed).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int TM = kTsTileW;    // weight rows per cluster tile (MMA M) = 256
constexpr int TN = kTsTileA;    // activation rows per cluster tile (MMA N) = 192
constexpr int HW = TM / 2;      // weight rows per CTA
constexpr int HA = TN / 2;      // activation rows per CTA
constexpr int BK = 128;         // codes per k-block
constexpr int SA = 6;           // activation ring depth
constexpr int SW = 6;           // packed-weight ring depth
constexpr int ST = 4;           // widened-weight stages in tensor memory
constexpr uint32_t kActStage = HA * BK;          // 12 KB
constexpr uint32_t kWStage = HW * (BK / 2);      // 8 KB
constexpr uint32_t kOffAct = 0;
constexpr uint32_t kOffW = kOffAct + SA * kActStage;
constexpr uint32_t kBox = 32 * 64;               // one 32 x 32 bf16 output block
constexpr uint32_t kOffEpi = kOffW + SW * kWStage;
constexpr uint32_t kSmemBytes = kOffEpi + 4 * 2 * kBox;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // slack for 1024-byte alignment
constexpr uint32_t kTmemA = 2 * TN;                  // first widened-weight column
constexpr uint32_t kTmemCols = 512;
static_assert(kTmemA + ST * 32 <= kTmemCols, "tensor memory budget");

// Warp roles (a warp runs on SM sub-partition warp % 4 and may only touch the
// tensor-memory lane quarter warp % 4).
constexpr int kWarpMma = 0;       // even CTA: MMA issuer
constexpr int kWarpTma = 1;       // TMA producer
constexpr int kEpiWarp0 = 2;      // warps 2..5: epilogue, one per quarter
constexpr int kWidenWarp0 = 6;    // warps 6..13: widen, two per quarter (k-block parity)
constexpr int kThreads = 14 * 32;

struct Bars {
  uint64_t act_full[SA];    // even CTA: one expect_tx arrival + the bytes of both CTAs
  uint64_t act_empty[SA];   // both CTAs: one multicast commit per phase
  uint64_t w_full[SW];      // local TMA transaction barrier
  uint64_t w_empty[SW];     // local: one arrival per quarter
  uint64_t a_full[ST];      // even CTA: 4 local + 4 remote widen-warp arrivals
  uint64_t a_empty[ST];     // both CTAs: one multicast commit per phase
  uint64_t acc_full[2];     // both CTAs: one multicast commit per phase
  uint64_t acc_empty[2];    // even CTA: 4 epilogue warps x 2 CTAs
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Packed fp32 pairs (sm_100 .f32x2 arithmetic) for the epilogue.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// One packed word (codes 8w .. 8w+7, code 8w+2b in the low nibble of byte b)
// to two words of bytes 16*q in natural order.  A signed nibble placed in the
// high half of a byte IS the signed byte 16*q, so no sign extension is needed.
__device__ __forceinline__ void widen_word_natural(uint32_t w, uint32_t& c0, uint32_t& c1) {
  const uint32_t hi = w & 0xF0F0F0F0u;           // 16*q of codes 1, 3, 5, 7
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;    // 16*q of codes 0, 2, 4, 6
  c0 = __byte_perm(lo, hi, 0x5140);              // codes 0, 1, 2, 3
  c1 = __byte_perm(lo, hi, 0x7362);              // codes 4, 5, 6, 7
}

// Ring position: slot index and phase parity, advanced once per k-block.
template <int S>
struct Ring {
  uint32_t slot = 0, phase = 0;
  __device__ __forceinline__ void next() {
    if (++slot == S) { slot = 0; phase ^= 1u; }
  }
};

template <int OUT_S32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ts_kernel(const __grid_constant__ CUtensorMap tmAct, const __grid_constant__ CUtensorMap tmW,
                   const __grid_constant__ CUtensorMap tmY, GemmArgs args) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Bars bars;
  __shared__ __align__(16) float epi_sx[2][TN];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int64_t M = args.M, N = args.N;
  const int num_m = static_cast<int>((M + TN - 1) / TN);   // activation tiles
  const int num_n = static_cast<int>((N + TM - 1) / TM);   // weight tiles
  const int tiles = num_m * num_n;
  const int num_kb = static_cast<int>((args.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&bars.act_full[s], 1);
      mbar_init(&bars.act_empty[s], 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(&bars.w_full[s], 1);
      mbar_init(&bars.w_empty[s], 4);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bars.a_full[s], 8);
      mbar_init(&bars.a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.acc_full[s], 1);
      mbar_init(&bars.acc_empty[s], 8);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmAct);
    tma_prefetch_desc(&tmW);
    if (!OUT_S32) tma_prefetch_desc(&tmY);
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
      constexpr uint32_t idesc = idesc_i8(TM, TN);
      Ring<SA> ra;
      Ring<ST> rt;
      uint32_t acc_ph = 0;
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
        const uint32_t d_tmem = tmem_base + ab * TN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&bars.act_full[ra.slot], ra.phase, abort_flag, args.status) ||
              !mbar_wait_cluster(&bars.a_full[rt.slot], rt.phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + kOffAct + ra.slot * kActStage));
          const uint32_t a_tmem = tmem_base + kTmemA + rt.slot * 32;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_i8_pair_ts(d_tmem, a_tmem + kk * 8, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_pair_mc(&bars.act_empty[ra.slot], 0x3);
          mma_commit_pair_mc(&bars.a_empty[rt.slot], 0x3);
          ra.next();
          rt.next();
        }
        if (ok) mma_commit_pair_mc(&bars.acc_full[ab], 0x3);
      }
      // every issued MMA completes before the tensor memory can be released
      mma_commit_pair_mc(&bars.drain, 0x1);
      (void)mbar_wait_cluster(&bars.drain, 0, nullptr, nullptr, 100000000ull);
    }
  } else if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      Ring<SA> ra;
      Ring<SW> rw;
      const uint32_t act_bar0 = mapa_shared(&bars.act_full[0], 0);   // the even CTA's barriers
      bool ok = true;
      for (int t = cluster; t < tiles && ok; t += nclusters) {
        const int mb = t % num_m, nb = t / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&bars.act_empty[ra.slot], ra.phase ^ 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&bars.act_full[ra.slot], 2 * kActStage);
          tma_load_2d_pair(smem + kOffAct + ra.slot * kActStage, &tmAct, act_bar0 + ra.slot * 8u, kb * BK,
                           mb * TN + static_cast<int>(rank) * HA);
          if (!mbar_wait(&bars.w_empty[rw.slot], rw.phase ^ 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.w_full[rw.slot], kWStage);
          tma_load_2d(smem + kOffW + rw.slot * kWStage, &tmW, &bars.w_full[rw.slot], kb * (BK / 2),
                      nb * TM + static_cast<int>(rank) * HW);
          ra.next();
          rw.next();
        }
      }
      if (*abort_flag) {
        // Some copies may still be in flight and their barriers may never
        // complete (the peer stopped too); a copy from L2/HBM lands within
        // microseconds, so a 1 ms pause lets them all land before the CTA's
        // shared memory is released.
        const unsigned long long t0 = global_ns();
        while (global_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp >= kWidenWarp0) {
    // ------------------------------------------------------------ widen warps
    const int q = warp & 3;
    const uint32_t par = static_cast<uint32_t>(warp - kWidenWarp0) >> 2;
    const int r = q * 32 + lane;          // weight row of this CTA's half tile = tensor-memory lane
    const int swz = (r >> 1) & 3;         // 64-byte swizzle of the packed row
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kTmemA;
    Ring<SW> rw;
    Ring<ST> rt;
    uint32_t g = 0;
    bool ok = true;
    for (int t = cluster; t < tiles && ok; t += nclusters) {
      for (int kb = 0; kb < num_kb; ++kb, ++g, rw.next(), rt.next()) {
        if ((g & 1u) != par) continue;
        if (!warp_wait(&bars.w_full[rw.slot], rw.phase, abort_flag, args.status) ||
            !warp_wait_cluster(&bars.a_empty[rt.slot], rt.phase ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        const uint8_t* src = smem + kOffW + rw.slot * kWStage + r * 64;
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 u = *reinterpret_cast<const uint4*>(src + ((j ^ swz) << 4));
          widen_word_natural(u.x, v[8 * j + 0], v[8 * j + 1]);
          widen_word_natural(u.y, v[8 * j + 2], v[8 * j + 3]);
          widen_word_natural(u.z, v[8 * j + 4], v[8 * j + 5]);
          widen_word_natural(u.w, v[8 * j + 6], v[8 * j + 7]);
        }
        tmem_st_32x32b_x32(t_lane + rt.slot * 32, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.w_empty[rw.slot]);
          if (rank == 0)
            mbar_arrive(&bars.a_full[rt.slot]);
          else
            mbar_arrive_remote_smem(&bars.a_full[rt.slot], 0);
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                       // tensor-memory lane quarter
    const int et = (warp - kEpiWarp0) * 32 + lane;
    uint8_t* boxes = smem + kOffEpi + (warp - kEpiWarp0) * 2 * kBox;
    const bool has_bias = args.bias != nullptr;
    uint32_t acc_ph = 0;
    int lt = 0;
    for (int t = cluster; t < tiles; t += nclusters, ++lt) {
      const int ab = lt & 1;
      const int mb = t % num_m, nb = t / num_m;
      const int64_t m_t0 = static_cast<int64_t>(mb) * TN;
      if (!OUT_S32) {
        // the tile's activation scales, staged once (double-buffered by tile)
        for (int j = et; j < TN; j += 128) {
          const int64_t m = m_t0 + j;
          epi_sx[ab][j] = m < M ? args.sx[m] : 0.0f;
        }
      }
      (void)warp_wait_cluster(&bars.acc_full[ab], (acc_ph >> ab) & 1, abort_flag, args.status);
      acc_ph ^= 1u << ab;
      // staged scales visible to the four warps; every wait above is bounded, so
      // all four always arrive here and then leave together on an abort
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (*abort_flag) break;
      tc_fence_after();
      const int64_t n0 = static_cast<int64_t>(nb) * TM + rank * HW + q * 32;   // this warp's first column
      const int64_t n = n0 + lane;
      const bool ncol = n < N;
      float swn = 0.0f, bn = 0.0f;
      if (!OUT_S32 && ncol) {
        swn = args.sw[n];
        if (has_bias) bn = __uint_as_float(static_cast<uint32_t>(args.bias[n]) << 16);
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * TN;
      uint32_t rr[2][32];
      tmem_ld_32x32b_x32(tbase, rr[0]);
#pragma unroll
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t (&cur)[32] = rr[c & 1];
        tmem_wait_ld();
        // the next chunk's tensor-memory load overlaps this chunk's math
        if (c + 1 < TN / 32) tmem_ld_32x32b_x32(tbase + (c + 1) * 32, rr[(c + 1) & 1]);
        const int64_t m0 = m_t0 + c * 32;
        if (m0 >= M || n0 >= N) continue;   // warp-uniform
        if (OUT_S32) {
          if (ncol) {
            int32_t* out = reinterpret_cast<int32_t*>(args.out);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (m0 + j < M) out[(m0 + j) * args.ldo + n] = static_cast<int32_t>(cur[j]) >> 4;
          }
        } else {
          uint8_t* box = boxes + (c & 1) * kBox;
          // the store that last read this box (two chunks ago) has finished reading it
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          const float* sxc = &epi_sx[ab][c * 32];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            // ((float)acc * sx) * sw (+ bias), each step rounded on its own
            const float2 s2 = *reinterpret_cast<const float2*>(sxc + j);
            const uint64_t a2 = pk2(__int2float_rn(static_cast<int32_t>(cur[j]) >> 4),
                                    __int2float_rn(static_cast<int32_t>(cur[j + 1]) >> 4));
            // the last multiply and the bias add are scalar __fmul_rn/__fadd_rn:
            // those are never contracted into an fma, while a paired
            // multiply followed by a paired add can be
            float t0, t1;
            upk2(mul2(a2, pk2(s2.x, s2.y)), t0, t1);
            float y0 = __fmul_rn(t0, swn), y1 = __fmul_rn(t1, swn);
            if (has_bias) {
              y0 = __fadd_rn(y0, bn);
              y1 = __fadd_rn(y1, bn);
            }
            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
            const uint32_t hv = *reinterpret_cast<const uint32_t*>(&h);
            // row j of the box is output row m0 + j; lane l is column n0 + l
            *reinterpret_cast<uint16_t*>(box + j * 64 + lane * 2) = static_cast<uint16_t>(hv & 0xFFFFu);
            *reinterpret_cast<uint16_t*>(box + (j + 1) * 64 + lane * 2) = static_cast<uint16_t>(hv >> 16);
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, box, static_cast<int32_t>(n0), static_cast<int32_t>(m0));
            bulk_commit_group();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_smem(&bars.acc_empty[ab], 0);
    }
    if (lane == 0) bulk_wait_group<0>();   // every store of y has completed
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
  if (cudaOccupancyMaxActiveClusters(&n, gemm_ts_kernel<OUT_S32>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  if (n > num_sms / 2) n = num_sms / 2;
  cached[dev] = n;
  return n;
}

template <int OUT_S32>
cudaError_t launch(const CUtensorMap& tmAct, const CUtensorMap& tmW, const CUtensorMap& tmY, const GemmArgs& a,
                   int64_t tiles, int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(gemm_ts_kernel<OUT_S32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, gemm_ts_kernel<OUT_S32>, tmAct, tmW, tmY, a);
}

}  // namespace

cudaError_t gemm_ts_launch(const CUtensorMap& tmAct, const CUtensorMap& tmW, const CUtensorMap& tmY,
                           const GemmArgs& a, int num_sms, cudaStream_t stream) {
  const int64_t tiles = ((a.M + TN - 1) / TN) * ((a.N + TM - 1) / TM);
  if (tiles == 0) return cudaSuccess;
  cudaError_t e = a.out_s32 ? launch<1>(tmAct, tmW, tmY, a, tiles, num_sms, stream)
                            : launch<0>(tmAct, tmW, tmY, a, tiles, num_sms, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a4
