// s4 x s4 -> s32 GEMM with the rank-one epilogue, on the sm_100a tensor cores.
//
// The page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels" (Description) applies the row and column scales only after the
// reduction over K: the inner loop multiplies integer codes into int32
// accumulators (|acc| <= 49*K), and y = acc * sx[m] * sw[n] (+ bias) is
// formed once per output.  Its kernel is an Ampere/Ada mma.sync s4 design; on sm_100a there is
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
//     four epilogue warps per CTA drain tile i while the MMAs of tile i+1 run:
//     the tile's column scales and bias are staged once in shared memory, the
//     tcgen05.ld of the next 32 columns is in flight while the current ones
//     are converted, and y = bf16(((float)acc * sx[m]) * sw[n] + bias[n]) is
//     formed with separately rounded fp32 steps (paired .f32x2 arithmetic);
//     each 32 x 32 bf16 block is staged in shared memory (64-byte swizzle)
//     and written with one TMA tensor store, which also clips the M/N tails.
//   * A second instance (CHAIN = g of the next layer) adds a requantising
//     epilogue for layer chains: after storing each 32-column chunk of y it
//     applies GELU (t * Phi(t) from a table in shared memory, which takes the
//     room of one packed stage) and the Walsh-Hadamard butterflies inside the
//     chunk, writes the chunk back over its accumulator columns, and after a
//     rotation group's last chunk runs the butterflies across the group's
//     chunks; one atomicMax per row and tile records the largest rotated
//     magnitude for the pass that quantises y for the next layer.
//   * The kernel is persistent: the clusters walk the tiles with a static
//     stride.  Every wait is bounded: an expired wait records W4A4_ERR_TIMEOUT
//     in the device status word, every role stops, the MMAs are drained and
//     the tensor memory is freed before the CTAs exit.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "gelu_table.cuh"
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
// Warp roles.  A warp runs on SM sub-partition (warp % 4).  The threads that
// issue tcgen05.mma and TMA instructions hold their sub-partition's issue
// slot for long stretches, so they share sub-partition 0 with one epilogue
// warp and no widen warp; the widen warps sit on sub-partitions 1..3 (nine
// slots: warps 1-3, 5-7, 9-11), next to one epilogue warp each (an epilogue
// warp may only read the tensor-memory lane quarter warp % 4).
// The widen warps can form kWGroups groups that take turns by k-block; with
// the shared-memory bandwidth as the limit, one group of eight warps (four
// 16-byte units per thread, the ninth slot idle) measured fastest.
constexpr int kWGroups = 1;
constexpr int kWidenWarps = 8;   // per group
constexpr int kEpiWarps = 4;
constexpr int kWarpMma = 0;
constexpr int kWarpTma = 4;
constexpr int kThreads = 16 * 32;
__device__ __forceinline__ bool is_epi_warp(int w) { return w == 8 || w >= 13; }
__device__ __forceinline__ bool is_widen_warp(int w) { return w != 0 && w != 4 && w != 8 && w < 12; }
// widen warps 1,2,3,5,6,7,9,10,11 -> 0..8
__device__ __forceinline__ int widen_index(int w) { return w - 1 - (w > 4) - (w > 8); }
static_assert(kWGroups * kWidenWarps <= 9, "nine widen warp slots");
constexpr int kTmemCols = 2 * BN;   // two int32 accumulators of BN columns

constexpr uint32_t kWideA = HM * BK;     // 16 KB
constexpr uint32_t kWideB = HN * BK;     // 16 KB
constexpr uint32_t kStage = kWideA + kWideB;
constexpr uint32_t kPackA = HM * BKP;    // 8 KB
constexpr uint32_t kPackB = HN * BKP;    // 8 KB
constexpr uint32_t kPStage = kPackA + kPackB;
constexpr uint32_t kOffPack = SWD * kStage;
// epilogue staging: per epilogue warp two 32 x 32 bf16 boxes (64-byte rows,
// 64-byte swizzle) for the TMA stores of y
constexpr uint32_t kStageBox = 32 * 64;
// Shared-memory plan by kernel form.  The requantising epilogue (CHAIN = the
// next layer's rotation group) keeps the GELU table in shared memory, in the
// room of one packed stage.
template <int CHAIN>
struct Plan {
  static constexpr int kSP = CHAIN ? SP - 1 : SP;   // packed ring depth
  static constexpr uint32_t kOffEpi = kOffPack + kSP * kPStage;
  static constexpr uint32_t kOffGelu = kOffEpi + 4 * 2 * kStageBox;
  static constexpr uint32_t kBytes = kOffGelu + (CHAIN ? kGeluTableSize * 4 : 0);
  static constexpr uint32_t kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
};

// packed 16-byte units per CTA and k-block: (HM + HN) rows x 4 units
constexpr int kUnits = (HM + HN) * (BKP / 16);
constexpr int kWidenThreads = kWidenWarps * 32;
constexpr int kUnitsPerThread = (kUnits + kWidenThreads - 1) / kWidenThreads;   // 4 (the last partly idle)

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
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

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
  for (int i = 0; i < kUnitsPerThread; ++i) {
    const int u = wt + i * kWidenThreads;
    if (u < kUnits) buf[i] = lds128(smem_u32(pstage) + u * 16);
  }
#pragma unroll
  for (int i = 0; i < kUnitsPerThread; ++i) {
    const int u = wt + i * kWidenThreads;
    if (u >= kUnits) break;
    const bool isA = u < HM * 4;
    const int uu = isA ? u : u - HM * 4;
    const int r = uu >> 2;
    const int part = uu & 3;
    uint4 c0, c1;
    widen_word16(buf[i].x, c0.x, c0.y);
    widen_word16(buf[i].y, c0.z, c0.w);
    widen_word16(buf[i].z, c1.x, c1.y);
    widen_word16(buf[i].w, c1.z, c1.w);
    const uint32_t rowp = smem_u32(stage) + (isA ? 0 : kWideA) + (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    sts128(rowp + (((2 * part) ^ sw) << 4), c0);
    sts128(rowp + (((2 * part + 1) ^ sw) << 4), c1);
  }
}

// Walsh-Hadamard butterflies over 32 values in natural (Sylvester) order,
// unnormalised.
__device__ __forceinline__ void fwht32(uint32_t (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i & h) continue;
      const float a = __uint_as_float(v[i]), b = __uint_as_float(v[i + h]);
      v[i] = __float_as_uint(a + b);
      v[i + h] = __float_as_uint(a - b);
    }
  }
}

template <int OUT_S32, int CHAIN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, GemmArgs args) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Bars bars;
  __shared__ __align__(16) float epi_sw[2][BN];
  __shared__ __align__(16) float epi_bias[2][BN];
  uint8_t* smem = align1024_shared(smem_dyn);
  constexpr int kSP = Plan<CHAIN>::kSP;
  float* gtab = reinterpret_cast<float*>(smem + Plan<CHAIN>::kOffGelu);   // requantising epilogue only

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
    for (int s = 0; s < kSP; ++s) {
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
  if constexpr (CHAIN > 0) {
    // the GELU table (filled by the host before any launch)
    for (int i = threadIdx.x; i < kGeluTableSize; i += kThreads) gtab[i] = args.gelu_tab[i];
  }
  tc_fence_before();
  cluster_sync();   // barriers and tensor memory of both CTAs are ready
  tc_fence_after();
  // launched with programmatic stream serialization: the set-up above may
  // overlap the previous kernel (the activation quantiser of a fused layer);
  // its outputs are read only after this point
  griddep_wait();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  // The tile's column scales and bias, staged once in shared memory
  // (double-buffered by tile) by the four epilogue warps, thread et taking
  // columns et, et + 128.
  auto stage_scales = [&](int t, int ab, int et) {
    if (OUT_S32) return;
    const int64_t nt0 = static_cast<int64_t>(t / num_m) * BN;
#pragma unroll
    for (int j = et; j < BN; j += 128) {
      const int64_t n = nt0 + j;
      epi_sw[ab][j] = n < N ? args.sw[n] : 0.0f;
      epi_bias[ab][j] = (n < N && args.bias != nullptr) ? __uint_as_float(static_cast<uint32_t>(args.bias[n]) << 16)
                                                        : 0.0f;
    }
  };
  // 32-column chunks [c_begin, c_end) of tile t's accumulator (buffer ab) for
  // this warp's 32 rows: y = bf16(((float)acc * sx) * sw (+ bias)) with each
  // step rounded on its own, staged per 32 x 32 block in two alternating
  // 2 KB boxes at `stage` (64-byte swizzle) and written by TMA stores.
  auto drain_chunks = [&](int t, int ab, int c_begin, int c_end, uint8_t* stage) {
    const int q = warp & 3;
    const int mb = t % num_m, nb = t / num_m;
    const int64_t nt0 = static_cast<int64_t>(nb) * BN;
    const float* sws = epi_sw[ab];
    const float* bs = epi_bias[ab];
    const int64_t m = static_cast<int64_t>(mb) * BM + rank * HM + q * 32 + lane;
    const bool mrow = m < M;
    float sxm = 0.0f;
    if (!OUT_S32 && mrow) sxm = args.sx[m];
    const uint64_t sx2 = pk2(sxm, sxm);
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * BN;
    // requantising epilogue: the largest |butterfly sum| of this row over the
    // tile's rotation groups
    float chain_amax_u = 0.0f;
    // After the butterflies inside each of a group's 32-column chunks (stored
    // back over the accumulator), the butterflies across its CHAIN / 32
    // chunks at every position; returns the group's largest |sum|.  H_g in
    // natural order is H_(g/32) on the chunk index times H_32 on the position.
    auto group_cross = [&](int c0) -> float {
      constexpr int NC = CHAIN > 0 ? CHAIN / 32 : 1;
      constexpr int PB = NC <= 4 ? 8 : 4;   // positions per pass
      float mx = 0.0f;
#pragma unroll 1
      for (int j = 0; j < 32; j += PB) {
        uint32_t v[NC][PB];
#pragma unroll
        for (int cc = 0; cc < NC; ++cc) {
          if constexpr (PB == 8) tmem_ld_32x32b_x8(tbase + (c0 + cc) * 32 + j, v[cc]);
          else tmem_ld_32x32b_x4(tbase + (c0 + cc) * 32 + j, v[cc]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int pp = 0; pp < PB; ++pp) {
          float a[NC];
#pragma unroll
          for (int cc = 0; cc < NC; ++cc) a[cc] = __uint_as_float(v[cc][pp]);
#pragma unroll
          for (int h = 1; h < NC; h <<= 1) {
#pragma unroll
            for (int cc = 0; cc < NC; ++cc) {
              if (cc & h) continue;
              const float x0 = a[cc], x1 = a[cc + h];
              a[cc] = x0 + x1;
              a[cc + h] = x0 - x1;
            }
          }
#pragma unroll
          for (int cc = 0; cc < NC; ++cc) mx = fmaxf(mx, fabsf(a[cc]));
        }
      }
      return mx;
    };
    // one chunk: its tensor-memory load (issued one chunk earlier) is waited
    // for, the next chunk's load is issued into the other buffer so that it
    // overlaps this chunk's math, and the chunk is converted and stored
    auto chunk = [&](int c, uint32_t (&cur)[32], uint32_t (&nxt)[32]) {
      tmem_wait_ld();
      if (c + 1 < c_end) tmem_ld_32x32b_x32(tbase + (c + 1) * 32, nxt);
      const int64_t n0 = nt0 + c * 32;
      if (n0 >= N) return;   // warp-uniform; the tensor-memory loads above stay aligned
      const bool full = n0 + 32 <= N;
      if (OUT_S32) {
        if (!mrow) return;
        int32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = static_cast<int32_t>(cur[i]) >> 8;
        int32_t* dst = reinterpret_cast<int32_t*>(args.out) + m * args.ldo + n0;
        if (full) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<int4*>(dst)[i] = make_int4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (n0 + i < N) dst[i] = v[i];
        }
        return;
      }
      uint32_t packed[16];
      const float* swc = sws + c * 32;
      const float* bc = bs + c * 32;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // ((float)acc * sx) * sw (+ bias), each step rounded on its own
        const uint64_t a2 = pk2(__int2float_rn(static_cast<int32_t>(cur[2 * i]) >> 8),
                                __int2float_rn(static_cast<int32_t>(cur[2 * i + 1]) >> 8));
        const float2 w2 = *reinterpret_cast<const float2*>(swc + 2 * i);
        uint64_t y2 = mul2(mul2(a2, sx2), pk2(w2.x, w2.y));
        if (args.bias != nullptr) {
          const float2 b2 = *reinterpret_cast<const float2*>(bc + 2 * i);
          y2 = add2(y2, pk2(b2.x, b2.y));
        }
        float y0, y1;
        upk2(y2, y0, y1);
        const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
        packed[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      // stage the 32 x 32 block (row = lane, 64-byte swizzle: chunk j of
      // row r at chunk j ^ ((r >> 1) & 3); conflict-free for this pattern)
      uint8_t* box = stage + ((c & 1) * kStageBox);
      // the store that last used this box (two chunks ago, possibly in the
      // previous tile) must have finished reading it
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(box + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      fence_async_shared();
      __syncwarp();
      // a box whose first row is past M stores nothing (rows past M inside
      // a box are clipped by the tensor map)
      if (lane == 0 && m < M) {
        tma_store_2d(&tmY, box, static_cast<int32_t>(n0), static_cast<int32_t>(m));
        bulk_commit_group();
      }
      if constexpr (CHAIN > 0) {
        // the next layer's input: GELU of the bf16 outputs just stored, then
        // the rotation's butterflies inside the chunk, written back over the
        // chunk's accumulator columns (nothing reads them after this tile)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // GELU = t * Phi(t), Phi from the table, as the activation kernel forms it
          float p0, p1;
          gelu_phi_word(packed[i], gtab, p0, p1);
          cur[2 * i] = __float_as_uint(__fmul_rn(__uint_as_float(packed[i] << 16), p0));
          cur[2 * i + 1] = __float_as_uint(__fmul_rn(__uint_as_float(packed[i] & 0xFFFF0000u), p1));
        }
        fwht32(cur);
        tmem_st_32x32b_x32(tbase + c * 32, cur);
        if ((c + 1) % (CHAIN / 32) == 0) {
          tmem_wait_st();
          chain_amax_u = fmaxf(chain_amax_u, group_cross(c + 1 - CHAIN / 32));
        }
      }
    };
    // chunk ranges start on an even chunk and hold an even number of them:
    // even chunks use buffer r0, odd ones r1 (static register indexing)
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(tbase + c_begin * 32, r0);
    for (int c = c_begin; c < c_end; c += 2) {
      chunk(c, r0, r1);
      chunk(c + 1, r1, r0);
    }
    if constexpr (CHAIN > 0) {
      // the row's amax over this tile's groups, as fp32 bits (non-negative
      // floats order like their bit patterns); 1/sqrt(g) applied once
      // (rounding is monotonic, so max fl(|u| / sqrt g) = fl(max |u| / sqrt g))
      constexpr float kNorm = CHAIN == 64 ? 0.125f : (CHAIN == 256 ? 0.0625f : 0.0883883476483184405f);
      if (mrow) atomicMax(args.chain_amax + m, __float_as_uint(chain_amax_u * kNorm));
    }
  };

  if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      uint32_t ws = 0, wph = 0, acc_ph = 0;
      int lt = 0;
      bool ok = true;
      for (int t = cluster; t < tiles && ok; t += nclusters, ++lt) {
        const int ab = lt & 1;
        if (!mbar_wait_cluster(&bars.acc_empty[ab], ((acc_ph >> ab) & 1) ^ 1, abort_flag, args.status, args.wait_ns)) {
          ok = false;
          break;
        }
        acc_ph ^= 1u << ab;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&bars.wide_full[ws], wph, abort_flag, args.status, args.wait_ns)) {
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
      // on the even CTA's barrier, published with a release fence restricted
      // to shared memory and a relaxed cluster arrive (a full cluster-scope
      // release costs about a microsecond).  The widen warps only release
      // locally; this thread forwards in the order the MMA consumes the slots.
      uint32_t ws = 0, wph = 0;
      for (int t = cluster; t < tiles; t += nclusters) {
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars.wide_full[ws], wph, abort_flag, args.status, args.wait_ns)) { ok = false; break; }
          mbar_arrive_remote_smem(&bars.wide_full[ws], 0);
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
          if (!mbar_wait(&bars.packed_empty[ps], ph ^ 1, abort_flag, args.status, args.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.packed_full[ps], kPStage);
          uint8_t* dst = smem + kOffPack + ps * kPStage;
          tma_load_2d(dst, &tmA, &bars.packed_full[ps], kb * BKP, mb * BM + static_cast<int>(rank) * HM);
          tma_load_2d(dst + kPackA, &tmB, &bars.packed_full[ps], kb * BKP, nb * BN + static_cast<int>(rank) * HN);
          ++issued;
          if (++ps == kSP) { ps = 0; ph ^= 1; }
        }
      }
      {
        // Let every copy this thread issued land before the CTA goes away:
        // after an abort some may never be consumed, and an abort raised by
        // another role after this loop ended would otherwise go unnoticed here.
        // In a normal run every phase waited for has completed already.
        for (int s2 = 0; s2 < kSP && s2 < issued; ++s2) {
          const int64_t n_s = issued / kSP + (s2 < issued % kSP ? 1 : 0);
          (void)mbar_wait(&bars.packed_full[s2], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (is_widen_warp(warp)) {
    // ------------------------------------------------------------ widen warps
    const int grp = widen_index(warp) / kWidenWarps;
    const int wt = (widen_index(warp) % kWidenWarps) * 32 + lane;
    uint32_t ps = 0, ph = 0, ws = 0, wph = 0;
    uint32_t gk = 0;
    bool ok = grp < kWGroups;   // spare warp slots stay idle
    for (int t = cluster; t < tiles && ok; t += nclusters) {
      for (int kb = 0; kb < num_kb; ++kb, ++gk) {
        if (static_cast<int>(gk % kWGroups) != grp) {
          if (++ps == kSP) { ps = 0; ph ^= 1; }
          if (++ws == SWD) { ws = 0; wph ^= 1; }
          continue;
        }
        if (!warp_wait(&bars.packed_full[ps], ph, abort_flag, args.status, args.wait_ns) ||
            !warp_wait_cluster(&bars.wide_empty[ws], wph ^ 1, abort_flag, args.status, args.wait_ns)) { ok = false; break; }
        widen_units(smem + kOffPack + ps * kPStage, smem + ws * kStage, wt);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.wide_full[ws]);
          mbar_arrive(&bars.packed_empty[ps]);
        }
        if (++ps == kSP) { ps = 0; ph ^= 1; }
        if (++ws == SWD) { ws = 0; wph ^= 1; }
      }
    }
  } else if (is_epi_warp(warp)) {
    // ------------------------------------------------------------ epilogue warps
    // every tile but the cluster's last (drained by all sixteen warps below)
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    const int et = q * 32 + lane;   // 0..127 across the four epilogue warps
    uint8_t* epi_stage = smem + Plan<CHAIN>::kOffEpi + q * 2 * kStageBox;
    uint32_t acc_ph = 0;
    int lt = 0;
    for (int t = cluster; t + nclusters < tiles; t += nclusters, ++lt) {
      const int ab = lt & 1;
      stage_scales(t, ab, et);
      (void)warp_wait_cluster(&bars.acc_full[ab], (acc_ph >> ab) & 1, abort_flag, args.status, args.wait_ns);
      acc_ph ^= 1u << ab;
      // staged scales visible to the four warps; every wait above is bounded, so
      // all four always arrive here.  The barrier ORs their views of the abort
      // flag, which another thread may raise at any moment, so all four leave
      // together (and meet the same barriers below) or none does.
      if (bar_sync_or(1, 128, *abort_flag != 0)) break;
      tc_fence_after();
      drain_chunks(t, ab, 0, BN / 32, epi_stage);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_smem(&bars.acc_empty[ab], 0);
    }
  }

  // ---- the cluster's last tile, drained by all sixteen warps: nothing else
  // overlaps this epilogue, so each of the four warps of a tensor-memory lane
  // quarter (warp % 4) takes two of the eight 32-column chunks, staging its
  // boxes in the widened ring (idle once the last accumulator is complete).
  // Every warp reaches the barrier below exactly once, also after an abort.
  __syncwarp();
  {
    const int lt_last = (tiles - cluster + nclusters - 1) / nclusters - 1;
    const int t_last = cluster + lt_last * nclusters;
    const int ab = lt_last & 1;
    if (is_epi_warp(warp)) {
      stage_scales(t_last, ab, (warp & 3) * 32 + lane);
      // the last accumulator's phase: uses of buffer ab before it, mod 2
      (void)warp_wait_cluster(&bars.acc_full[ab], static_cast<uint32_t>((lt_last >> 1) & 1), abort_flag,
                              args.status, args.wait_ns);
    }
    // one verdict for all sixteen warps (nothing raises the flag after this
    // barrier, but the OR makes the branch uniform by construction)
    const bool aborted = bar_sync_or(2, 512, *abort_flag != 0);
    if (!aborted) {
      tc_fence_after();
      if constexpr (CHAIN > 0) {
        // a rotation group spans several chunks: the four epilogue warps
        // drain the whole tile, as for the other tiles
        if (is_epi_warp(warp)) drain_chunks(t_last, ab, 0, BN / 32, smem + Plan<CHAIN>::kOffEpi + (warp & 3) * 2 * kStageBox);
      } else {
        const int part = warp >> 2;   // 0..3 within the lane quarter
        drain_chunks(t_last, ab, 2 * part, 2 * part + 2, smem + warp * 2 * kStageBox);
      }
    }
    if (lane == 0) bulk_wait_group_read<0>();   // every store has read its staging box
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
template <int OUT_S32, int CHAIN>
int max_clusters(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
  if (cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Plan<CHAIN>::kAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<OUT_S32, CHAIN>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  if (n > num_sms / 2) n = num_sms / 2;
  cached[dev] = n;
  return n;
}

template <int OUT_S32, int CHAIN>
cudaError_t launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY, const GemmArgs& a,
                   int64_t tiles, int num_sms, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<OUT_S32, CHAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Plan<CHAIN>::kAlloc));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t cmax = max_clusters<OUT_S32, CHAIN>(num_sms);
  const int grid = static_cast<int>(2 * (tiles < cmax ? tiles : cmax));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Plan<CHAIN>::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<OUT_S32, CHAIN>, tmA, tmB, tmY, a);
}

}  // namespace

cudaError_t gemm_tc_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY, const GemmArgs& a,
                           int num_sms, cudaStream_t stream) {
  const int64_t tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  if (tiles == 0) return cudaSuccess;
  cudaError_t e;
  if (a.out_s32) {
    e = launch<1, 0>(tmA, tmB, tmY, a, tiles, num_sms, stream);
  } else if (a.chain_g == 0) {
    e = launch<0, 0>(tmA, tmB, tmY, a, tiles, num_sms, stream);
  } else if (a.chain_g == 64) {
    e = launch<0, 64>(tmA, tmB, tmY, a, tiles, num_sms, stream);
  } else if (a.chain_g == 128) {
    e = launch<0, 128>(tmA, tmB, tmY, a, tiles, num_sms, stream);
  } else if (a.chain_g == 256) {
    e = launch<0, 256>(tmA, tmB, tmY, a, tiles, num_sms, stream);
  } else {
    return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a4
