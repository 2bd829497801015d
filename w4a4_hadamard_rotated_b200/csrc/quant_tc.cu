// Rotate + per-row int4 quantise + pack with the blockwise Walsh-Hadamard
// transform on the tensor cores (bf16 rows, no activation, g in {64, 128},
// K / g <= 128).  Same result as the register-butterfly kernel of quant.cu
// (the ConvRot activation pass of page "[PR #63] int4_tensorwise: W4A4 layout
// (+ConvRot) with fused CUDA kernels", Description), with the rotation done as
// the dense product it is: the group sums u = x_group . H_g, with H_g the
// Sylvester Hadamard matrix (entries +-1, exact in bf16), are exact products
// of bf16 values summed in fp32 -- only the order of the fp32 additions
// differs from the butterflies.
//
// B200 design
//   * A tile is P whole rows, viewed as P * K/g rows of g elements (one row
//     per group): one TMA load of the 3-D view {64 elements, K/g groups, P
//     rows} per 64-element chunk lands them as consecutive 128-byte rows in
//     the 128-byte-swizzle K-major layout the MMA reads, group j of row p at
//     row p * K/g + j.  The ring is 2 tiles deep and two CTAs share an SM.
//   * One thread issues g/16 tcgen05.mma.kind::f16 (M = 128 group rows, N = g,
//     K = 16) per tile against H_g, which every CTA builds once in shared
//     memory; fp32 accumulators in tensor memory, double-buffered.
//   * Two groups of four epilogue warps take alternate tiles; thread = tensor
//     memory lane = (row p, group j).  Pass 1 reads its g sums and reduces
//     the row amax with shared-memory atomics on the float bits (one named
//     barrier per tile, triple-buffered slots); pass 2 reads them again and
//     quantises with the arithmetic of quant.cu: s = amax / 7 in fp32, code =
//     round-half-even of u * (norm / s) by one fused multiply-add with a magic
//     number, packed 8 codes per word by a Horner chain, 64 contiguous bytes
//     per thread.
//   * Every wait is bounded; an expired wait records W4A4_ERR_TIMEOUT and
//     every role stops, drains and frees tensor memory before the CTA exits.
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4.h"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int kLanes = 128;        // MMA M: one (row, group) per tensor-memory lane
constexpr int kStages = 2;         // x ring depth (tiles); two CTAs share an SM
constexpr int kEpiGroups = 2;      // epilogue warp groups, alternating tiles
constexpr int kThreadsTc = (2 + 4 * kEpiGroups) * 32;
constexpr int kMaxRowsTile = 128;

// 1.5 * 2^23 + 8: adding it to |q| <= 7.5 rounds q to an integer k, half to
// even, and leaves k + 8 (in 1..15) in the low four bits of the sum.
constexpr float kMagic8 = 12582920.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;   // bits of 1.5 * 2^23
// Horner-packing eight sums (kMagicBits + n_e) as sum_e bits_e * 16^e leaves
// this constant on top of the nibbles n_e (mod 2^32).
constexpr uint32_t kHornerBias = kMagicBits * 0x11111111u;

template <int G>
struct TcLayout {
  static constexpr int kChunks = G / 64;                    // 128-byte K chunks per group row
  static constexpr uint32_t kChunkBytes = kLanes * 128;     // one K chunk of the 128-row A tile
  static constexpr uint32_t kStage = kChunks * kChunkBytes;
  static constexpr uint32_t kHChunk = G * 128;               // one K chunk of H (G rows x 128 B)
  static constexpr uint32_t kOffH = 0;
  static constexpr uint32_t kOffX = kOffH + kChunks * kHChunk;
  static constexpr uint32_t kBytes = kOffX + kStages * kStage;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 2 * G;               // two accumulators of G fp32 columns
  static_assert(kOffX % 1024 == 0, "1024-byte aligned stages");
};

struct TcBars {
  uint64_t full[kStages];       // TMA transaction barrier
  uint64_t empty[kStages];      // one MMA commit
  uint64_t acc_full[2];         // one MMA commit
  uint64_t acc_empty[2];        // four epilogue warps
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  unsigned int row_amax[kEpiGroups][3][kMaxRowsTile];
};

__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

template <int G>
__global__ void __launch_bounds__(kThreadsTc, 2)
    rotate_quant_tc_kernel(const __grid_constant__ CUtensorMap tmX, int64_t M, int K, int rows_per_tile,
                           int8_t* __restrict__ out, float* __restrict__ scale, unsigned int* status,
                           unsigned long long wait_ns) {
  using Lay = TcLayout<G>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ TcBars bars;
  uint8_t* smem = align1024_shared(smem_dyn);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = rows_per_tile;
  const int Gg = K / G;                 // groups per row
  const int64_t ntiles = (M + P - 1) / P;
  const float norm = G == 64 ? 0.125f : 0.0883883476483184405f;   // 1/sqrt(g) in fp32

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 4);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();   // the barriers are visible to the copy engine
    tma_prefetch_desc(&tmX);
    // Launched with programmatic stream serialization: x may be the previous
    // kernel's output, so it is read only after that grid has finished.  The
    // first ring stages are issued now, ahead of the set-up below.
    griddep_wait();
    int pre = 0;
    for (int64_t t = blockIdx.x; t < ntiles && pre < kStages; t += gridDim.x, ++pre) {
      mbar_arrive_expect_tx(&bars.full[pre], Lay::kChunks * 128u * Gg * P);
#pragma unroll
      for (int h = 0; h < Lay::kChunks; ++h)
        tma_load_3d(smem + Lay::kOffX + pre * Lay::kStage + h * Lay::kChunkBytes, &tmX, &bars.full[pre], h * 64, 0,
                    static_cast<int32_t>(t * P));
    }
  }
  for (int i = threadIdx.x; i < kEpiGroups * 3 * kMaxRowsTile; i += blockDim.x) (&bars.row_amax[0][0][0])[i] = 0u;
  // H_g as the MMA's B operand (N = g output columns c, K = g inputs k),
  // K-major in 128-byte chunks of 64 inputs, 128-byte swizzle: 16-byte unit
  // u of row c in chunk h at unit u ^ (c & 7).  H[k][c] = (-1)^popcount(k & c).
  for (int idx = threadIdx.x; idx < Lay::kChunks * G * 8; idx += blockDim.x) {
    const int h = idx / (G * 8);
    const int c = (idx / 8) % G;
    const int u = idx % 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k0 = h * 64 + u * 8 + 2 * e;
      const uint32_t lo = (__popc(k0 & c) & 1) ? 0xBF80u : 0x3F80u;
      const uint32_t hi = (__popc((k0 + 1) & c) & 1) ? 0xBF80u : 0x3F80u;
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(smem + Lay::kOffH + h * Lay::kHChunk + (c >> 3) * 1024 + (c & 7) * 128 +
                              ((u ^ (c & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  fence_async_shared();   // H is read by the tensor cores
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // nothing below writes global memory before the previous grid has finished;
  // only then may the next kernel of the stream (the GEMM of a fused layer)
  // be scheduled -- it waits for this grid's writes before it reads them
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++issued) {
        const int s = issued % kStages;
        if (issued < kStages) continue;   // issued before the set-up
        if (!mbar_wait(&bars.empty[s], ((issued / kStages) & 1) ^ 1, abort_flag, status, wait_ns)) break;
        mbar_arrive_expect_tx(&bars.full[s], Lay::kChunks * 128u * Gg * P);
#pragma unroll
        for (int h = 0; h < Lay::kChunks; ++h)
          tma_load_3d(smem + Lay::kOffX + s * Lay::kStage + h * Lay::kChunkBytes, &tmX, &bars.full[s], h * 64, 0,
                      static_cast<int32_t>(t * P));
      }
      {
        // Let every copy this thread issued land before the CTA goes away:
        // after an abort some are never consumed, and an abort raised by
        // another role after this loop ended would otherwise go unnoticed
        // here.  In a normal run these phases have all completed already.
        for (int s = 0; s < kStages && s < issued; ++s) {
          const int n_s = issued / kStages + (s < issued % kStages ? 1 : 0);
          (void)mbar_wait(&bars.full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kLanes, G);
      int i = 0;
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
        const int s = i % kStages;
        const int b = i & 1;
        if (!mbar_wait(&bars.acc_empty[b], ((i >> 1) & 1) ^ 1, abort_flag, status, wait_ns)) break;
        if (!mbar_wait(&bars.full[s], (i / kStages) & 1, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + b * G;
#pragma unroll
        for (int h = 0; h < Lay::kChunks; ++h) {
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + Lay::kOffX + s * Lay::kStage + h * Lay::kChunkBytes));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + Lay::kOffH + h * Lay::kHChunk));
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) mma_bf16(d, ad + 2 * ks, bd + 2 * ks, idesc, (h | ks) != 0 ? 1u : 0u);
        }
        mma_commit(&bars.empty[s]);
        mma_commit(&bars.acc_full[b]);
      }
      // every issued MMA completes before tensor memory is released
      mma_commit(&bars.drain);
      (void)mbar_wait(&bars.drain, 0, nullptr, nullptr, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // group e takes the CTA's tiles i with i % 2 == e (accumulator e); warps
    // 2..5 and 6..9 cover the four tensor-memory lane quarters (warp % 4)
    const int e = (warp - 2) / 4;
    const int q = warp & 3;
    const int li = q * 32 + lane;           // tensor-memory lane = (row p, group j)
    const int p = li / Gg;
    const int j = li - p * Gg;
    const bool lane_used = p < P;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint64_t mg2 = pk2(kMagic8, kMagic8);
    int i = 0, k = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      if ((i & 1) != e) continue;
      const int b = e;
      const int set = k % 3;
      // An expired wait makes every later one return at once; the group still
      // reaches its named barrier on every tile, so no warp is left waiting.
      bool ok = *abort_flag == 0 && warp_wait(&bars.acc_full[b], (i >> 1) & 1, abort_flag, status, wait_ns);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;   // warp-uniform: the tensor-memory loads are collective
      tc_fence_after();
      const int64_t row = t * P + p;
      const bool valid = ok && lane_used && row < M;
      // pass 1: this group's largest |u|
      float mx = 0.0f;
      if (ok) {
        // two 32-column loads in flight per round trip
#pragma unroll 1
        for (int c = 0; c < G / 32; c += 2) {
          uint32_t v[2][32];
          tmem_ld_32x32b_x32(tl + b * G + c * 32, v[0]);
          tmem_ld_32x32b_x32(tl + b * G + c * 32 + 32, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 32; ++n) mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(v[0][n])), fabsf(__uint_as_float(v[1][n]))));
        }
      }
      // max_k fl(|u_k| * norm) = fl(max_k |u_k| * norm): rounding is monotonic
      if (valid) atomicMax(&bars.row_amax[e][set][p], __float_as_uint(mx * norm));
      asm volatile("bar.sync %0, 128;" ::"r"(1 + e) : "memory");
      // the slots of (k + 2) % 3 were last read one tile ago and are next
      // written after the coming barrier
      if (li < P) bars.row_amax[e][(k + 2) % 3][li] = 0u;
      float ni = 0.0f;
      int8_t* dst = out;
      if (valid) {
        const float amax_r = __uint_as_float(bars.row_amax[e][set][p]);
        const float sc = amax_r / 7.0f;   // fp32 division, as the method states
        if (j == 0) scale[row] = sc;
        ni = sc > 0.0f ? norm * (1.0f / sc) : 0.0f;
        dst = out + row * static_cast<int64_t>(K / 2) + j * (G / 2);
      }
      if (ok) {
        // pass 2: codes, eight per word (low nibble first), 16 bytes per 32
        // sums; every lane of the warp runs the collective loads, only the
        // lanes of real rows store
        const uint64_t ni2 = pk2(ni, ni);
        uint32_t vb[2][32];
        tmem_ld_32x32b_x32(tl + b * G, vb[0]);
#pragma unroll
        for (int c = 0; c < G / 32; ++c) {
          uint32_t (&v)[32] = vb[c & 1];
          tmem_wait_ld();
          // the next chunk's load overlaps this chunk's arithmetic
          if (c + 1 < G / 32) tmem_ld_32x32b_x32(tl + b * G + (c + 1) * 32, vb[(c + 1) & 1]);
          uint32_t wd[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t acc = 0u;
#pragma unroll
            for (int n = 7; n >= 1; n -= 2) {
              const uint64_t f = fma2(pk2(__uint_as_float(v[8 * w + n]), __uint_as_float(v[8 * w + n - 1])), ni2, mg2);
              float f1, f0;
              upk2(f, f1, f0);
              acc = acc * 16u + __float_as_uint(f1);
              acc = acc * 16u + __float_as_uint(f0);
            }
            wd[w] = (acc - kHornerBias) ^ 0x88888888u;
          }
          if (valid) *reinterpret_cast<uint4*>(dst + c * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[b]);
      ++k;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

template <int G>
cudaError_t launch_tc(const uint16_t* x, int64_t M, int K, int64_t ldx, int8_t* out, float* scale, int num_sms,
                      unsigned int* status, cudaStream_t stream) {
  using Lay = TcLayout<G>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(rotate_quant_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Lay::kAlloc));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // P whole rows per tile (P * K/g <= 128 lanes).  The CTAs walk the tiles
  // with a grid stride, so the last CTA to finish does ceil(tiles / CTAs)
  // tiles of P rows: P minimises that row count (the larger P on a tie).
  const int Gg = K / G;
  const int64_t ctas = 2 * static_cast<int64_t>(num_sms);   // two resident per SM
  int P = 1;
  int64_t best = -1;
  for (int cand = kLanes / Gg; cand >= 1; --cand) {
    const int64_t tiles_c = (M + cand - 1) / cand;
    const int64_t rows_last = (tiles_c + ctas - 1) / ctas * cand;
    if (best < 0 || rows_last < best) {
      best = rows_last;
      P = cand;
    }
  }
  CUtensorMap tm;
  if (group_rows_map(&tm, x, M, K, ldx, G, P) != W4A4_OK) return cudaErrorInvalidValue;
  const int64_t ntiles = (M + P - 1) / P;
  const int grid = static_cast<int>(ntiles < ctas ? ntiles : ctas);
  // programmatic stream serialization: the set-up (barriers, H, tensor
  // memory) may overlap the previous kernel's tail; the kernel waits for it
  // before touching global memory
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = Lay::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, rotate_quant_tc_kernel<G>, tm, M, K, P, out, scale, status, wait_limit_ns());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t rotate_quant_bf16_tc(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                                 int num_sms, unsigned int* status, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  if (K % g != 0 || K / g > kLanes) return cudaErrorNotSupported;
  if (g == 64) return launch_tc<64>(x, M, K, ldx, out, scale, num_sms, status, stream);
  if (g == 128) return launch_tc<128>(x, M, K, ldx, out, scale, num_sms, status, stream);
  return cudaErrorNotSupported;
}

}  // namespace w4a4
