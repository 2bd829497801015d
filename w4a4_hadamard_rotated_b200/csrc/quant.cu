// Fused ConvRot rotate + per-row int4 quantise + pack (the activation kernel
// of page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels", Description: "FHT rotation ... + rowwise int4 quantize + pack in
// one pass").  The same kernel, with fp32 input, prepares the weights offline.
//
// B200 design (an HBM-bound pass that is close to ALU-bound as well: 2 bytes
// read, half a byte written, ~log2(g) adds per code)
//   * Every row is split into S = K/128 slabs of 128 consecutive elements and
//     each thread owns one slab, entirely in registers, as 64 packed fp32
//     pairs (element i, element i + 64).  Six radix-2 Walsh-Hadamard stages run
//     as paired sm_100 add/sub.f32x2 instructions (two lanes per instruction),
//     the seventh (distance 64, g >= 128) pairs the two halves of a register;
//     g = 256 spans two slabs held by adjacent lanes and takes one shuffle
//     stage.
//   * The kernel is persistent: a CTA walks row tiles (P whole rows) with a
//     grid stride, and one thread streams the rows of the coming tiles into a
//     3-4 deep shared-memory ring with bulk-async (TMA) copies, so HBM reads
//     stay in flight during the arithmetic and every SM gets the same, fully
//     coalesced request pattern.  The one CTA barrier per tile (for the row
//     amax) also frees the ring slot that tile used.
//   * A lane reads its slab from shared memory in XOR-swizzled 16-byte chunks
//     (chunk j from position j ^ L, L = lane & 7), which keeps the 128-bit
//     shared loads free of bank conflicts.  Permuting the input of a Walsh-Hadamard
//     transform by an XOR of the index only flips signs of the output:
//     H(x[. ^ a])[i] = (-1)^popcount(i & a) H(x)[i].  The sign of each output
//     chunk is folded into the quantisation multiplier; the quantiser is odd
//     (round-half-even and the clamp are symmetric), so the codes are exact.
//   * The row amax is reduced with shared-memory atomics on the float bits
//     (triple-buffered slots, one barrier per tile), and s = amax / 7 in fp32.
//     The code is round-half-even of r * (1/s) in fp32: a reciprocal multiply
//     (with 1/sqrt(g) and the chunk sign folded in) and a magic-number rounding
//     put the code in the low mantissa bits, and a Horner chain of integer
//     multiply-adds packs 8 codes per word as they are made.  The product is
//     within 3 ulp of the quotient r / s, so a code can differ from the one of
//     the exact quotient only for values within ~4e-7 (relative) of a rounding
//     boundary; exact ties with power-of-two scales stay exact.
//   * Codes are stored low nibble first, 64 contiguous bytes per thread, with
//     128-bit stores.  A second output mode (used by the fused layer, whose
//     tensor-core GEMM reads the activation operand as bytes) stores every
//     code as one int8, 128 contiguous bytes per thread, from the same
//     magic-number sums Horner-packed four per word.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {

constexpr int kSlab = 128;     // elements per thread
constexpr int kHalf = 64;      // packed pairs per thread
constexpr int kMaxRows = 64;   // rows per CTA tile

template <typename TIn>
struct InTraits;
template <>
struct InTraits<uint16_t> {  // bf16 bits
  static constexpr int kChunkElems = 8;
  static constexpr int kMaxThreads = 256;
};
template <>
struct InTraits<float> {     // fp32 weights (offline)
  static constexpr int kChunkElems = 4;
  static constexpr int kMaxThreads = 192;
};
constexpr int kMaxStages = 4;
constexpr size_t kRingBytes = 200 * 1024;   // shared memory for the row ring

// ---- packed fp32 pairs (sm_100 .f32x2 arithmetic)
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ float gelu_erf(float t) {
  return 0.5f * t * (1.0f + erff(t * 0.70710678118654752f));
}

// Element e of a 16-byte chunk as fp32.
__device__ __forceinline__ float elem(const uint4 w, int e, const uint16_t*) {
  const uint32_t word = e < 2 ? w.x : (e < 4 ? w.y : (e < 6 ? w.z : w.w));
  return (e & 1) ? __uint_as_float(word & 0xFFFF0000u) : __uint_as_float(word << 16);
}
__device__ __forceinline__ float elem(const uint4 w, int e, const float*) {
  return __uint_as_float(e == 0 ? w.x : (e == 1 ? w.y : (e == 2 ? w.z : w.w)));
}

// One radix-2 butterfly stage at distance H (< 64) over the packed pairs.
template <int H>
__device__ __forceinline__ void fht_stage2(uint64_t (&V)[kHalf]) {
#pragma unroll
  for (int i0 = 0; i0 < kHalf; i0 += 2 * H) {
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const uint64_t a = V[i0 + i], c = V[i0 + i + H];
      V[i0 + i] = add2(a, c);
      V[i0 + i + H] = sub2(a, c);
    }
  }
}

// 1.5 * 2^23 + 8: adding it to |q| <= 7.5 rounds q to an integer k, half to
// even, and leaves k + 8 (in 1..15) in the low four bits of the sum.
constexpr float kMagic8 = 12582920.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;   // bits of 1.5 * 2^23
// Horner-packing eight sums (kMagicBits + n_e) as sum_e bits_e * 16^e leaves
// this constant on top of the nibbles n_e (mod 2^32).
constexpr uint32_t kHornerBias = kMagicBits * 0x11111111u;
// The same for four sums per word in base 256 (one byte per code).
constexpr uint32_t kHornerBias8 = kMagicBits * 0x01010101u;
// Bytes n in 1..15 (code + 8) to the int8 codes n - 8, without borrows
// between bytes: every byte is 0x81..0x8F before the subtraction.
__device__ __forceinline__ uint32_t bytes_to_codes(uint32_t nb) {
  return ((nb | 0x80808080u) - 0x08080808u) ^ 0x80808080u;
}

template <typename TIn, int G, int ACT, int OUT8>
__global__ void __launch_bounds__(InTraits<TIn>::kMaxThreads, 1)
    rotate_quant_pack_kernel(const TIn* __restrict__ x, int64_t M, int K, int64_t ldx, int rows_per_tile,
                             int nstages, int8_t* __restrict__ out, float* __restrict__ scale,
                             unsigned int* status) {
  constexpr int C = InTraits<TIn>::kChunkElems;
  constexpr int NCH = kSlab / C;   // 16-byte chunks per slab

  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kMaxStages];
  __shared__ unsigned int row_amax[3][kMaxRows];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int S = K / kSlab;
  const int P = rows_per_tile;
  const int p = tid / S;       // row inside the tile
  const int s = tid - p * S;   // slab inside the row
  const bool active = p < P;
  const int L = lane & 7;      // chunk swizzle of this lane
  const float norm = G == 64 ? 0.125f : (G == 256 ? 0.0625f : 0.0883883476483184405f);
  const int64_t ntiles = (M + P - 1) / P;
  const size_t row_bytes = static_cast<size_t>(K) * sizeof(TIn);
  const size_t stage_bytes = static_cast<size_t>(P) * row_bytes;

  for (int i = tid; i < 3 * kMaxRows; i += blockDim.x) (&row_amax[0][0])[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < kMaxStages; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // Thread 0 streams tile `tl` into ring slot `st`.
  auto issue = [&](int64_t tl, int st) {
    const int64_t r0 = tl * P;
    const int rows = static_cast<int>(M - r0 < P ? M - r0 : P);
    uint8_t* dst = ring + st * stage_bytes;
    mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(rows * row_bytes));
    if (ldx == K) {
      bulk_load(dst, x + r0 * ldx, static_cast<uint32_t>(rows * row_bytes), &full[st]);
    } else {
      for (int r = 0; r < rows; ++r)
        bulk_load(dst + r * row_bytes, x + (r0 + r) * ldx, static_cast<uint32_t>(row_bytes), &full[st]);
    }
  };
  int64_t issued = 0;   // copies thread 0 has issued (counts only in thread 0)
  if (tid == 0) {
    for (int i = 0; i < nstages; ++i) {
      const int64_t tl = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
      if (tl < ntiles) {
        issue(tl, i);
        ++issued;
      }
    }
  }

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int st = it % nstages;
    const int64_t row = tile * P + p;
    const bool ok = warp_wait(&full[st], static_cast<uint32_t>((it / nstages) & 1), &abort_flag, status);
    const bool valid = active && row < M && ok;

    // Slot chunk j (j < NCH/2) fills the low halves of V[C*j .. C*j+C), slot
    // chunk j + NCH/2 the high halves: V[i] = (element i, element i + 64).
    uint64_t V[kHalf];
    {
      const uint8_t* src = ring + st * stage_bytes + p * row_bytes + static_cast<size_t>(s) * kSlab * sizeof(TIn);
#pragma unroll
      for (int j = 0; j < NCH / 2; ++j) {
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = make_uint4(0u, 0u, 0u, 0u);
        if (valid) {
          lo = *reinterpret_cast<const uint4*>(src + ((j ^ L) << 4));
          hi = *reinterpret_cast<const uint4*>(src + (((j + NCH / 2) ^ L) << 4));
        }
#pragma unroll
        for (int e = 0; e < C; ++e) {
          float a = elem(lo, e, x);
          float b = elem(hi, e, x);
          if (ACT == 1) {
            a = gelu_erf(a);
            b = gelu_erf(b);
          }
          V[j * C + e] = pk2(a, b);
        }
      }
    }

    // Walsh-Hadamard butterflies: distances 1..32 on the pairs, 64 inside a pair.
    fht_stage2<1>(V);
    fht_stage2<2>(V);
    fht_stage2<4>(V);
    fht_stage2<8>(V);
    fht_stage2<16>(V);
    fht_stage2<32>(V);
    if (G >= 128) {
#pragma unroll
      for (int i = 0; i < kHalf; ++i) {
        float a, b;
        upk2(V[i], a, b);
        V[i] = pk2(a + b, a - b);
      }
    }
    if (G == 256) {
      // Last stage across the two slabs of a group, held by lanes l and l^1
      // (their swizzles L differ in bit 0, so chunk j carries the relative
      // sign (-1)^j; both halves of V[i] lie in chunks of the same parity).
      // Lower slab: a + b; upper slab: a - b.
      const float ss = (s & 1) ? -1.0f : 1.0f;
      const uint64_t ss2 = pk2(ss, ss);
#pragma unroll
      for (int i = 0; i < kHalf; ++i) {
        const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, V[i], 1);
        V[i] = ((i / C) & 1) ? sub2(mul2(V[i], ss2), other) : fma2(V[i], ss2, other);
      }
    }
    float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kHalf; ++i) {
      float a, b;
      upk2(V[i], a, b);
      am[i & 7] = fmaxf(am[i & 7], fmaxf(fabsf(a), fabsf(b)));
    }
    const float amax = fmaxf(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])),
                             fmaxf(fmaxf(am[4], am[5]), fmaxf(am[6], am[7])));
    // max_k fl(|u_k| * norm) = fl(max_k |u_k| * norm): rounding is monotonic
    if (valid) atomicMax(&row_amax[it % 3][p], __float_as_uint(amax * norm));
    __syncthreads();   // every thread has its slab: ring slot st is free again
    if (abort_flag) break;
    if (tid == 0) {
      const int64_t nt = tile + static_cast<int64_t>(nstages) * gridDim.x;
      if (nt < ntiles) {
        issue(nt, st);
        ++issued;
      }
    }
    // slots of it % 3 are read below; those of (it + 2) % 3 were last read in
    // the previous tile and are next written after the coming barrier
    if (tid < P) row_amax[(it + 2) % 3][tid] = 0u;
    if (!valid) continue;

    const float amax_r = __uint_as_float(row_amax[it % 3][p]);
    const float sc = amax_r / 7.0f;   // fp32 division, as the method states
    if (s == 0) scale[row] = sc;
    if (OUT8) {
      // one int8 code per byte: words w and w + 16 take elements 4w..4w+3 and
      // 64+4w..64+4w+3 (the low and high halves of V[4w .. 4w+4))
      uint32_t codes[kSlab / 4];
      if (sc > 0.0f) {
        const float ni = norm * (1.0f / sc);
        const uint64_t magic2 = pk2(kMagic8, kMagic8);
#pragma unroll
        for (int w = 0; w < kHalf / 4; ++w) {
          uint32_t lo_acc = 0u, hi_acc = 0u;
#pragma unroll
          for (int e = 3; e >= 0; --e) {
            const int i = 4 * w + e;
            const float m = (__popc((i / C) & L) & 1) ? -ni : ni;
            const uint64_t f = add2(mul2(V[i], pk2(m, m)), magic2);
            float f0, f1;
            upk2(f, f0, f1);
            lo_acc = lo_acc * 256u + __float_as_uint(f0);
            hi_acc = hi_acc * 256u + __float_as_uint(f1);
          }
          codes[w] = bytes_to_codes(lo_acc - kHornerBias8);
          codes[w + kHalf / 4] = bytes_to_codes(hi_acc - kHornerBias8);
        }
      } else {
#pragma unroll
        for (int w = 0; w < kSlab / 4; ++w) codes[w] = 0u;
      }
      uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K) + static_cast<int64_t>(s) * kSlab);
#pragma unroll
      for (int w = 0; w < kSlab / 16; ++w)
        dst[w] = make_uint4(codes[4 * w], codes[4 * w + 1], codes[4 * w + 2], codes[4 * w + 3]);
      continue;
    }
    uint32_t packed[kSlab / 8];
    if (sc > 0.0f) {
      const float ni = norm * (1.0f / sc);
      const uint64_t magic2 = pk2(kMagic8, kMagic8);
      // Pairs V[8w .. 8w+8) hold the codes of words w (low halves) and w + 8
      // (high halves): quantise and Horner-pack them together, so only the
      // sixteen words stay live next to the slab.
#pragma unroll
      for (int w = 0; w < kHalf / 8; ++w) {
        uint32_t lo_acc = 0u, hi_acc = 0u;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          const int i = 8 * w + e;
          // sign of output chunk i / C (both halves share it, since L < 8)
          const float m = (__popc((i / C) & L) & 1) ? -ni : ni;
          const uint64_t f = add2(mul2(V[i], pk2(m, m)), magic2);
          float f0, f1;
          upk2(f, f0, f1);
          lo_acc = lo_acc * 16u + __float_as_uint(f0);
          hi_acc = hi_acc * 16u + __float_as_uint(f1);
        }
        packed[w] = (lo_acc - kHornerBias) ^ 0x88888888u;
        packed[w + kHalf / 8] = (hi_acc - kHornerBias) ^ 0x88888888u;
      }
    } else {
#pragma unroll
      for (int w = 0; w < kSlab / 8; ++w) packed[w] = 0u;
    }
    uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K / 2) +
                                          static_cast<int64_t>(s) * (kSlab / 2));
#pragma unroll
    for (int w = 0; w < kSlab / 32; ++w)
      dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1], packed[4 * w + 2], packed[4 * w + 3]);
  }
  // After an abort, let every copy thread 0 issued land before the CTA exits.
  if (tid == 0 && abort_flag) {
    for (int st = 0; st < nstages && st < issued; ++st) {
      const int64_t n_st = issued / nstages + (st < issued % nstages ? 1 : 0);
      (void)mbar_wait(&full[st], static_cast<uint32_t>((n_st - 1) & 1), nullptr, nullptr, 100000000ull);
    }
  }
}

// Rows per tile and threads per CTA for a row of S slabs: as many whole rows
// as fit in the thread limit (at most kMaxRows).
static void rq_shape(int S, int max_threads, int* P, int* threads) {
  int p = max_threads / S;
  if (p < 1) p = 1;
  if (p > kMaxRows) p = kMaxRows;
  *P = p;
  *threads = ((p * S + 31) / 32) * 32;
}

template <typename TIn, int G, int ACT, int OUT8>
static cudaError_t launch_rq(const TIn* x, int64_t M, int K, int64_t ldx, int8_t* out, float* scale, int num_sms,
                             unsigned int* status, cudaStream_t stream) {
  const int S = K / kSlab;
  if (S > InTraits<TIn>::kMaxThreads) return cudaErrorInvalidValue;
  int P, threads;
  rq_shape(S, InTraits<TIn>::kMaxThreads, &P, &threads);
  const size_t stage_bytes = static_cast<size_t>(P) * K * sizeof(TIn);
  int nst = static_cast<int>(kRingBytes / stage_bytes);
  if (nst > kMaxStages) nst = kMaxStages;
  if (nst < 1) return cudaErrorInvalidValue;
  const size_t smem = nst * stage_bytes;
  auto kern = rotate_quant_pack_kernel<TIn, G, ACT, OUT8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = (M + P - 1) / P;
  const int64_t grid = tiles < num_sms ? tiles : num_sms;
  kern<<<static_cast<unsigned>(grid), threads, smem, stream>>>(x, M, K, ldx, P, nst, out, scale, status);
  return cudaGetLastError();
}

template <typename TIn, int OUT8>
static cudaError_t dispatch_rq(const TIn* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                               float* scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  if (act == 0) {
    if (g == 64) return launch_rq<TIn, 64, 0, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 128) return launch_rq<TIn, 128, 0, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 256) return launch_rq<TIn, 256, 0, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
  } else {
    if (g == 64) return launch_rq<TIn, 64, 1, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 128) return launch_rq<TIn, 128, 1, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 256) return launch_rq<TIn, 256, 1, OUT8>(x, M, K, ldx, out, scale, num_sms, status, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t rotate_quant_bf16(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                              float* scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<uint16_t, 0>(x, M, K, ldx, g, act, out, scale, num_sms, status, stream);
}

cudaError_t rotate_quant_bf16_i8(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                                 float* scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<uint16_t, 1>(x, M, K, ldx, g, act, out, scale, num_sms, status, stream);
}

cudaError_t rotate_quant_f32(const float* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                             int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<float, 0>(x, M, K, ldx, g, 0, out, scale, num_sms, status, stream);
}

}  // namespace w4a4
