// Fused ConvRot rotate + per-row int4 quantise + pack (the activation kernel
// of page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels", Description: "FHT rotation ... + rowwise int4 quantize + pack in
// one pass").  The same kernel, with fp32 input, prepares the weights offline.
//
// B200 design
//   * A CTA owns a tile of P rows.  Every row is split into S = K/128 slabs of
//     128 consecutive elements and each thread owns one slab, entirely in
//     registers: the Walsh-Hadamard butterflies of a group (g = 64 or 128) run
//     on registers with no shuffles; g = 256 spans two slabs held by adjacent
//     lanes and takes one shuffle stage.
//   * Rows reach shared memory through bulk-async (TMA) copies into a double
//     buffer, so the copy of the next tile overlaps the arithmetic of this one.
//   * A lane reads its slab in XOR-swizzled 16-byte chunks (chunk j from
//     position j ^ L, L = lane & 7), which keeps the 128-bit shared loads free
//     of bank conflicts.  Permuting the input of a Walsh-Hadamard transform by
//     an XOR of the index only flips signs of the output: H(x[. ^ a])[i] =
//     (-1)^popcount(i & a) H(x)[i].  The sign of each output chunk is folded
//     into the quantisation multiplier, and since the quantiser is odd
//     (round-half-even and the clamp are symmetric) the codes are exact.
//   * The row amax is reduced with shared-memory atomics on the float bits,
//     then each thread quantises its slab (RNE of r / s with s = amax / 7,
//     taken in fp32 exactly as r / s: a reciprocal multiply is used away from
//     rounding boundaries and an exact division near them), packs 8 nibbles per
//     32-bit word low nibble first and writes 64 bytes with 128-bit stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {

constexpr int kSlab = 128;  // elements per thread

template <typename TIn>
struct InTraits;
template <>
struct InTraits<uint16_t> {  // bf16 bits
  static constexpr int kChunkElems = 8;
  static constexpr int kMaxThreads = 384;
};
template <>
struct InTraits<float> {
  static constexpr int kChunkElems = 4;
  static constexpr int kMaxThreads = 192;
};

__device__ __forceinline__ float gelu_erf(float t) {
  return 0.5f * t * (1.0f + erff(t * 0.70710678118654752f));
}

// Load one 16-byte chunk of the slab into 8 (bf16) or 4 (fp32) floats.
__device__ __forceinline__ void load_chunk(const uint16_t* src, float* dst) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = __uint_as_float(ws[i] << 16);
    dst[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load_chunk(const float* src, float* dst) {
  const float4 w = *reinterpret_cast<const float4*>(src);
  dst[0] = w.x;
  dst[1] = w.y;
  dst[2] = w.z;
  dst[3] = w.w;
}

template <typename TIn, int G, int ACT>
__global__ void __launch_bounds__(InTraits<TIn>::kMaxThreads, 1)
    rotate_quant_pack_kernel(const TIn* __restrict__ x, int64_t M, int K, int64_t ldx, int rows_per_tile,
                             int8_t* __restrict__ out, float* __restrict__ scale,
                             unsigned int* status) {
  constexpr int C = InTraits<TIn>::kChunkElems;
  constexpr int NCH = kSlab / C;  // chunks per slab
  constexpr int GS = G < kSlab ? G : kSlab;  // group span inside one slab

  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t full_bar[2];
  __shared__ unsigned int row_amax[2][64];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int S = K / kSlab;
  const int P = rows_per_tile;
  const int64_t ntiles = (M + P - 1) / P;
  const size_t row_bytes = static_cast<size_t>(K) * sizeof(TIn);
  TIn* buf[2] = {reinterpret_cast<TIn*>(smem_raw), reinterpret_cast<TIn*>(smem_raw + P * row_bytes)};

  if (tid == 0) {
    mbar_init(&full_bar[0], 1);
    mbar_init(&full_bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < 2 * 64; i += blockDim.x) (&row_amax[0][0])[i] = 0u;
  __syncthreads();

  auto issue = [&](int64_t tile, int b) {
    const int64_t r0 = tile * P;
    const int rows = static_cast<int>(M - r0 < P ? M - r0 : P);
    mbar_arrive_expect_tx(&full_bar[b], static_cast<uint32_t>(rows * row_bytes));
    if (ldx == K) {
      bulk_load(buf[b], x + r0 * ldx, static_cast<uint32_t>(rows * row_bytes), &full_bar[b]);
    } else {
      for (int r = 0; r < rows; ++r)
        bulk_load(reinterpret_cast<uint8_t*>(buf[b]) + r * row_bytes, x + (r0 + r) * ldx,
                  static_cast<uint32_t>(row_bytes), &full_bar[b]);
    }
  };

  if (tid == 0 && blockIdx.x < ntiles) issue(blockIdx.x, 0);

  const int p = tid / S;       // row inside the tile
  const int s = tid - p * S;   // slab inside the row
  const bool active = p < P;
  const int L = lane & 7;      // chunk swizzle of this lane
  const float norm = G == 64 ? 0.125f : (G == 256 ? 0.0625f : 0.0883883476483184405f);

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int b = it & 1;
    const int64_t next = tile + gridDim.x;
    if (tid == 0 && next < ntiles) issue(next, b ^ 1);

    const int64_t row = tile * P + p;
    const bool valid = active && row < M;
    // Every thread waits (bounded) so that no copy is in flight into a buffer
    // that the CTA has stopped tracking.
    const bool ok = mbar_wait(&full_bar[b], (it >> 1) & 1, &abort_flag, status);

    float v[kSlab];
    float amax = 0.0f;
    if (valid && ok) {
      const TIn* src = buf[b] + static_cast<size_t>(p) * K + static_cast<size_t>(s) * kSlab;
#pragma unroll
      for (int j = 0; j < NCH; ++j) load_chunk(src + ((j ^ L) * C), &v[j * C]);
      if (ACT == 1) {
#pragma unroll
        for (int i = 0; i < kSlab; ++i) v[i] = gelu_erf(v[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < kSlab; ++i) v[i] = 0.0f;
    }
    // Radix-2 Walsh-Hadamard butterflies inside each group of the slab (all
    // lanes run them, so the g = 256 shuffle stage below stays convergent).
#pragma unroll
    for (int h = 1; h < GS; h <<= 1) {
#pragma unroll
      for (int i0 = 0; i0 < kSlab; i0 += 2 * h) {
#pragma unroll
        for (int i = i0; i < i0 + h; ++i) {
          const float a = v[i], c = v[i + h];
          v[i] = a + c;
          v[i + h] = a - c;
        }
      }
    }
    if (G == 256) {
      // Last stage across the two slabs of a group, held by lanes l and l^1
      // (their swizzles L differ in bit 0, so chunk j carries the relative
      // sign (-1)^j).  Lower slab: a + b; upper slab: a - b.
      const float self_sign = (s & 1) ? -1.0f : 1.0f;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
#pragma unroll
        for (int e = 0; e < C; ++e) {
          const int i = j * C + e;
          const float other = __shfl_xor_sync(0xFFFFFFFFu, v[i], 1);
          const float t = (j & 1) ? -other : other;
          v[i] = fmaf(v[i], self_sign, t);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kSlab; ++i) amax = fmaxf(amax, fabsf(v[i]));
    if (valid && ok) atomicMax(&row_amax[it & 1][p], __float_as_uint(amax * norm));
    __syncthreads();
    if (tid < 64) row_amax[(it + 1) & 1][tid] = 0u;   // next tile's slots (last read a tile ago)

    if (valid && ok) {
      const float amax_r = __uint_as_float(row_amax[it & 1][p]);
      const float sc = amax_r / 7.0f;                  // fp32 division, as the method states
      if (s == 0) scale[row] = sc;
      uint32_t packed[kSlab / 8];
      if (sc > 0.0f) {
        const float inv = 1.0f / sc;
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          // sign of output chunk j: (-1)^popcount(j & L)
          const float sgn = (__popc(j & L) & 1) ? -1.0f : 1.0f;
          const float mul = norm * inv * sgn;
#pragma unroll
          for (int e = 0; e < C; ++e) {
            const int i = j * C + e;
            float q = v[i] * mul;
            float k = rintf(q);
            // Near a rounding boundary take the decision on r / s exactly.
            if (fabsf(q - k) > 0.5f - 4e-7f * fabsf(q) - 1e-30f) {
              const float r = __fmul_rn(v[i] * sgn, norm);
              k = rintf(__fdiv_rn(r, sc));
            }
            v[i] = k;
          }
        }
#pragma unroll
        for (int w = 0; w < kSlab / 8; ++w) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) word |= (static_cast<uint32_t>(static_cast<int>(v[w * 8 + e])) & 0xFu) << (4 * e);
          packed[w] = word;
        }
      } else {
#pragma unroll
        for (int w = 0; w < kSlab / 8; ++w) packed[w] = 0u;
      }
      uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K / 2) + static_cast<int64_t>(s) * (kSlab / 2));
#pragma unroll
      for (int w = 0; w < kSlab / 32; ++w)
        dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1], packed[4 * w + 2], packed[4 * w + 3]);
    }
    __syncthreads();   // buffer b and row_amax[it & 1] are free after this
    if (abort_flag) break;
  }
  // After an abort, let any copy this CTA issued land before it exits.
  if (abort_flag && tid == 0) {
    (void)mbar_wait(&full_bar[0], 0, nullptr, nullptr, 1000000ull);
    (void)mbar_wait(&full_bar[1], 0, nullptr, nullptr, 1000000ull);
  }
}

// Host-side launch.  Returns a cudaError_t.
template <typename TIn, int G, int ACT>
static cudaError_t launch_rq(const TIn* x, int64_t M, int K, int64_t ldx, int8_t* out, float* scale,
                             int num_sms, unsigned int* status, cudaStream_t stream) {
  const int S = K / kSlab;
  const int maxT = InTraits<TIn>::kMaxThreads;
  int P = maxT / S;
  if (P < 1) return cudaErrorInvalidValue;
  if (P > 64) P = 64;
  if (G == 256 && (P * S) % 2) --P;  // never happens (S is even for g = 256)
  int threads = ((P * S + 31) / 32) * 32;
  const size_t smem = 2 * static_cast<size_t>(P) * K * sizeof(TIn);
  auto kern = rotate_quant_pack_kernel<TIn, G, ACT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (M + P - 1) / P;
  const int grid = static_cast<int>(ntiles < num_sms ? ntiles : num_sms);
  kern<<<grid, threads, smem, stream>>>(x, M, K, ldx, P, out, scale, status);
  return cudaGetLastError();
}

template <typename TIn>
static cudaError_t dispatch_rq(const TIn* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                               float* scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  if (act == 0) {
    if (g == 64) return launch_rq<TIn, 64, 0>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 128) return launch_rq<TIn, 128, 0>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 256) return launch_rq<TIn, 256, 0>(x, M, K, ldx, out, scale, num_sms, status, stream);
  } else {
    if (g == 64) return launch_rq<TIn, 64, 1>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 128) return launch_rq<TIn, 128, 1>(x, M, K, ldx, out, scale, num_sms, status, stream);
    if (g == 256) return launch_rq<TIn, 256, 1>(x, M, K, ldx, out, scale, num_sms, status, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t rotate_quant_bf16(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                              float* scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<uint16_t>(x, M, K, ldx, g, act, out, scale, num_sms, status, stream);
}

cudaError_t rotate_quant_f32(const float* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                             int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<float>(x, M, K, ldx, g, 0, out, scale, num_sms, status, stream);
}

}  // namespace w4a4
