// Tiny-M (M <= kGemvMaxM) W4A4 linear: weight streaming on the CUDA cores.
//
// With one to a few activation rows the layer reads N*K/2 weight bytes and
// does 2*M multiply-adds per weight byte: it is HBM-bound, and a tensor-core
// MMA (whose N side is at least 16 activation rows) would pad the work 16x
// and be limited by its per-instruction cost instead of the weight stream.
// The arithmetic is the same s4 x s4 -> s32 product and rank-one epilogue as
// the other GEMM kernels (page "[PR #63] int4_tensorwise: W4A4 layout
// (+ConvRot) with fused CUDA kernels", Description: integer main loop,
// scales applied once per output).
//
// Design
//   * The packed activations (M x K/2 bytes) are widened once per CTA into
//     shared memory: each packed word (8 codes) becomes two words whose bytes
//     are 16*q for codes (1,3,5,7) and (0,2,4,6) -- a signed nibble in the
//     high half of a byte is the signed byte 16*q.
//   * A warp owns RPW consecutive weight rows at a time; lane l reads 16-byte
//     chunks l, l + 32, ... of each row straight from HBM (512 contiguous
//     bytes per row per warp step, read-only path, no L1 allocation), widens
//     them the same way and accumulates with dp4a against the shared widened
//     activations, which each lane reads once per step for all RPW rows.
//     Both operands carry the same byte order, so the sums are 256 * acc
//     exactly (|256 acc| <= 12544 K < 2^31).
//   * A warp-wide integer reduction (redux.sync) gives each output; lanes
//     0 .. RPW*M-1 apply y = bf16(((float)acc * sx[m]) * sw[n] + bias[n]) with
//     separately rounded fp32 steps, or store acc for the int32 entry.
//   * Grid: warps walk row groups with a grid stride over ~2 CTAs per SM.
//     In the fused layer each warp first requests all of its weight rows into
//     L2 with bulk prefetches, before the grid-dependency wait, so the weight
//     stream overlaps the activation quantiser.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = kGemvWarps * 32;

__device__ __forceinline__ void widen_word16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  o0 = w & 0xF0F0F0F0u;
  o1 = (w << 4) & 0xF0F0F0F0u;
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// xw: widened activations, [M][K/8] pairs (o0, o1) of packed word w.
template <int M, int RPW, int OUT_S32, int U>
__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_kernel(const int8_t* __restrict__ xq, const float* __restrict__ sx, const int8_t* __restrict__ wq,
                const float* __restrict__ sw, const uint16_t* __restrict__ bias, void* __restrict__ out,
                int64_t N, int64_t K, int64_t ldo, int early_w) {
  extern __shared__ uint2 xw[];
  const int words = static_cast<int>(K / 8);   // packed 32-bit words per row
  const int chunks = words / 4;                // 16-byte chunks per row (K % 32 == 0)
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * kGemvWarps + (threadIdx.x >> 5);
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * kGemvWarps;
  const int64_t groups = (N + RPW - 1) / RPW;
  // With early_w the weights were complete before this kernel started (the
  // fused entry's quantiser lets it start only after its own grid-dependency
  // wait): every weight row this warp will read is
  // requested into L2 now (one bulk prefetch per row, spread over the lanes),
  // so the weight stream overlaps that kernel.  (Issued after the wait, the
  // prefetches overlap nothing and measured slower than the plain loads.)
  if (early_w) {
    int idx = 0;
    for (int64_t grp = warp_global; grp < groups; grp += warps_total)
      for (int r = 0; r < RPW; ++r, ++idx) {
        const int64_t n = grp * RPW + r;
        if (n < N && (idx & 31) == lane) bulk_prefetch_l2(wq + n * (K / 2), static_cast<uint32_t>(K / 2));
      }
  }
  // The packed activations may come from the previous kernel of the stream
  // (the activation quantiser of a fused layer).
  griddep_wait();
  for (int i = threadIdx.x; i < M * words; i += kGemvThreads) {
    const int m = i / words;
    const int w = i - m * words;
    const uint32_t v = reinterpret_cast<const uint32_t*>(xq + static_cast<int64_t>(m) * (K / 2))[w];
    uint2 o;
    widen_word16(v, o.x, o.y);
    xw[i] = o;
  }
  __syncthreads();

  for (int64_t grp = warp_global; grp < groups; grp += warps_total) {
    const int64_t n0 = grp * RPW;
    int32_t acc[RPW][M];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[r][m] = 0;
    const uint4* rowp[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int64_t n = n0 + r < N ? n0 + r : N - 1;   // a ragged last group re-reads the last row
      rowp[r] = reinterpret_cast<const uint4*>(wq + n * (K / 2));
    }
    // U steps of the row in flight at once (all of a K = 3072 row when U = 3)
#pragma unroll U
    for (int c = lane; c < chunks; c += 32) {
      uint4 wv[RPW];
#pragma unroll
      for (int r = 0; r < RPW; ++r) wv[r] = ldg_stream(rowp[r] + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint2 xv[M];
#pragma unroll
        for (int m = 0; m < M; ++m) xv[m] = xw[m * words + 4 * c + j];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const uint32_t w = j == 0 ? wv[r].x : (j == 1 ? wv[r].y : (j == 2 ? wv[r].z : wv[r].w));
          uint32_t w0, w1;
          widen_word16(w, w0, w1);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            acc[r][m] = __dp4a(static_cast<int>(xv[m].x), static_cast<int>(w0), acc[r][m]);
            acc[r][m] = __dp4a(static_cast<int>(xv[m].y), static_cast<int>(w1), acc[r][m]);
          }
        }
      }
    }
    // warp sums; lane r * M + m keeps output (m, n0 + r)
    int32_t mine = 0;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int32_t s = __reduce_add_sync(0xFFFFFFFFu, acc[r][m]);
        if (lane == r * M + m) mine = s;
      }
    if (lane < RPW * M) {
      const int r = lane / M;
      const int m = lane - r * M;
      const int64_t n = n0 + r;
      if (n < N) {
        const int32_t a = mine >> 8;   // exact: every term is a multiple of 256
        if (OUT_S32) {
          reinterpret_cast<int32_t*>(out)[m * ldo + n] = a;
        } else {
          float y = __fmul_rn(__fmul_rn(__int2float_rn(a), sx[m]), sw[n]);
          if (bias != nullptr) y = __fadd_rn(y, __uint_as_float(static_cast<uint32_t>(bias[n]) << 16));
          reinterpret_cast<uint16_t*>(out)[m * ldo + n] = f_to_bf16(y);
        }
      }
    }
  }
}

template <int M, int RPW, int OUT_S32, int U>
cudaError_t launch_m(const GemvArgs& a, int num_sms, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(M) * static_cast<size_t>(a.K / 8) * sizeof(uint2);
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(gemv_kernel<M, RPW, OUT_S32, U>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kGemvMaxSmem));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t groups = (a.N + RPW - 1) / RPW;
  const int64_t want = (groups + kGemvWarps - 1) / kGemvWarps;
  const int64_t cap = 2 * static_cast<int64_t>(num_sms);
  const int grid = static_cast<int>(want < cap ? want : cap);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kGemvThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_kernel<M, RPW, OUT_S32, U>, a.xq, a.sx, a.wq, a.sw, a.bias, a.out, a.N, a.K,
                         a.ldo, a.early_w);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int M, int RPW, int OUT_S32>
cudaError_t launch_u(const GemvArgs& a, int num_sms, cudaStream_t stream) {
  // loads in flight per lane: the whole row for up to three 32-lane steps
  // (K <= 3072, and multiples of three steps up to K = 6144), four steps at a
  // time otherwise (measured: 12288 x 3072 5.4 vs 6.1 us with U = 3 rather
  // than 2; 3072 x 12288 7.1 vs 9.9 us with U = 4)
  const int64_t steps = (a.K / 32 + 31) / 32;
  if (steps <= 3 || (steps % 3 == 0 && steps <= 6)) return launch_m<M, RPW, OUT_S32, 3>(a, num_sms, stream);
  return launch_m<M, RPW, OUT_S32, 4>(a, num_sms, stream);
}

template <int M, int OUT_S32>
cudaError_t launch_rpw(const GemvArgs& a, int num_sms, cudaStream_t stream) {
  // four rows per warp step when there are enough rows to keep every SM's
  // warps streaming, fewer otherwise
  const int64_t warps = 2 * static_cast<int64_t>(num_sms) * kGemvWarps;
  if (a.N >= 4 * warps) return launch_u<M, 4, OUT_S32>(a, num_sms, stream);
  if (a.N >= 2 * warps) return launch_u<M, 2, OUT_S32>(a, num_sms, stream);
  return launch_u<M, 1, OUT_S32>(a, num_sms, stream);
}

template <int OUT_S32>
cudaError_t launch_out(const GemvArgs& a, int num_sms, cudaStream_t stream) {
  switch (a.M) {
    case 1: return launch_rpw<1, OUT_S32>(a, num_sms, stream);
    case 2: return launch_rpw<2, OUT_S32>(a, num_sms, stream);
    case 3: return launch_rpw<3, OUT_S32>(a, num_sms, stream);
    case 4: return launch_rpw<4, OUT_S32>(a, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t gemv_launch(const GemvArgs& a, int num_sms, cudaStream_t stream) {
  if (a.M < 1 || a.M > kGemvMaxM || a.N < 1) return cudaErrorInvalidValue;
  if (static_cast<size_t>(a.M) * static_cast<size_t>(a.K / 8) * sizeof(uint2) > kGemvMaxSmem)
    return cudaErrorInvalidValue;
  return a.out_s32 ? launch_out<1>(a, num_sms, stream) : launch_out<0>(a, num_sms, stream);
}

}  // namespace w4a4
