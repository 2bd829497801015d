// Fused ConvRot rotate + per-row int4 quantise + pack (the activation kernel
// of page "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA
// kernels", Description: the rotation, the per-row quantisation and the
// packing happen in a single kernel pass over the activations).  The same
// kernel, with fp32 input, prepares the weights offline.
//
// B200 design (an HBM-bound pass that is close to ALU-bound as well: 2 bytes
// read, half a byte written, ~log2(g) adds per code)
//   * Every row is split into S = K/64 slabs of 64 consecutive elements and
//     each thread owns one slab in registers, as 32 packed fp32 pairs
//     (element i, element i + 32).  Five radix-2 Walsh-Hadamard stages run as
//     paired sm_100 add/sub.f32x2 instructions, the sixth (distance 32) pairs
//     the two halves of a register; g = 128 and g = 256 span two and four
//     slabs held by neighbouring lanes and take one and two shuffle stages.
//     At about 100 registers per thread, two or three CTAs share an SM, so the
//     latency of one CTA's barrier and loads hides behind the others' math.
//   * The kernel is persistent: a CTA walks row tiles (P whole rows) with a
//     grid stride, and one thread streams the rows of the coming tiles into a
//     shared-memory ring with bulk-async (TMA) copies, so HBM reads stay in
//     flight during the arithmetic.  P is chosen on the host so that the rows
//     spread evenly over the resident CTAs.  The one CTA barrier per tile (for
//     the row amax) also frees the ring slot that tile used.
//   * A lane reads its slab from shared memory in XOR-swizzled 16-byte chunks
//     (chunk j from position j ^ L, L = lane & 7), which keeps the 128-bit
//     shared loads free of bank conflicts.  Permuting the input of a
//     Walsh-Hadamard transform by an XOR of the index only flips signs of the
//     output: H(x[. ^ a])[i] = (-1)^popcount(i & a) H(x)[i].  The shuffle
//     stages combine lanes whose swizzles differ in one bit, which makes the
//     partner's value a known sign times the true one; the remaining sign of
//     each output chunk is folded into the quantisation multiplier, and the
//     quantiser is odd (round-half-even and the clamp are symmetric), so the
//     codes are exact.
//   * The row amax is reduced with shared-memory atomics on the float bits
//     (triple-buffered slots, one barrier per tile), and s = amax / 7 in fp32.
//     The code is round-half-even of u * (norm/s): one fused multiply-add of
//     the butterfly sum u by the reciprocal multiplier (with 1/sqrt(g) and the
//     chunk sign folded in) and a magic number rounds the exact product to an
//     integer and leaves it in the low mantissa bits, and a Horner chain of
//     integer multiply-adds packs 8 codes per word as they are made.  The
//     multiplier is within 2 ulp of 1/s, so a code can differ from the one of
//     the exact quotient r / s only for values within ~3e-7 (relative) of a
//     rounding boundary; exact ties with power-of-two scales stay exact.
//   * Codes are stored low nibble first, 32 contiguous bytes per thread, with
//     128-bit stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gelu_table.cuh"
#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {

__device__ float g_gelu_table[kGeluTableSize];

constexpr int kSlab = 64;      // elements per thread
constexpr int kHalf = 32;      // packed pairs per thread
constexpr int kMaxRows = 64;   // rows per CTA tile
constexpr int kMaxThreads = 512;
constexpr int kMaxStages = 4;
constexpr int kMinStages = 2;
constexpr size_t kRingBytesPerSm = 200 * 1024;   // shared memory for the rings of one SM

template <typename TIn>
struct InTraits;
template <>
struct InTraits<uint16_t> {  // bf16 bits
  static constexpr int kChunkElems = 8;
};
template <>
struct InTraits<float> {     // fp32 weights (offline)
  static constexpr int kChunkElems = 4;
};

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

// bf16 bits of element e of a 16-byte chunk.
__device__ __forceinline__ uint32_t bits16(const uint4 w, int e) {
  const uint32_t word = e < 2 ? w.x : (e < 4 ? w.y : (e < 6 ? w.z : w.w));
  return (e & 1) ? (word >> 16) : (word & 0xFFFFu);
}

// Element e of a 16-byte chunk as fp32.
__device__ __forceinline__ float elem(const uint4 w, int e, const uint16_t*) {
  const uint32_t word = e < 2 ? w.x : (e < 4 ? w.y : (e < 6 ? w.z : w.w));
  return (e & 1) ? __uint_as_float(word & 0xFFFF0000u) : __uint_as_float(word << 16);
}
__device__ __forceinline__ float elem(const uint4 w, int e, const float*) {
  return __uint_as_float(e == 0 ? w.x : (e == 1 ? w.y : (e == 2 ? w.z : w.w)));
}

// One radix-2 butterfly stage at distance H (< 32) over the packed pairs.
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

// Butterfly stage across lanes: the group's two halves at distance 64 * D
// (D = 1 or 2) are held by lanes l and l ^ D.  Values are kept "twisted":
// V[i] holds t(i) times the true value, with a sign t(i) that depends only on
// the lane and i.  The partner's swizzle differs in bit log2(D), so its twist
// differs from ours by rho(i) = (-1)^bit(log2 D) of the chunk index -- the
// same for both halves of V[i], which lie 4 chunks (bf16) or 8 chunks (fp32)
// apart.  With sigma = +1 in the lower half and -1 in the upper half, the
// new twisted value is sigma * own + rho * partner; this stage stores rho
// times it, fma(own, sigma * rho, partner), and the extra factor rho(i) joins
// the twist that the quantiser multiplier undoes.
template <int D, int C>
__device__ __forceinline__ void fht_cross(uint64_t (&V)[kHalf], bool upper) {
  const float sg = upper ? -1.0f : 1.0f;
  const uint64_t sr_pos = pk2(sg, sg), sr_neg = pk2(-sg, -sg);
#pragma unroll
  for (int i = 0; i < kHalf; ++i) {
    const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, V[i], D);
    V[i] = fma2(V[i], (((i / C) / D) & 1) ? sr_neg : sr_pos, other);
  }
}

// 1.5 * 2^23 + 8: adding it to |q| <= 7.5 rounds q to an integer k, half to
// even, and leaves k + 8 (in 1..15) in the low four bits of the sum.
constexpr float kMagic8 = 12582920.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;   // bits of 1.5 * 2^23
// Horner-packing eight sums (kMagicBits + n_e) as sum_e bits_e * 16^e leaves
// this constant on top of the nibbles n_e (mod 2^32).
constexpr uint32_t kHornerBias = kMagicBits * 0x11111111u;

template <typename TIn, int G, int ACT>
__global__ void __maxnreg__(96)
    rotate_quant_pack_kernel(const TIn* __restrict__ x, int64_t M, int K, int64_t ldx, int rows_per_tile,
                             int nstages, int8_t* __restrict__ out, float* __restrict__ scale,
                             unsigned int* status, unsigned long long wait_ns) {
  constexpr int C = InTraits<TIn>::kChunkElems;
  constexpr int NCH = kSlab / C;   // 16-byte chunks per slab

  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ float gelu_tab[ACT == 1 ? kGeluTableSize : 1];
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

  // Set-up that reads nothing a previous kernel may write (the GELU table is
  // filled by a synchronous host copy before any launch that uses it).
  for (int i = tid; i < 3 * kMaxRows; i += blockDim.x) (&row_amax[0][0])[i] = 0u;
  if (ACT == 1)
    for (int i = tid; i < kGeluTableSize; i += blockDim.x) gelu_tab[i] = g_gelu_table[i];
  if (tid == 0) {
    for (int i = 0; i < kMaxStages; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  // Launched with programmatic stream serialization, so the set-up above may
  // overlap the previous kernel; x is read and the outputs written only after
  // that grid has finished.  Only then may the next kernel of the stream (the
  // GEMM of a fused layer) be scheduled: it waits for this grid's writes
  // before it reads them, and whatever ran before this kernel has finished
  // before it starts (the fused layer's weight streaming relies on that).
  griddep_wait();
  griddep_launch_dependents();
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

  // sign of the two halves of V[i] in this lane's swizzle: chunks i / C and
  // i / C + NCH / 2 (bit log2(NCH / 2) of the chunk index is outside L for
  // fp32, inside it for bf16)
  const bool hi_flip = (NCH / 2 < 8) && ((L >> 2) & 1);

  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int st = it % nstages;
    const int64_t row = tile * P + p;
    const bool ok = warp_wait(&full[st], static_cast<uint32_t>((it / nstages) & 1), &abort_flag, status, wait_ns);
    const bool valid = active && row < M && ok;

    // Slot chunk j (j < NCH/2) fills the low halves of V[C*j .. C*j+C), slot
    // chunk j + NCH/2 the high halves: V[i] = (element i, element i + 32).
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
          V[j * C + e] = pk2(elem(lo, e, x), elem(hi, e, x));
          if (ACT == 1 && (e & 1)) {
            // GELU = t * Phi(t): the Phi of elements e-1, e of both chunks
            // come from one table lookup per 32-bit word
            float pa0, pa1, pb0, pb1;
            gelu_phi_word(bits16(lo, e - 1) | (bits16(lo, e) << 16), gelu_tab, pa0, pa1);
            gelu_phi_word(bits16(hi, e - 1) | (bits16(hi, e) << 16), gelu_tab, pb0, pb1);
            V[j * C + e - 1] = mul2(V[j * C + e - 1], pk2(pa0, pb0));
            V[j * C + e] = mul2(V[j * C + e], pk2(pa1, pb1));
          }
        }
      }
    }

    // Walsh-Hadamard butterflies: distances 1..16 on the pairs, 32 inside a
    // pair, then 64 and 128 across lanes.
    fht_stage2<1>(V);
    fht_stage2<2>(V);
    fht_stage2<4>(V);
    fht_stage2<8>(V);
    fht_stage2<16>(V);
#pragma unroll
    for (int i = 0; i < kHalf; ++i) {
      float a, b;
      upk2(V[i], a, b);
      V[i] = pk2(a + b, a - b);
    }
    if (G >= 128) fht_cross<1, C>(V, (s & 1) != 0);
    if (G == 256) fht_cross<2, C>(V, (s & 2) != 0);

    float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kHalf; ++i) {
      float a, b;
      upk2(V[i], a, b);
      am[i & 3] = fmaxf(am[i & 3], fmaxf(fabsf(a), fabsf(b)));
    }
    const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
    // max_k fl(|u_k| * norm) = fl(max_k |u_k| * norm): rounding is monotonic
    if (valid) atomicMax(&row_amax[it % 3][p], __float_as_uint(amax * norm));
    // Every thread has its slab: ring slot st is free again.  The barrier ORs
    // the threads' views of the abort flag (a warp of this CTA may raise it in
    // the next tile's wait while a slower one still reads it here), so all
    // leave the loop at the same tile or none does.
    if (__syncthreads_or(abort_flag != 0)) break;
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
    const float ni = sc > 0.0f ? norm * (1.0f / sc) : 0.0f;
    const uint64_t magic2 = pk2(kMagic8, kMagic8);
    // Quantiser multipliers per output chunk c of the low half: ni times the
    // twist of chunk c -- the swizzle sign (-1)^popcount(c & L) and the rho
    // factor of each shuffle stage; the high half (chunk c + NCH/2) adds the
    // swizzle bit log2(NCH/2) when that bit lies inside L (bf16).
    uint64_t mult[NCH / 2];
#pragma unroll
    for (int c = 0; c < NCH / 2; ++c) {
      int par = __popc(c & L);
      if (G >= 128) par += c & 1;
      if (G == 256) par += (c >> 1) & 1;
      const float m = (par & 1) ? -ni : ni;
      mult[c] = pk2(m, hi_flip ? -m : m);
    }
    {
      // words w and w + 4 take elements 8w..8w+7 and 32+8w..32+8w+7
      uint32_t packed[kSlab / 8];
#pragma unroll
      for (int w = 0; w < kHalf / 8; ++w) {
        uint32_t lo_acc = 0u, hi_acc = 0u;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          const int i = 8 * w + e;
          const uint64_t f = fma2(V[i], mult[i / C], magic2);
          float f0, f1;
          upk2(f, f0, f1);
          lo_acc = lo_acc * 16u + __float_as_uint(f0);
          hi_acc = hi_acc * 16u + __float_as_uint(f1);
        }
        packed[w] = (lo_acc - kHornerBias) ^ 0x88888888u;
        packed[w + kHalf / 8] = (hi_acc - kHornerBias) ^ 0x88888888u;
      }
      uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K / 2) +
                                            static_cast<int64_t>(s) * (kSlab / 2));
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
  }
  // After an abort, let every copy thread 0 issued land before the CTA exits.
  if (tid == 0 && abort_flag) {
    for (int st = 0; st < nstages && st < issued; ++st) {
      const int64_t n_st = issued / nstages + (st < issued % nstages ? 1 : 0);
      (void)mbar_wait(&full[st], static_cast<uint32_t>((n_st - 1) & 1), nullptr, nullptr, 100000000ull);
    }
  }
}

// Fills the GELU table of the current device once: every bf16 t with
// 2^-12 <= |t| < 8 gets fp32(Phi(t)) = fp32((1 + erf(t / sqrt 2)) / 2)
// evaluated in double precision, except t = -(8 - 2^-5), whose entry also
// serves every t <= -8 and holds 0.  The copy is synchronous, so the first
// GELU call on a device must not be inside a stream capture.
static cudaError_t ensure_gelu_table() {
  static bool ready[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (ready[dev]) return cudaSuccess;
  static float host[kGeluTableSize];
  for (int sgn = 0; sgn < 2; ++sgn)
    for (uint32_t ex = 0; ex < kGeluExps; ++ex)
      for (uint32_t f = 0; f < 128; ++f) {
        const uint32_t bits = (static_cast<uint32_t>(sgn) << 15) | ((kGeluFirstExp + ex) << 7) | f;
        const uint32_t fb = bits << 16;
        float tf;
        std::memcpy(&tf, &fb, sizeof(tf));
        const double t = static_cast<double>(tf);
        host[2 * (ex * 128 + f) + sgn] = static_cast<float>(0.5 * (1.0 + std::erf(t / std::sqrt(2.0))));
      }
  host[2 * (kGeluMags - 1) + 1] = 0.0f;   // the clamped negative end: GELU(t <= -8) = -0
  e = cudaMemcpyToSymbol(g_gelu_table, host, sizeof(host));
  if (e != cudaSuccess) return e;
  ready[dev] = true;
  return cudaSuccess;
}

// Registers per thread of one kernel instantiation (queried once).
template <typename TIn, int G, int ACT>
static int kernel_regs() {
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes a;
    regs = cudaFuncGetAttributes(&a, rotate_quant_pack_kernel<TIn, G, ACT>) == cudaSuccess && a.numRegs > 0
               ? a.numRegs
               : 128;
  }
  return regs;
}

struct RqPlan {
  int P = 0, threads = 0, nst = 0;
  int64_t grid = 0;
};

// Launch shape: rows per tile P, ring depth and grid.  Every row of S slabs
// takes S threads; the CTAs that fit on an SM (registers, threads, ring
// memory) run side by side, each on its own tiles.  The plan minimises the
// estimated time of the busiest SM: the rows it holds, divided by the warps
// that share them (up to 16, beyond which an SM is saturated) and by the
// fraction of lanes that carry a slab.
static RqPlan plan_rq(int64_t M, int K, size_t elem_bytes, int regs, int num_sms, size_t static_bytes) {
  const int S = K / kSlab;
  const size_t row_bytes = static_cast<size_t>(K) * elem_bytes;
  const int regs_warp = (regs * 32 + 255) / 256 * 256;
  RqPlan best;
  double best_t = 1e30;
  const int pmax = kMaxThreads / S < kMaxRows ? kMaxThreads / S : kMaxRows;
  for (int P = 1; P <= pmax; ++P) {
    const int threads = (P * S + 31) / 32 * 32;
    const int warps = threads / 32;
    int cps = 65536 / (warps * regs_warp);
    if (2048 / threads < cps) cps = 2048 / threads;
    if (cps > 8) cps = 8;
    const int64_t tiles = (M + P - 1) / P;
    for (int c = 1; c <= cps; ++c) {
      const size_t ring_budget = kRingBytesPerSm > c * static_bytes ? kRingBytesPerSm - c * static_bytes : 0;
      int nst = static_cast<int>(ring_budget / (static_cast<size_t>(c) * P * row_bytes));
      if (nst > kMaxStages) nst = kMaxStages;
      if (nst < kMinStages) break;
      const int64_t grid = tiles < static_cast<int64_t>(num_sms) * c ? tiles : static_cast<int64_t>(num_sms) * c;
      const int64_t per_cta = (tiles + grid - 1) / grid;
      const int64_t ctas_sm = (grid + num_sms - 1) / num_sms;
      const double sm_rows = static_cast<double>(per_cta * P * ctas_sm);
      const double w = static_cast<double>(warps * ctas_sm) < 16.0 ? static_cast<double>(warps * ctas_sm) : 16.0;
      const double eff = static_cast<double>(P * S) / threads;
      const double t = sm_rows / (w * eff) * (1.0 + 0.02 * (kMaxStages - nst));
      if (t < best_t - 1e-9) {
        best_t = t;
        best.P = P;
        best.threads = threads;
        best.nst = nst;
        best.grid = grid;
      }
    }
  }
  return best;
}

template <typename TIn, int G, int ACT>
static cudaError_t launch_rq(const TIn* x, int64_t M, int K, int64_t ldx, int8_t* out, float* scale, int num_sms,
                             unsigned int* status, cudaStream_t stream) {
  const int S = K / kSlab;
  if (S < 1 || S > kMaxThreads) return cudaErrorInvalidValue;
  const RqPlan pl = plan_rq(M, K, sizeof(TIn), kernel_regs<TIn, G, ACT>(), num_sms,
                            ACT == 1 ? kGeluTableSize * sizeof(float) : 0);
  if (pl.P < 1) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(pl.nst) * pl.P * K * sizeof(TIn);
  auto kern = rotate_quant_pack_kernel<TIn, G, ACT>;
  // the dynamic shared-memory limit is raised only when a launch needs more
  // than this device has been given so far (the attribute call costs host time)
  static size_t granted[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > granted[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    granted[dev] = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(pl.threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, x, M, K, ldx, pl.P, pl.nst, out, scale, status, wait_limit_ns());
  if (e != cudaSuccess) return e;
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

// The tensor-core rotation (quant_tc.cu) takes bf16 rows without activation
// for g in {64, 128} and K / g <= 128, from rotate_tc_min_rows() rows up.
// Measured on B200 (CUDA-graph replay): alone it is faster from a few
// hundred rows up (4608 x 3072: 9.7 vs 11.1 us; 32760 x 5120: 64 vs 91 us),
// but inside the fused layer, ahead of the GEMM, only the 32760-row shapes
// gain (0.7%) while 4608-row layers lose 1-2 us, so by default it serves
// batches of 8192 rows and more.  W4A4_ROTATE_TC_MIN_ROWS=<n> moves the
// threshold and W4A4_ROTATE_TC=0 selects the register-butterfly kernel
// always (both read once per process); w4a4_quantize_activation_path picks a
// kernel per call.
static int64_t rotate_tc_min_rows() {
  static int64_t v = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    v = 8192;
    const char* off = std::getenv("W4A4_ROTATE_TC");
    if (off != nullptr && off[0] == '0' && off[1] == '\0') {
      v = INT64_MAX;
      return;
    }
    const char* e = std::getenv("W4A4_ROTATE_TC_MIN_ROWS");
    if (e != nullptr) {
      const long long x = std::strtoll(e, nullptr, 10);
      if (x >= 1) v = x;
    }
  });
  return v;
}

static bool tc_applies(int K, int g, int act) { return act == 0 && (g == 64 || g == 128) && K / g <= 128; }

int rotate_quant_bf16_route(int64_t M, int K, int g, int act) {
  return tc_applies(K, g, act) && M >= rotate_tc_min_rows() ? 2 : 1;
}

cudaError_t rotate_quant_bf16(const uint16_t* x, int64_t M, int K, int64_t ldx, int g, int act, int8_t* out,
                              float* scale, int num_sms, unsigned int* status, cudaStream_t stream, int path) {
  if (path == 0) path = rotate_quant_bf16_route(M, K, g, act);
  if (path == 2) {
    if (!tc_applies(K, g, act)) return cudaErrorNotSupported;
    return rotate_quant_bf16_tc(x, M, K, ldx, g, out, scale, num_sms, status, stream);
  }
  if (act == 1) {
    const cudaError_t e = ensure_gelu_table();
    if (e != cudaSuccess) return e;
  }
  return dispatch_rq<uint16_t>(x, M, K, ldx, g, act, out, scale, num_sms, status, stream);
}

cudaError_t rotate_quant_f32(const float* x, int64_t M, int K, int64_t ldx, int g, int8_t* out, float* scale,
                             int num_sms, unsigned int* status, cudaStream_t stream) {
  return dispatch_rq<float>(x, M, K, ldx, g, 0, out, scale, num_sms, status, stream);
}

// ---- Second pass of a requantising GEMM epilogue: GELU, rotation and
// quantisation of a layer's bf16 output with the row amax already known
// (the GEMM's epilogue reported it), so no row reduction and no barrier.
// Thread = one 64-element slab; a warp takes 32 consecutive slabs of the
// row-major [M, K] slab grid, so a rotation group (g / 64 slabs) sits in
// lanes l, l ^ 1 (and l ^ 2) of one warp.  Each warp streams its slabs
// through a two-stage ring of its own in shared memory with 16-byte
// cp.async copies (the next block of 32 slabs is in flight while the warp
// computes the current one; a lane's slab sits at lane * 128 bytes with
// 16-byte chunk j at j ^ (lane & 7), so the copies and the reads are free of
// bank conflicts).  The arithmetic is the register quantiser's: the GELU
// table, f32x2 butterflies, one shuffle stage per 64 elements beyond 64,
// codes by one fused multiply-add with the magic number and a Horner chain.
constexpr int kRqThreads = 128;
constexpr int kRqCtasPerSm = 4;
constexpr int kRqStages = 2;
constexpr int kRqStageBytes = 32 * kSlab * 2;   // 4 KB: one warp's 32 slabs
constexpr int kRqSmem = kGeluTableSize * 4 + (kRqThreads / 32) * kRqStages * kRqStageBytes;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Row and slab of slab index i over S slabs per row; 32-bit division where
// the slab count fits (I32).
template <bool I32>
__device__ __forceinline__ int64_t rq_row(int64_t i, int S) {
  if (I32) return static_cast<int64_t>(static_cast<uint32_t>(i) / static_cast<uint32_t>(S));
  return i / S;
}

template <int G, bool I32>
__global__ void __launch_bounds__(kRqThreads, kRqCtasPerSm)
    requant_kernel(const uint16_t* __restrict__ y, int64_t M, int K, int64_t ldy,
                   const unsigned int* __restrict__ amax_bits, int8_t* __restrict__ out, float* __restrict__ scale) {
  extern __shared__ __align__(128) uint8_t rq_smem[];
  float* gelu_tab = reinterpret_cast<float*>(rq_smem);
  for (int i = threadIdx.x; i < kGeluTableSize; i += blockDim.x) gelu_tab[i] = g_gelu_table[i];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const uint32_t ring = smem_u32(rq_smem + kGeluTableSize * 4 + wib * kRqStages * kRqStageBytes) + lane * (kSlab * 2);
  const int L = lane & 7;
  const int S = K / kSlab;
  const int64_t total = M * S;
  const float norm = G == 64 ? 0.125f : (G == 256 ? 0.0625f : 0.0883883476483184405f);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kRqThreads / 32);
  const uint64_t magic2 = pk2(kMagic8, kMagic8);
  // y and the row amax come from the GEMM launched before this kernel
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();

  // copies of the slab block at `b` into ring stage `st` (lanes past the end
  // copy nothing; their stage contents are never used)
  auto fetch = [&](int64_t b, int st) {
    const int64_t sl = b + lane;
    if (sl < total) {
      const int64_t r = rq_row<I32>(sl, S);
      const uint16_t* src = y + r * ldy + (sl - r * S) * kSlab;
#pragma unroll
      for (int j = 0; j < 8; ++j) cp_async16(ring + st * kRqStageBytes + ((j ^ L) << 4), src + 8 * j);
    }
    cp_async_commit();
  };
  int64_t base = (static_cast<int64_t>(blockIdx.x) * (kRqThreads / 32) + wib) * 32;
#pragma unroll
  for (int k = 0; k < kRqStages - 1; ++k) fetch(base + k * warps * 32, k);   // empty groups past the end
  for (int it = 0; base < total; base += warps * 32, ++it) {
    const int st = it % kRqStages;
    fetch(base + (kRqStages - 1) * warps * 32, (it + kRqStages - 1) % kRqStages);
    cp_async_wait<kRqStages - 1>();      // this stage's copies have landed
    __syncwarp();
    const int64_t slab = base + lane;
    const bool valid = slab < total;   // whole rotation groups are valid or not (S % (G / 64) == 0)
    const int64_t row = valid ? rq_row<I32>(slab, S) : 0;
    const int s = valid ? static_cast<int>(slab - row * S) : 0;
    uint64_t V[kHalf];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // V[i] = (element i, element i + 32): chunk j gives the low halves of
      // V[8j .. 8j+7], chunk j + 4 the high halves
      const uint4 lo = lds128(ring + st * kRqStageBytes + ((j ^ L) << 4));
      const uint4 hi = lds128(ring + st * kRqStageBytes + (((j + 4) ^ L) << 4));
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        V[8 * j + e] = pk2(elem(lo, e, y), elem(hi, e, y));
        if (e & 1) {
          float pa0, pa1, pb0, pb1;
          gelu_phi_word(bits16(lo, e - 1) | (bits16(lo, e) << 16), gelu_tab, pa0, pa1);
          gelu_phi_word(bits16(hi, e - 1) | (bits16(hi, e) << 16), gelu_tab, pb0, pb1);
          V[8 * j + e - 1] = mul2(V[8 * j + e - 1], pk2(pa0, pb0));
          V[8 * j + e] = mul2(V[8 * j + e], pk2(pa1, pb1));
        }
      }
    }
    // every lane has read this stage: the next fetch may overwrite it
    __syncwarp();
    fht_stage2<1>(V);
    fht_stage2<2>(V);
    fht_stage2<4>(V);
    fht_stage2<8>(V);
    fht_stage2<16>(V);
#pragma unroll
    for (int i = 0; i < kHalf; ++i) {
      float a, b;
      upk2(V[i], a, b);
      V[i] = pk2(a + b, a - b);
    }
    // across slabs: the lower slab of a pair keeps a + b, the upper one a - b
    if (G >= 128) {
      const float sg = (s & 1) ? -1.0f : 1.0f;
      const uint64_t sg2 = pk2(sg, sg);
#pragma unroll
      for (int i = 0; i < kHalf; ++i) V[i] = fma2(V[i], sg2, __shfl_xor_sync(0xFFFFFFFFu, V[i], 1));
    }
    if (G == 256) {
      const float sg = (s & 2) ? -1.0f : 1.0f;
      const uint64_t sg2 = pk2(sg, sg);
#pragma unroll
      for (int i = 0; i < kHalf; ++i) V[i] = fma2(V[i], sg2, __shfl_xor_sync(0xFFFFFFFFu, V[i], 2));
    }
    if (!valid) continue;
    const float amax_r = __uint_as_float(amax_bits[row]);
    const float sc = amax_r / 7.0f;   // fp32 division, as the method states
    if (s == 0) scale[row] = sc;
    const float ni = sc > 0.0f ? norm * (1.0f / sc) : 0.0f;
    const uint64_t mult = pk2(ni, ni);
    uint32_t packed[kSlab / 8];
#pragma unroll
    for (int w = 0; w < kHalf / 8; ++w) {
      uint32_t lo_acc = 0u, hi_acc = 0u;
#pragma unroll
      for (int e = 7; e >= 0; --e) {
        const uint64_t f = fma2(V[8 * w + e], mult, magic2);
        float f0, f1;
        upk2(f, f0, f1);
        lo_acc = lo_acc * 16u + __float_as_uint(f0);
        hi_acc = hi_acc * 16u + __float_as_uint(f1);
      }
      packed[w] = (lo_acc - kHornerBias) ^ 0x88888888u;
      packed[w + kHalf / 8] = (hi_acc - kHornerBias) ^ 0x88888888u;
    }
    uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K / 2) + static_cast<int64_t>(s) * (kSlab / 2));
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
  cp_async_wait<0>();   // no copy outlives the CTA
}

cudaError_t gelu_table_device(const float** table) {
  const cudaError_t e = ensure_gelu_table();
  if (e != cudaSuccess) return e;
  void* p = nullptr;
  const cudaError_t e2 = cudaGetSymbolAddress(&p, g_gelu_table);
  if (e2 != cudaSuccess) return e2;
  *table = static_cast<const float*>(p);
  return cudaSuccess;
}

cudaError_t requant_bf16(const uint16_t* y, int64_t M, int K, int64_t ldy, int g, const unsigned int* amax,
                         int8_t* out, float* scale, int num_sms, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const cudaError_t e = ensure_gelu_table();
  if (e != cudaSuccess) return e;
  const int64_t warps_needed = (M * (K / kSlab) + 31) / 32;
  int64_t ctas = static_cast<int64_t>(num_sms) * kRqCtasPerSm;
  const int64_t need = (warps_needed + kRqThreads / 32 - 1) / (kRqThreads / 32);
  if (ctas > need) ctas = need;
  static bool attr_set[64][6] = {};
  int dev = 0;
  cudaError_t ea = cudaGetDevice(&dev);
  if (ea != cudaSuccess) return ea;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const bool i32 = M * (K / kSlab) + static_cast<int64_t>(ctas) * kRqThreads * 2 < (int64_t(1) << 31);
  using Fn = void (*)(const uint16_t*, int64_t, int, int64_t, const unsigned int*, int8_t*, float*);
  Fn fn = nullptr;
  if (g == 64) fn = i32 ? requant_kernel<64, true> : requant_kernel<64, false>;
  else if (g == 128) fn = i32 ? requant_kernel<128, true> : requant_kernel<128, false>;
  else if (g == 256) fn = i32 ? requant_kernel<256, true> : requant_kernel<256, false>;
  else return cudaErrorInvalidValue;
  const int gi = (g == 64 ? 0 : (g == 128 ? 1 : 2)) * 2 + (i32 ? 1 : 0);
  if (!attr_set[dev][gi]) {
    ea = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kRqSmem);
    if (ea != cudaSuccess) return ea;
    attr_set[dev][gi] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg.blockDim = dim3(kRqThreads, 1, 1);
  cfg.dynamicSmemBytes = kRqSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t r = cudaLaunchKernelEx(&cfg, fn, y, M, K, ldy, amax, out, scale);
  if (r != cudaSuccess) return r;
  return cudaGetLastError();
}

}  // namespace w4a4
