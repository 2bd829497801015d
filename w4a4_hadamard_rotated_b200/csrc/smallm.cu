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
//     two CTAs run on every SM.  One thread issues the TMA loads of all the
//     CTA's k-blocks at once (an 8-deep ring), so every SM keeps tens of KB of
//     weight reads in flight from the first cycle.
//   * Widening the weights in shared memory would cost six bytes of
//     shared-memory traffic per streamed byte, more than an SM sustains at
//     HBM rate; so four warps widen each packed weight row (one thread per
//     row, read from a 64-byte-swizzled tile) into tensor memory with
//     tcgen05.st, and the MMA reads its A operand from there.  The few
//     activation rows are widened into shared memory (the B operand).  Each
//     nibble q becomes the byte 16*q (no sign extension) in the byte order
//     (1,3,5,7, 0,2,4,6) for both operands, so the MMA accumulates 256*acc.
//   * The K slices of one weight tile run as one cluster of up to 8 CTAs.
//     Each CTA parks its int32 partial tile in its shared memory; after a
//     cluster barrier it pushes the rows every other CTA owns into that
//     CTA's shared memory with one bulk copy per owner (distributed shared
//     memory, completing on the owner's barrier).  CTA c sums its share of
//     the rows (integer addition: exact in any order), applies the epilogue
//     and writes y.  The reduction never leaves the chip, and the kernel
//     needs no workspace.
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
constexpr int SP = 8;          // packed ring depth (loads in flight per CTA), at most
constexpr int ST = 6;          // widened stages (weights in tensor memory, activations in shared memory), at most
constexpr int kWorkWarps = 4;  // widen + epilogue warps, one per tensor-memory lane quarter
constexpr int kGroups = 2;     // widen groups of kWorkWarps warps, taking turns by k-block
constexpr int kThreads = (2 + kGroups * kWorkWarps) * 32;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemA = 64;   // first widened-weight column (the accumulator takes NP <= 64)
constexpr int kMaxSplits = 8;     // K slices per weight tile at most (the portable cluster size)

// Two CTAs share an SM, so each keeps its rings within ~110 KB of shared
// memory: NP = 64 (8 KB widened activations per stage) takes shallower rings.
template <int NP>
struct Layout {
  static constexpr int kSP = NP == 64 ? 6 : SP;
  static constexpr int kST = NP == 64 ? 4 : ST;
  static constexpr uint32_t kPackW = WM * BKP;    // 8 KB
  static constexpr uint32_t kPackX = NP * BKP;    // <= 4 KB
  static constexpr uint32_t kWideX = NP * BK;     // <= 8 KB
  static constexpr uint32_t kOffWideX = 0;        // 1024-aligned stages (128-byte swizzle)
  static constexpr uint32_t kOffPackW = kOffWideX + kST * kWideX;   // 1024-aligned (64-byte swizzle)
  static constexpr uint32_t kOffPackX = kOffPackW + kSP * kPackW;
  static constexpr uint32_t kBytes = kOffPackX + kSP * kPackX;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kOffPackW % 1024 == 0, "alignment");
  // After the main loop: the parked partial tile (WM rows x NP int32) and the
  // receive slots of the split-K reduction (at most WM + kMaxSplits rows), both
  // in the idle ring memory.
  static constexpr int kChunkMask = (NP / 4 < 8 ? NP / 4 : 8) - 1;
  static constexpr uint32_t kOffPark = 0;
  static constexpr uint32_t kOffRecv = kOffPark + WM * NP * 4;
  static_assert(kOffRecv + (WM + kMaxSplits) * NP * 4 <= kBytes, "reduction buffers fit in the rings");
};

struct Bars {
  float sx[64];          // activation scales (epilogue operands, staged early)
  float sw[WM];          // this tile's weight scales
  float bias[WM];        // this tile's bias (fp32)
  uint64_t full[SP];     // TMA transaction barrier (weights + activations of one k-block)
  uint64_t empty[SP];    // kWorkWarps arrivals (packed data read)
  uint64_t wfull[ST];    // kWorkWarps arrivals (widened stage written)
  uint64_t wempty[ST];   // one MMA commit
  uint64_t acc_full;
  uint64_t recv_full;    // the other K slices' rows of this CTA's share (split-K reduction)
  uint32_t tmem_base;
  int abort_flag;
  unsigned int last;
};

// Each nibble q of a packed word to the byte 16*q: codes 1,3,5,7 and 0,2,4,6
// (a signed nibble in the high half of a byte IS the signed byte 16*q).
__device__ __forceinline__ void widen_word16(uint32_t w, uint32_t& o0, uint32_t& o1) {
  o0 = w & 0xF0F0F0F0u;
  o1 = (w << 4) & 0xF0F0F0F0u;
}

// D[tmem] (+)= A[tmem] * B[smem]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
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

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from this CTA's shared memory at `src` to CTA `rank` of this cluster at the
// shared::cta offset `dst`; the transfer completes on the barrier at offset
// `bar` in CTA `rank`.
__device__ __forceinline__ void bulk_push(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 rd, rb;\n\t"
      "mapa.shared::cluster.u32 rd, %0, %4;\n\t"
      "mapa.shared::cluster.u32 rb, %3, %4;\n\t"
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [rd], [%1], %2, [rb];\n\t}" ::"r"(dst),
      "r"(src), "r"(bytes), "r"(bar), "r"(rank)
      : "memory");
}

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

template <int NP, int OUT_S32>
__global__ void __launch_bounds__(kThreads, 2)
    smallm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, SmallMArgs args,
                  int kb_per_split, int splits) {
  using Lay = Layout<NP>;
  extern __shared__ uint8_t smem_dyn[];
  __shared__ Bars bars;
  uint8_t* smem = align1024_shared(smem_dyn);

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
    for (int s = 0; s < Lay::kSP; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], kWorkWarps);
    }
    for (int s = 0; s < Lay::kST; ++s) {
      mbar_init(&bars.wfull[s], kWorkWarps);
      mbar_init(&bars.wempty[s], 1);
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.recv_full, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();   // the barriers are visible to the copy engine
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    if (args.early_w) {
      // The packed weights were complete before this kernel started (the
      // caller guarantees it), so their first ring stages stream in from the
      // first cycle, before tensor memory is allocated and while the
      // previous kernel (the activation quantiser) is still running.
      const int pre = min(Lay::kSP, nkb);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&bars.full[i], Lay::kPackW + Lay::kPackX);
        tma_load_2d(smem + Lay::kOffPackW + i * Lay::kPackW, &tmW, &bars.full[i], (kb0 + i) * BKP, ntile * WM);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // A kernel launched after this one with programmatic stream serialization
  // may start its own set-up now; it reads nothing this kernel writes before
  // its grid-dependency wait, which returns only once this grid has finished.
  griddep_launch_dependents();
  // launched with programmatic stream serialization: the set-up above may
  // overlap the previous kernel (the activation quantiser of a fused layer);
  // its outputs are read only after this point
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t ps = 0, ph = 0;
      int issued = 0;
      bool ok = true;
      const int pre = args.early_w ? min(Lay::kSP, nkb) : 0;   // weight stages already in flight
      for (int kb = kb0; kb < kb1; ++kb) {
        if (kb - kb0 >= pre) {
          if (!mbar_wait(&bars.empty[ps], ph ^ 1, abort_flag, args.status, args.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.full[ps], Lay::kPackW + Lay::kPackX);
          tma_load_2d(smem + Lay::kOffPackW + ps * Lay::kPackW, &tmW, &bars.full[ps], kb * BKP, ntile * WM);
        }
        tma_load_2d(smem + Lay::kOffPackX + ps * Lay::kPackX, &tmX, &bars.full[ps], kb * BKP, 0);
        ++issued;
        if (++ps == Lay::kSP) { ps = 0; ph ^= 1; }
      }
      {
        // every copy this thread issued lands before the CTA can exit (after an
        // abort some are never consumed; in a normal run these phases have all
        // completed already)
        for (int s = 0; s < Lay::kSP && s < issued; ++s) {
          const int n_s = issued / Lay::kSP + (s < issued % Lay::kSP ? 1 : 0);
          (void)mbar_wait(&bars.full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(WM, NP);
      uint32_t ws = 0, wph = 0;
      for (int i = 0; i < nkb; ++i) {
        if (!mbar_wait(&bars.wfull[ws], wph, abort_flag, args.status, args.wait_ns)) break;
        tc_fence_after();
        const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + Lay::kOffWideX + ws * Lay::kWideX));
        const uint32_t a_tmem = tmem_base + kTmemA + ws * 32;
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          mma_i8_ts(tmem_base, a_tmem + kk * 8, bd + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        mma_commit(&bars.wempty[ws]);
        if (++ws == Lay::kST) { ws = 0; wph ^= 1; }
      }
      mma_commit(&bars.acc_full);   // also the drain point on an abort
    }
  } else {
    // ------------------------------------------------------------ widen warps
    // Weights: thread r (= tensor-memory lane) widens weight row r of the
    // tile, read from the 64-byte-swizzled tile (chunk j of row r at
    // j ^ ((r >> 1) & 3)), into 32 columns of tensor memory.  Activations:
    // unit u (16 packed bytes) is part u % 4 of row u / 4; its 32 widened
    // bytes go to chunks 2 * part and 2 * part + 1 of that row in the
    // 128-byte-swizzle K-major layout of the B operand.
    if (!OUT_S32) {
      // epilogue operands; read only after the cluster barrier that precedes
      // the reduction, so their latency hides behind the weight stream
      const int t = threadIdx.x - 64;
      if (t < WM) {
        const int64_t n = static_cast<int64_t>(ntile) * WM + t;
        bars.sw[t] = n < N ? args.sw[n] : 0.0f;
        bars.bias[t] = (n < N && args.bias != nullptr) ? bf16_to_f(args.bias[n]) : 0.0f;
      } else if (t < WM + 64) {
        bars.sx[t - WM] = t - WM < M ? args.sx[t - WM] : 0.0f;
      }
    }
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int grp = (warp - 2) / kWorkWarps;
    const int wt = threadIdx.x - 64 - grp * kWorkWarps * 32;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kTmemA;
    uint32_t ps = 0, ph = 0, ws = 0, wph = 0;
    bool ok = true;
    for (int i = 0; i < nkb; ++i, ps = (ps + 1 == Lay::kSP ? 0 : ps + 1), ph ^= (ps == 0 ? 1u : 0u),
             ws = (ws + 1 == Lay::kST ? 0 : ws + 1), wph ^= (ws == 0 ? 1u : 0u)) {
      if (i % kGroups != grp) continue;
      if (!warp_wait(&bars.full[ps], ph, abort_flag, args.status, args.wait_ns) ||
          !warp_wait(&bars.wempty[ws], wph ^ 1, abort_flag, args.status, args.wait_ns)) { ok = false; break; }
      {
        const uint8_t* src = smem + Lay::kOffPackW + ps * Lay::kPackW + r * BKP;
        const int swz = (r >> 1) & 3;
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 u = *reinterpret_cast<const uint4*>(src + ((j ^ swz) << 4));
          widen_word16(u.x, v[8 * j + 0], v[8 * j + 1]);
          widen_word16(u.y, v[8 * j + 2], v[8 * j + 3]);
          widen_word16(u.z, v[8 * j + 4], v[8 * j + 5]);
          widen_word16(u.w, v[8 * j + 6], v[8 * j + 7]);
        }
        tmem_st_32x32b_x32(t_lane + ws * 32, v);
      }
      {
        constexpr int kUnits = NP * BKP / 16;
        const uint8_t* src = smem + Lay::kOffPackX + ps * Lay::kPackX;
        uint8_t* dst = smem + Lay::kOffWideX + ws * Lay::kWideX;
#pragma unroll
        for (int u = wt; u < kUnits; u += kWorkWarps * 32) {
          const uint4 w = *reinterpret_cast<const uint4*>(src + u * 16);
          const int rr = u >> 2, part = u & 3;
          uint4 c0, c1;
          widen_word16(w.x, c0.x, c0.y);
          widen_word16(w.y, c0.z, c0.w);
          widen_word16(w.z, c1.x, c1.y);
          widen_word16(w.w, c1.z, c1.w);
          uint8_t* rowp = dst + (rr >> 3) * 1024 + (rr & 7) * 128;
          *reinterpret_cast<uint4*>(rowp + (((2 * part) ^ (rr & 7)) << 4)) = c0;
          *reinterpret_cast<uint4*>(rowp + (((2 * part + 1) ^ (rr & 7)) << 4)) = c1;
        }
      }
      tmem_wait_st();
      fence_async_shared();   // generic-proxy writes, read by the tensor cores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.wfull[ws]);
        mbar_arrive(&bars.empty[ps]);
      }
    }
    // The first group parks this CTA's partial tile in shared memory (the
    // rings are idle once the accumulator is complete): row r of the tile is
    // NP consecutive int32 values, its 16-byte chunk j stored at chunk
    // j ^ (r & kChunkMask), so the rows that go to one owner are contiguous.
    if (grp == 0) {
      if (ok) (void)warp_wait(&bars.acc_full, 0, abort_flag, args.status, args.wait_ns);
      if (*abort_flag == 0) {
        tc_fence_after();
        uint32_t acc[NP];
        tmem_ld_cols<NP>(tmem_base + (static_cast<uint32_t>(q * 32) << 16), acc);
        tmem_wait_ld();
        uint8_t* row = smem + Lay::kOffPark + r * (NP * 4);
#pragma unroll
        for (int j = 0; j < NP / 4; ++j) {
          const int4 c = make_int4(static_cast<int32_t>(acc[4 * j]) >> 8, static_cast<int32_t>(acc[4 * j + 1]) >> 8,
                                   static_cast<int32_t>(acc[4 * j + 2]) >> 8, static_cast<int32_t>(acc[4 * j + 3]) >> 8);
          *reinterpret_cast<int4*>(row + ((j ^ (r & Lay::kChunkMask)) << 4)) = c;
        }
        fence_async_shared();   // read next by bulk copies
      }
    }
  }

  // ---- K-slice reduction across the cluster (one cluster per weight tile,
  // one CTA per K slice).  CTA c owns rows [c*R, c*R + R) of the tile.  After
  // a cluster barrier (every CTA's rings are idle and its partial tile is
  // parked) each CTA pushes the rows every other CTA owns into that CTA's
  // receive slot for this rank with one bulk copy, which completes on the
  // owner's barrier; the owner sums its own rows and the received ones
  // (integer addition: exact in any order), applies the epilogue and writes
  // those outputs.  Nothing is read remotely, so no second barrier is needed:
  // an owner leaves only once every byte sent to it has landed, and a sender
  // only once its copies have read its shared memory.  That holds after an
  // abort too: the expected byte count is armed before the barrier and every
  // CTA pushes unconditionally after it, so the receive wait ignores the
  // abort flag (and the debug wait limit) and always waits for the bytes.
  const int R = (WM + splits - 1) / splits;
  const int own_rows = min(WM - split * R, R);
  const uint32_t slot_bytes = static_cast<uint32_t>(R) * NP * 4;
  if (threadIdx.x == 0 && splits > 1)
    mbar_arrive_expect_tx(&bars.recv_full, static_cast<uint32_t>(splits - 1) * own_rows * NP * 4);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // every CTA of the cluster is done with its rings and has parked its partial tile
  if (threadIdx.x == 0 && splits > 1) {
    for (int c = 0; c < splits; ++c) {
      if (c == split) continue;
      const int rows_c = min(WM - c * R, R);
      bulk_push(smem_u32(smem + Lay::kOffRecv) + split * slot_bytes,
                smem_u32(smem + Lay::kOffPark) + static_cast<uint32_t>(c) * slot_bytes,
                static_cast<uint32_t>(rows_c) * NP * 4, smem_u32(&bars.recv_full), static_cast<uint32_t>(c));
    }
    bulk_commit_group();
  }
  bool got = true;
  if (splits > 1) got = warp_wait(&bars.recv_full, 0, nullptr, args.status);
  if (got && *abort_flag == 0) {
    // item = (owned row, chunk of four activation rows); consecutive threads
    // take consecutive rows, so the stores of one activation row coalesce
    const int chunks = (static_cast<int>(M) + 3) / 4;
    for (int it = threadIdx.x; it < own_rows * chunks; it += kThreads) {
      const int j = it / own_rows;
      const int rl = it - j * own_rows;
      const int rr = split * R + rl;   // row in the tile
      const uint32_t coff = static_cast<uint32_t>(((j ^ (rr & Lay::kChunkMask)) << 4));
      int4 sum = *reinterpret_cast<const int4*>(smem + Lay::kOffPark + rr * (NP * 4) + coff);
      for (int c = 0; c < splits; ++c) {
        if (c == split) continue;
        const int4 v = *reinterpret_cast<const int4*>(smem + Lay::kOffRecv + c * slot_bytes + rl * (NP * 4) + coff);
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      const int64_t n = static_cast<int64_t>(ntile) * WM + rr;   // weight row = output column
      if (n >= N) continue;
      const int32_t s4[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t m = 4 * j + e;
        if (m >= M) break;
        if (OUT_S32) {
          reinterpret_cast<int32_t*>(args.out)[m * args.ldo + n] = s4[e];
        } else {
          float y = __fmul_rn(__fmul_rn(__int2float_rn(s4[e]), bars.sx[m]), bars.sw[rr]);
          if (args.bias != nullptr) y = __fadd_rn(y, bars.bias[rr]);
          reinterpret_cast<uint16_t*>(args.out)[m * args.ldo + n] = f_to_bf16(y);
        }
      }
    }
  }
  if (threadIdx.x == 0 && splits > 1) bulk_wait_group_read<0>();   // the pushes have read the parked tile
  if (warp == 1) {
    // the MMA thread's final commit arrives when every MMA has completed
    if (lane == 0) (void)mbar_wait(&bars.acc_full, 0, nullptr, nullptr, 100000000ull);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int NP, int OUT_S32>
void fill_cfg(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, int ctas, int splits, cudaStream_t stream) {
  *cfg = cudaLaunchConfig_t{};
  cfg->gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  cfg->blockDim = dim3(kThreads, 1, 1);
  cfg->dynamicSmemBytes = Layout<NP>::kAlloc;
  cfg->stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

// Split plan: K slices per 128-row weight tile.  Two CTAs fit on an SM
// (registers, shared memory and tensor memory each allow two), and clusters
// pack into the GPCs with some loss, so the plan keeps the grid within 85% of
// 2 CTAs per SM (2 x 148 on a B200) -- every cluster is then resident at once (a second wave of a
// few clusters would double the kernel's time) -- with at most kMaxSplits
// slices and at least one k-block per slice.
void smallm_plan(int64_t N, int64_t K, int num_sms, int* ntiles, int* kb_per, int* splits) {
  const int kMaxCtas = static_cast<int>(0.85 * 2 * num_sms);
  const int nt = static_cast<int>((N + WM - 1) / WM);
  const int num_kb = static_cast<int>((K + BK - 1) / BK);
  int s = kMaxCtas / nt;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s > num_kb) s = num_kb;
  const int per = (num_kb + s - 1) / s;
  *ntiles = nt;
  *kb_per = per;
  *splits = (num_kb + per - 1) / per;
}

template <int NP, int OUT_S32>
cudaError_t launch_cfg(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a, cudaStream_t stream) {
  using Lay = Layout<NP>;
  static bool attrs_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attrs_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(smallm_kernel<NP, OUT_S32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Lay::kAlloc);
    if (e != cudaSuccess) return e;
    // the whole unified L1/shared array as shared memory, so that two CTAs fit per SM
    e = cudaFuncSetAttribute(smallm_kernel<NP, OUT_S32>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attrs_set[dev] = true;
  }
  int nt, per, splits;
  smallm_plan(a.N, a.K, a.num_sms, &nt, &per, &splits);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  fill_cfg<NP, OUT_S32>(&cfg, attr, nt * splits, splits, stream);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, smallm_kernel<NP, OUT_S32>, tmW, tmX, a, per, splits);
}

template <int NP>
cudaError_t launch_np(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a, cudaStream_t stream) {
  cudaError_t e = a.out_s32 ? launch_cfg<NP, 1>(tmW, tmX, a, stream) : launch_cfg<NP, 0>(tmW, tmX, a, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t smallm_launch_tm(const CUtensorMap& tmW, const CUtensorMap& tmX, const SmallMArgs& a,
                             cudaStream_t stream) {
  if (a.M <= 16) return launch_np<16>(tmW, tmX, a, stream);
  if (a.M <= 32) return launch_np<32>(tmW, tmX, a, stream);
  return launch_np<64>(tmW, tmX, a, stream);
}

int smallm_rows_padded(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

}  // namespace w4a4
