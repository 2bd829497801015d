// Comparison kernel: the s4 x s4 -> s32 GEMM in the design of the page
// "[PR #63] int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA kernels"
// (Description: a main loop of warp-level mma.m16n8k64.s4 fed from shared
// memory, with the scales kept out of the K loop), written fresh for sm_100a
// so that it can be measured against the tcgen05 kernel.  It produces raw
// int32 accumulators only (w4a4_gemm_s32, path 2).
//
// Design
//   * One CTA per 128 x 128 output tile; eight warps of 64 x 32 (4 x 4
//     m16n8 tiles, 64 int32 accumulators per thread).
//   * One thread TMA-loads the packed A and B rows of a k-block (128 codes =
//     64 bytes per row) into a 4-deep ring; the tile lands with the 64-byte
//     swizzle (16-byte chunk c of row r at c ^ ((r >> 1) & 3)), so the
//     ldmatrix row reads are free of bank conflicts.
//   * A fragments come from ldmatrix.x4 (8 x 16-byte rows per matrix = 8 rows
//     x 32 codes; thread t receives codes 8 (t % 4) .. 8 (t % 4) + 7 of row
//     t / 4, the layout of the m16n8k64 s4 A and B fragments), B fragments
//     from ldmatrix.x4 covering two n8 tiles.
//   * Waits on the ring are bounded like every other wait of the library.
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int LT = 128;         // tile rows (A) and columns (B)
constexpr int LBK = 128;        // codes per k-block
constexpr int LBKP = LBK / 2;   // packed bytes per row per k-block
constexpr int LS = 4;           // ring depth
constexpr int kLWarps = 8;
constexpr int kLThreads = (kLWarps + 1) * 32;   // eight MMA warps + one producer warp
constexpr uint32_t kLStage = 2 * LT * LBKP;     // A + B, 16 KB
constexpr uint32_t kLSmem = LS * kLStage + 1024;

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_s4(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k64.row.col.s32.s4.s4.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory address of 16-byte chunk `c` (0..3) of packed row `r` in a
// 64-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw64(uint32_t base, int r, int c) {
  return base + r * LBKP + ((c ^ ((r >> 1) & 3)) << 4);
}

__global__ void __launch_bounds__(kLThreads, 1)
    gemm_legacy_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       int32_t* __restrict__ out, int64_t M, int64_t N, int64_t K, int64_t ldo,
                       unsigned int* status) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ uint64_t full[LS], empty[LS];
  __shared__ int abort_flag;
  uint8_t* smem = align1024_shared(smem_dyn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_n = static_cast<int>((N + LT - 1) / LT);
  const int mb = blockIdx.x / num_n, nb = blockIdx.x % num_n;
  const int num_kb = static_cast<int>((K + LBK - 1) / LBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < LS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kLWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kLWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(&full[s], kLStage);
        uint8_t* dst = smem + s * kLStage;
        tma_load_2d(dst, &tmA, &full[s], kb * LBKP, mb * LT);
        tma_load_2d(dst + LT * LBKP, &tmB, &full[s], kb * LBKP, nb * LT);
        ++issued;
        if (++s == LS) { s = 0; ph ^= 1; }
      }
      if (abort_flag) {
        for (int s2 = 0; s2 < LS && s2 < issued; ++s2) {
          const int n_s = issued / LS + (s2 < issued % LS ? 1 : 0);
          (void)mbar_wait(&full[s2], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ MMA warps
  const int wm = warp >> 2;   // 0..1: 64-row half
  const int wn = warp & 3;    // 0..3: 32-column quarter
  int acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;
  // ldmatrix.x4 row address of this lane: matrix lane / 8 (rows +8 for odd
  // matrices, 16-byte chunk +1 for matrices 2 and 3 of A)
  const int lr = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lc = lane >> 4;
  uint32_t s = 0, ph = 0;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!warp_wait(&full[s], ph, &abort_flag, status)) break;
    const uint32_t a_base = smem_u32(smem + s * kLStage);
    const uint32_t b_base = a_base + LT * LBKP;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {   // two k64 steps per k-block
      uint32_t a[4][4], b[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        ldmatrix_x4(sw64(a_base, wm * 64 + i * 16 + lr, 2 * ks + lc), a[i][0], a[i][1], a[i][2], a[i][3]);
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        // matrices: n rows 0-7 chunk k0, n rows 0-7 chunk k1, n rows 8-15 chunk k0, n rows 8-15 chunk k1
        const int br = wn * 32 + j * 8 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int bc = 2 * ks + ((lane >> 3) & 1);
        ldmatrix_x4(sw64(b_base, br, bc), b[j][0], b[j][1], b[j + 1][0], b[j + 1][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_s4(acc[i][j], a[i], b[j][0], b[j][1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == LS) { s = 0; ph ^= 1; }
  }
  if (abort_flag) return;
  // c0, c1: row gid, columns 2 tig, 2 tig + 1; c2, c3: row gid + 8
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = static_cast<int64_t>(nb) * LT + wn * 32 + j * 8 + 2 * tig;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t m = static_cast<int64_t>(mb) * LT + wm * 64 + i * 16 + gid + 8 * h;
        if (m >= M) continue;
        if (n < N) out[m * ldo + n] = acc[i][j][2 * h];
        if (n + 1 < N) out[m * ldo + n + 1] = acc[i][j][2 * h + 1];
      }
    }
  }
}

}  // namespace

cudaError_t gemm_legacy_launch(const CUtensorMap& tmA, const CUtensorMap& tmB, int32_t* out, int64_t M, int64_t N,
                               int64_t K, int64_t ldo, unsigned int* status, cudaStream_t stream) {
  const int64_t tiles = ((M + LT - 1) / LT) * ((N + LT - 1) / LT);
  if (tiles == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gemm_legacy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kLSmem));
  if (e != cudaSuccess) return e;
  gemm_legacy_kernel<<<static_cast<unsigned>(tiles), kLThreads, kLSmem, stream>>>(tmA, tmB, out, M, N, K, ldo,
                                                                                 status);
  return cudaGetLastError();
}

}  // namespace w4a4
