// Dynamic LoRA on top of the W4A4 layer: y += scale * (x_rot A_rot^T) B^T.
//
// Page "Comfy-INT4-HIPtest README", section "LoRA modes": the Dynamic mode
// keeps the LoRA matrices separate and applies their deltas at inference
// time.  Page "ComfyUI-INT4-Fast" (features list, "Dynamic LoRA Patching"):
// the LoRA down projection is rotated with the layer's Hadamard transform so
// that it stays coherent with the rotated basis.  The rotation is orthogonal
// ((H / sqrt g)^2 = I), so the rotated activation against the rotated down
// projection is exactly x A^T; these kernels form that product from the bf16
// activation and the unrotated A, which is the same quantity with the
// rotation's roundings left out.
//
// B200 design (two small tcgen05 kernels, bf16 operands, fp32 accumulation):
//   * lora_down: t[M, r] = x[M, K] A[r, K]^T.  A CTA takes 128 rows of x and
//     one K slice (about two CTAs per SM over the row tiles).  TMA streams
//     64-element chunks of x (128 rows) and of A (r rows) into a 4-deep ring
//     in the 128-byte-swizzle K-major layout, one thread issues
//     tcgen05.mma.kind::f16 (M = 128, N = r, K = 16) into an fp32
//     accumulator in tensor memory, and each CTA writes its partial tile to
//     the workspace.  A small kernel then sums the slices' partials in a fixed
//     order (deterministic) and stores t in bf16 with a row stride of 64
//     elements, zero beyond r.  (Reducing the slices on chip, within a CTA
//     cluster, measured slower: only 15 clusters of eight fit at once.)
//   * lora_up: y[M, N] = bf16(y + scale * t B^T).  A persistent CTA (one
//     per SM) takes 128 x 256 output tiles: TMA loads the t tile (128 x 64),
//     the B tile (256 x 64, zero beyond r) and the y tile (four 64-column
//     boxes) into one of two stages, one thread issues r / 16 MMAs (M = 128,
//     N = 256, K = 16) into 256 fp32 columns of tensor memory, and eight
//     epilogue warps (two per lane quarter, one per half of the columns) add
//     scale * delta to the staged y in place; one thread then writes the
//     boxes back with TMA stores, which clip the M and N tails.
//   Every wait is bounded; an expired wait records W4A4_ERR_TIMEOUT, every
//   role stops, copies and MMAs drain and tensor memory is freed.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "w4a4_internal.h"

namespace w4a4 {
namespace {

constexpr int kRows = 128;         // MMA M: rows of x / y per tile
constexpr int kChunk = 64;         // bf16 elements per 128-byte row chunk
constexpr int kMaxSlices = 32;     // K slices per row tile at most

// ---------------------------------------------------------------- lora_down
constexpr int kDownStages = 4;
constexpr int kDownThreads = 128;  // warp 0: TMA, warp 1: MMA; all four: partial tile and reduction
constexpr uint32_t kDownX = kRows * 128;            // 16 KB: x chunk
constexpr uint32_t kDownA = kLoraMaxRank * 128;     // 8 KB: A chunk (r rows)
constexpr uint32_t kDownStage = kDownX + kDownA;
constexpr uint32_t kDownBytes = kDownStages * kDownStage;
constexpr uint32_t kDownAlloc = kDownBytes + 1024;

struct DownBars {
  uint64_t full[kDownStages];
  uint64_t empty[kDownStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// grid: (row tiles) x slices; slice s writes its partial sums to partial[s].
__global__ void __launch_bounds__(kDownThreads)
    lora_down_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                     float* __restrict__ partial, int64_t M, int64_t K, int r, int slices, int chunks_per_slice,
                     unsigned int* status, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ DownBars bars;
  uint8_t* smem = align1024_shared(smem_dyn);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x / slices;
  const int slice = blockIdx.x - tile * slices;   // = cluster rank
  const int nchunks_total = static_cast<int>((K + kChunk - 1) / kChunk);
  const int c0 = slice * chunks_per_slice;
  const int c1 = min(nchunks_total, c0 + chunks_per_slice);
  const int nch = c1 - c0;                         // >= 1 by construction
  const uint32_t a_bytes = static_cast<uint32_t>(r) * 128u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDownStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    mbar_init(&bars.acc_full, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmA);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 64);
    tmem_relinquish();
  }
  // x may be the previous kernel's output (launched with programmatic
  // stream serialization): nothing global is read before this point
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nch; ++i) {
        const int s = i % kDownStages;
        // row tiles start at different chunks of the slice, so that the CTAs
        // of one slice do not all read the same chunk of A at once
        const int c = c0 + (i + tile) % nch;
        if (!mbar_wait(&bars.empty[s], ((i / kDownStages) & 1) ^ 1, abort_flag, status, wait_ns)) break;
        mbar_arrive_expect_tx(&bars.full[s], kDownX + a_bytes);
        uint8_t* st = smem + s * kDownStage;
        tma_load_2d(st, &tmX, &bars.full[s], c * kChunk, tile * kRows);
        tma_load_2d(st + kDownX, &tmA, &bars.full[s], c * kChunk, 0);
        ++issued;
      }
      // every issued copy lands before the ring is reused or the CTA exits
      for (int s = 0; s < kDownStages && s < issued; ++s) {
        const int n_s = issued / kDownStages + (s < issued % kDownStages ? 1 : 0);
        (void)mbar_wait(&bars.full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kRows, r);
      for (int i = 0; i < nch; ++i) {
        const int s = i % kDownStages;
        if (!mbar_wait(&bars.full[s], (i / kDownStages) & 1, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * kDownStage));
        const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * kDownStage + kDownX));
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k) mma_bf16(tmem_base, ad + 2 * k, bd + 2 * k, idesc, (i | k) != 0 ? 1u : 0u);
        mma_commit(&bars.empty[s]);
      }
      mma_commit(&bars.acc_full);   // also the drain point after an abort
    }
  }
  __syncwarp();
  // ---- this slice's partial tile to the workspace: thread = row (tensor-
  // memory lane), 64 fp32 per row (zero beyond r).  The verdict is
  // warp-uniform: the tensor-memory loads are collective and are skipped
  // after an abort (the MMAs may still be running then).
  bool have = warp_wait(&bars.acc_full, 0, abort_flag, status, wait_ns) && *abort_flag == 0;
  have = __shfl_sync(0xFFFFFFFFu, have ? 1 : 0, 0) != 0;
  tc_fence_after();
  if (have) {
    const int row = warp * 32 + lane;
    const int64_t m = static_cast<int64_t>(tile) * kRows + row;
    float* dst = partial + (static_cast<int64_t>(slice) * M + m) * kLoraMaxRank;
    for (int c = 0; c < kLoraMaxRank; c += 16) {
      uint32_t v[16];
      if (c < r) {
        tmem_ld_x16(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + c, v);
        tmem_wait_ld();
      }
      if (m < M) {
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const uint4 w = c < r ? make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]) : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(dst + c + j) = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) (void)mbar_wait(&bars.acc_full, 0, nullptr, nullptr, 100000000ull);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 64);
  }
}

// ---------------------------------------------------------------- lora_reduce
// t[m, c] = bf16(sum over the slices s of partial[s][m][c]), summed in the
// order s = 0, 1, ... (deterministic); one thread per four columns of a row.
__global__ void __launch_bounds__(256)
    lora_reduce_kernel(const float* __restrict__ partial, uint16_t* __restrict__ t, int64_t M, int slices) {
  griddep_wait();   // the partial sums come from the previous kernel of the stream
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;   // (row, 4-column group)
  const int64_t m = i / (kLoraMaxRank / 4);
  if (m >= M) return;
  const int c = static_cast<int>(i % (kLoraMaxRank / 4)) * 4;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* src = partial + m * kLoraMaxRank + c;
  const int64_t slab = M * kLoraMaxRank;
  for (int s0 = 0; s0 < slices; s0 += 8) {
    // eight loads in flight, then the sums in slice order
    float4 p[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      p[k] = s0 + k < slices ? *reinterpret_cast<const float4*>(src + (s0 + k) * slab) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (s0 + k >= slices) break;
      sum.x += p[k].x;
      sum.y += p[k].y;
      sum.z += p[k].z;
      sum.w += p[k].w;
    }
  }
  *reinterpret_cast<uint2*>(t + m * kLoraMaxRank + c) = make_uint2(pack_bf16x2(sum.x, sum.y), pack_bf16x2(sum.z, sum.w));
}

// ---------------------------------------------------------------- lora_up
constexpr int kUpCols = 256;       // output columns per tile (MMA N)
constexpr int kUpStages = 2;       // operand + y buffers
constexpr int kUpEpiWarps = 8;     // two per tensor-memory lane quarter, one per half of the columns
constexpr int kUpThreads = (2 + kUpEpiWarps) * 32;   // warp 0: TMA, warp 1: MMA, warps 2-9: epilogue
constexpr uint32_t kUpT = kRows * 128;      // 16 KB: t tile (128 rows x 64)
constexpr uint32_t kUpB = kUpCols * 128;    // 32 KB: B tile (256 rows x 64)
constexpr uint32_t kUpBox = kRows * 128;    // 16 KB: 64 columns x 128 rows of y (128-byte swizzle)
constexpr uint32_t kUpY = 4 * kUpBox;       // 64 KB: the y tile (128 x 256), four boxes
constexpr uint32_t kUpStage = kUpT + kUpB + kUpY;
constexpr uint32_t kUpBytes = kUpStages * kUpStage;   // 224 KB
constexpr uint32_t kUpAlloc = kUpBytes + 1024;

struct UpBars {
  uint64_t full[kUpStages];     // t and B of a tile landed
  uint64_t yfull[kUpStages];    // the tile's y landed
  uint64_t op_empty[kUpStages]; // the MMA has read t and B
  uint64_t y_empty[kUpStages];  // the stores of the tile's y have read the buffer
  uint64_t acc_full;
  uint64_t acc_empty;           // kUpEpiWarps epilogue warps
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kUpThreads)
    lora_up_kernel(const __grid_constant__ CUtensorMap tmT, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, int64_t M, int64_t N, int r, float scale,
                   unsigned int* status, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_dyn[];
  __shared__ UpBars bars;
  uint8_t* smem = align1024_shared(smem_dyn);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = static_cast<int>((M + kRows - 1) / kRows);
  const int num_n = static_cast<int>((N + kUpCols - 1) / kUpCols);
  const int tiles = num_m * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kUpStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.yfull[s], 1);
      mbar_init(&bars.op_empty[s], 1);
      mbar_init(&bars.y_empty[s], 1);
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.acc_empty, kUpEpiWarps);
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
    tma_prefetch_desc(&tmT);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kUpCols);
    tmem_relinquish();
  }
  // t and y come from the previous kernels of the stream
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars.tmem_base;
  volatile int* abort_flag = &bars.abort_flag;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++issued) {
        const int s = issued % kUpStages;
        const uint32_t par = ((issued / kUpStages) & 1) ^ 1;
        if (!mbar_wait(&bars.op_empty[s], par, abort_flag, status, wait_ns) ||
            !mbar_wait(&bars.y_empty[s], par, abort_flag, status, wait_ns))
          break;
        // t and B (the MMA's operands) on one barrier, y on another, so that
        // the MMA need not wait for y; y boxes wholly past N are not loaded
        // (the epilogue stores none of them either)
        mbar_arrive_expect_tx(&bars.full[s], kUpT + kUpB);
        uint8_t* st = smem + s * kUpStage;
        const int mb = t / num_n, nb = t % num_n;   // CTAs running side by side share t and B tiles in L2
        tma_load_2d(st, &tmT, &bars.full[s], 0, mb * kRows);
        tma_load_2d(st + kUpT, &tmB, &bars.full[s], 0, nb * kUpCols);
        const int64_t nrem = N - static_cast<int64_t>(nb) * kUpCols;
        const int boxes = nrem >= kUpCols ? 4 : static_cast<int>((nrem + 63) / 64);
        mbar_arrive_expect_tx(&bars.yfull[s], static_cast<uint32_t>(boxes) * kUpBox);
        for (int b = 0; b < boxes; ++b)
          tma_load_2d(st + kUpT + kUpB + b * kUpBox, &tmY, &bars.yfull[s], nb * kUpCols + 64 * b, mb * kRows);
      }
      // every issued copy lands before the CTA can exit
      for (int s = 0; s < kUpStages && s < issued; ++s) {
        const int n_s = issued / kUpStages + (s < issued % kUpStages ? 1 : 0);
        (void)mbar_wait(&bars.full[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
        (void)mbar_wait(&bars.yfull[s], static_cast<uint32_t>((n_s - 1) & 1), nullptr, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kRows, kUpCols);
      int i = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int s = i % kUpStages;
        if (!mbar_wait(&bars.acc_empty, (i & 1) ^ 1, abort_flag, status, wait_ns)) break;
        if (!mbar_wait(&bars.full[s], (i / kUpStages) & 1, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * kUpStage));
        const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * kUpStage + kUpT));
        for (int k = 0; k < r / 16; ++k) mma_bf16(tmem_base, ad + 2 * k, bd + 2 * k, idesc, k != 0 ? 1u : 0u);
        mma_commit(&bars.op_empty[s]);
        mma_commit(&bars.acc_full);
      }
      mma_commit(&bars.drain);
      (void)mbar_wait(&bars.drain, 0, nullptr, nullptr, 100000000ull);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // Warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (= rows of the tile)
    // and the half (w - 2) / 4 of its columns.  The tile's y arrived in shared
    // memory by TMA (four 64-column boxes, 128-byte swizzle: 16-byte chunk c
    // of row m at chunk c ^ (m & 7)); each thread adds scale * delta to its
    // row's values in place, and one thread stores the boxes with TMA, which
    // also clips the M and N tails.
    const int q = warp & 3;
    const int half = (warp - 2) / 4;
    const int row = q * 32 + lane;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int s = i % kUpStages;
      bool ok = warp_wait(&bars.yfull[s], (i / kUpStages) & 1, abort_flag, status, wait_ns) &&
                warp_wait(&bars.acc_full, i & 1, abort_flag, status, wait_ns);
      // one verdict for the eight warps: they meet named barriers below
      if (bar_sync_or(1, kUpEpiWarps * 32, !ok)) break;
      tc_fence_after();
      const uint32_t ybuf = smem_u32(smem + s * kUpStage + kUpT + kUpB);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        const int c = half * (kUpCols / 2) + 32 * ch;   // first column of the chunk in the tile
        uint32_t v[32];
        tmem_ld_32x32b_x32(tl + c, v);
        tmem_wait_ld();
        const uint32_t box = ybuf + (c / 64) * kUpBox + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int cc = ((c % 64) / 8) + u;   // 16-byte chunk within the 128-byte box row
          const uint32_t a = box + ((cc ^ (row & 7)) << 4);
          uint4 w = lds128(a);
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // y + scale * delta with one rounding (a fused multiply-add), then bf16
            const float lo = __fmaf_rn(scale, __uint_as_float(v[8 * u + 2 * e]), __uint_as_float(wp[e] << 16));
            const float hi =
                __fmaf_rn(scale, __uint_as_float(v[8 * u + 2 * e + 1]), __uint_as_float(wp[e] & 0xFFFF0000u));
            wp[e] = pack_bf16x2(lo, hi);
          }
          sts128(a, w);
        }
      }
      tc_fence_before();
      fence_async_shared();   // the updated y is read next by the TMA stores
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty);   // the accumulator is free for the next tile
      asm volatile("bar.sync 2, %0;" ::"n"(kUpEpiWarps * 32) : "memory");
      if (warp == 2 && lane == 0) {
        const int mb = t / num_n, nb = t % num_n;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int64_t n0 = static_cast<int64_t>(nb) * kUpCols + 64 * b;
          if (n0 < N) tma_store_2d(&tmY, smem + s * kUpStage + kUpT + kUpB + b * kUpBox, static_cast<int32_t>(n0),
                                   mb * kRows);
        }
        bulk_commit_group();
        bulk_wait_group_read<0>();   // the stores have read the buffer
        mbar_arrive(&bars.y_empty[s]);
      }
    }
    if (warp == 2 && lane == 0) bulk_wait_group_read<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kUpCols);
  }
}

// 2-D map over a bf16 matrix [rows, cols] with row stride ld elements, box
// {64, box_rows}, 128-byte swizzle; out-of-range elements read as zero.
int bf16_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  return tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rows, cols, ld * 2, 64, box_rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// K slices of the down projection: about two CTAs per SM of a B200 (2 x 148)
// over the row tiles, at most kMaxSlices, at least one 64-element chunk
// each.  A fixed target keeps the workspace size a function of the shape.
int lora_slices(int64_t M, int64_t K) {
  const int64_t tiles = (M + kRows - 1) / kRows;
  const int64_t chunks = (K + kChunk - 1) / kChunk;
  int64_t s = 296 / (tiles > 0 ? tiles : 1);
  if (s > kMaxSlices) s = kMaxSlices;
  if (s < 1) s = 1;
  if (s > chunks) s = chunks;
  const int64_t per = (chunks + s - 1) / s;
  return static_cast<int>((chunks + per - 1) / per);   // every slice has at least one chunk
}

namespace {
}  // namespace

cudaError_t lora_down_launch(const uint16_t* x, int64_t ldx, const uint16_t* A, float* partial, uint16_t* t,
                             int64_t M, int64_t K, int r, unsigned int* status, cudaStream_t stream) {
  CUtensorMap tmX, tmA;
  if (bf16_map(&tmX, x, M, K, ldx, kRows) != 0 || bf16_map(&tmA, A, r, K, K, r) != 0)
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(lora_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDownAlloc);
    if (e != cudaSuccess) return e;
    // the whole unified L1/shared array as shared memory, so that two CTAs fit per SM
    e = cudaFuncSetAttribute(lora_down_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t tiles = (M + kRows - 1) / kRows;
  const int chunks = static_cast<int>((K + kChunk - 1) / kChunk);
  const int slices = lora_slices(M, K);
  const int per = (chunks + slices - 1) / slices;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * slices), 1, 1);
  cfg.blockDim = dim3(kDownThreads, 1, 1);
  cfg.dynamicSmemBytes = kDownAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, lora_down_kernel, tmX, tmA, partial, M, K, r, slices, per, status, wait_limit_ns());
  if (e != cudaSuccess) return e;
  // t = bf16(sum of the slices' partial sums)
  const int64_t threads = M * (kLoraMaxRank / 4);
  cudaLaunchConfig_t rc = {};
  rc.gridDim = dim3(static_cast<unsigned>((threads + 255) / 256), 1, 1);
  rc.blockDim = dim3(256, 1, 1);
  rc.stream = stream;
  rc.attrs = attr;
  rc.numAttrs = 1;
  e = cudaLaunchKernelEx(&rc, lora_reduce_kernel, static_cast<const float*>(partial), t, M, slices);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t lora_up_launch(const uint16_t* t, const uint16_t* B, uint16_t* y, int64_t ldy, int64_t M, int64_t N,
                           int r, float scale, int num_sms, unsigned int* status, cudaStream_t stream) {
  CUtensorMap tmT, tmB, tmY;
  if (bf16_map(&tmT, t, M, kLoraMaxRank, kLoraMaxRank, kRows) != 0 || bf16_map(&tmB, B, N, r, r, kUpCols) != 0 ||
      bf16_map(&tmY, y, M, N, ldy, kRows) != 0)
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(lora_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUpAlloc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lora_up_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t tiles = ((M + kRows - 1) / kRows) * ((N + kUpCols - 1) / kUpCols);
  const int64_t cap = static_cast<int64_t>(num_sms);   // one CTA per SM (224 KB of shared memory)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < cap ? tiles : cap), 1, 1);
  cfg.blockDim = dim3(kUpThreads, 1, 1);
  cfg.dynamicSmemBytes = kUpAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, lora_up_kernel, tmT, tmB, tmY, M, N, r, scale, status, wait_limit_ns());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a4
