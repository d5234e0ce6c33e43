// A = X^T X / N on the tcgen05 tensor cores (bf16 X, fp32 accumulation).
//
// GIFT review page, "What carries the argument": the input-side K-FAC factor
// A = E[a a^T] over the layer inputs; refreshed every K steps (section V.E,
// Algorithm 1).  This is the one dense contraction of the refresh:
// 2 N d^2 flops for d^2 outputs, so it is tensor-core bound.
//
// Tiling: output tiles of 128 (i) x 256 (j) covering the upper triangle
// (tiles whose j-range reaches i); the token dimension N is the MMA K
// dimension, streamed in 64-row chunks by TMA.  Both operands come straight
// from X's rows: X[n][i] has i contiguous, so A-operand (M = i) and
// B-operand (N = j) are MN-major 128-byte-swizzled tiles, one 64-column box
// per 64 features.  One launch covers a batch of layers (the batched factor
// refresh): a work item is (layer, tile, token split), and one persistent CTA
// per SM takes every gridDim.x-th item, the load ring and the accumulators
// running on from one item to the next so that a tile's stores overlap the
// next tile's MMAs.  Roles:
//   warp 8     TMA producer (4-stage ring, 48 KB per stage)
//   warp 9     TMEM allocation and the single-thread MMA issue
//   warps 0-7  epilogue: TMEM -> registers -> A (j >= i only, mirrored),
//              or raw partial sums when the token range is split.
// The tensor core's fp32 accumulation drifts low over long chains (measured
// ~3e-4 relative after 65536 tokens in one accumulator), so each TMEM
// accumulator only sums 2048 tokens; two accumulators alternate and the
// epilogue adds the blocks in fp32 registers with round-to-nearest.
#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {

cudaError_t launch_syrk_reduce(const float* part, int splits, int d, float* A, float scale, cudaStream_t s);

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;             // two 64-feature boxes
constexpr int B_BYTES = BN * BK * 2;             // four 64-feature boxes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 48 KB
constexpr int BOX_BYTES = 64 * BK * 2;           // 8 KB: 64 tokens x 128 B
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t TMEM_COLS = 512;   // two 256-column accumulators
constexpr int KB = 32;                // 64-token chunks per TMEM accumulation block (2048 tokens)
constexpr int THREADS = 320;
constexpr uint32_t IDESC = umma_idesc_bf16(BM, BN, /*a MN-major*/ 1, /*b MN-major*/ 1);
constexpr uint32_t kWaitLimit = 1u << 22;

struct alignas(64) SyrkLayer {
  CUtensorMap tmX;  // bf16 X [N][d], box [64 tokens][64 features], 128-byte swizzle
  int d;
  int tile_begin;   // first tile of this layer in the launch
  int64_t N;
  int64_t rows_per_split;
  float scale;
  float* A;         // direct output (splits == 1)
  float* part;      // splits x d x d raw partial sums (splits > 1)
  uint32_t* err;    // optional device status word
};
constexpr int kSyrkMaxBatch = 64;
struct SyrkBatch {
  SyrkLayer L[kSyrkMaxBatch];
  int n;
  int splits;
};
static_assert(sizeof(SyrkBatch) <= 32760, "kernel parameter space");

__device__ void tile_of(int t, int d, int* I, int* J2) {
  const int nI = d / BM, nJ = (d + BN - 1) / BN;
  int i = 0;
  while (i < nI && t >= nJ - i / 2) {
    t -= nJ - i / 2;
    ++i;
  }
  *I = i;
  *J2 = i / 2 + t;
}

// Work item `it` of a launch: layer, tile (I, J2) and token range.
struct Item {
  int l, I, J2, split, nk;
  int64_t n_begin;
};
__device__ Item item_of(const SyrkBatch& p, int it) {
  Item w;
  w.split = it % p.splits;
  const int tile = it / p.splits;
  int l = 0;
  while (l + 1 < p.n && tile >= p.L[l + 1].tile_begin) ++l;
  w.l = l;
  const SyrkLayer& a = p.L[l];
  tile_of(tile - a.tile_begin, a.d, &w.I, &w.J2);
  w.n_begin = (int64_t)w.split * a.rows_per_split;
  int64_t n_end = w.n_begin + a.rows_per_split;
  if (n_end > a.N) n_end = a.N;
  w.nk = n_end > w.n_begin ? (int)((n_end - w.n_begin + BK - 1) / BK) : 0;
  return w;
}

// Persistent: CTA b takes items b, b + gridDim.x, ...  The ring's chunk
// counter and the accumulation-block counter run on across items, so the
// epilogue's stores of one tile overlap the MMAs of the next.
__global__ void __launch_bounds__(THREADS, 1) syrk_tc_kernel(const __grid_constant__ SyrkBatch p, int items) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2] count 1
  uint64_t* acc_empty = acc_full + 2;    // [2] count 256
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 4);
  __shared__ int failed;
  __shared__ int failed_layer;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    failed = 0;
    failed_layer = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 256);
    }
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      uint32_t kg = 0;  // chunks loaded so far
      for (int it = blockIdx.x; it < items && !failed; it += gridDim.x) {
        const Item w = item_of(p, it);
        const CUtensorMap& tmX = p.L[w.l].tmX;
        tma_prefetch_desc(&tmX);
        for (int k = 0; k < w.nk; ++k, ++kg) {
          const int s = (int)(kg % STAGES);
          if (kg >= STAGES && !mbar_wait(&empty[s], ((kg / STAGES) - 1) & 1u, kWaitLimit)) {
            failed_layer = w.l;
            failed = 1;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          const int y = (int)(w.n_begin + (int64_t)k * BK);
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &tmX, &full[s], w.I * BM, y);
          tma_load_2d(sa + BOX_BYTES, &tmX, &full[s], w.I * BM + 64, y);
#pragma unroll
          for (int b = 0; b < 4; ++b) tma_load_2d(sb + b * BOX_BYTES, &tmX, &full[s], w.J2 * BN + b * 64, y);
        }
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      uint32_t kg = 0, bg = 0;  // chunks and accumulation blocks consumed so far
      for (int it = blockIdx.x; it < items && !failed; it += gridDim.x) {
        const Item w = item_of(p, it);
        for (int k = 0; k < w.nk; ++k, ++kg) {
          const int s = (int)(kg % STAGES);
          const uint32_t bgk = bg + (uint32_t)(k / KB);
          const int b = (int)(bgk & 1u);
          if (!mbar_wait(&full[s], (kg / STAGES) & 1u, kWaitLimit)) {
            failed_layer = w.l;
            failed = 1;
            break;
          }
          if (k % KB == 0 && bgk >= 2 && !mbar_wait(&acc_empty[b], ((bgk >> 1) - 1) & 1u, kWaitLimit)) {
            failed_layer = w.l;
            failed = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // 16 tokens = 16 rows of 128 B; MN groups (64 features) one box apart
            const uint64_t ad = umma_desc_sw128(a0 + kk * 2048, BOX_BYTES, 1024);
            const uint64_t bd = umma_desc_sw128(b0 + kk * 2048, BOX_BYTES, 1024);
            umma_bf16(tbase + b * BN, ad, bd, IDESC, (k % KB > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (k % KB == KB - 1 || k == w.nk - 1) umma_commit(&acc_full[b]);
        }
        bg += (uint32_t)((w.nk + KB - 1) / KB);
      }
    }
  } else {
    // epilogue: warp w owns rows 32*(w%4).. (its TMEM lane quarter) and
    // columns 128*(w/4)..+128 of the tile; blocks are summed in registers
    const int wq = warp & 3, wh = warp >> 2;
    uint32_t bg = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const Item w = item_of(p, it);
      const SyrkLayer& a = p.L[w.l];
      float sum[128];
#pragma unroll
      for (int t = 0; t < 128; ++t) sum[t] = 0.0f;
      const int nblk = (w.nk + KB - 1) / KB;
      const uint32_t trow = tbase + ((uint32_t)(wq * 32) << 16) + wh * 128;
      bool stop = false;
      for (int bk = 0; bk < nblk; ++bk, ++bg) {
        const int b = (int)(bg & 1u);
        if (!mbar_wait(&acc_full[b], (bg >> 1) & 1u, kWaitLimit)) {
          failed_layer = w.l;
          failed = 1;
          stop = true;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t r[32];
          tmem_ld32(trow + b * BN + g * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) sum[g * 32 + t] += __uint_as_float(r[t]);
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[b]);
      }
      if (stop) break;
      const int i = w.I * BM + wq * 32 + lane;
      const int j0 = w.J2 * BN + wh * 128;
      if (p.splits == 1) {
        // row i, columns j0 .. j0 + 127 (j >= i, j < d): 16-byte stores where
        // four columns are all kept; the mirror A[j][i] is coalesced over i
#pragma unroll
        for (int t = 0; t < 128; t += 4) {
          const int j = j0 + t;
          if (j >= i && j + 3 < a.d) {
            *reinterpret_cast<float4*>(a.A + (int64_t)i * a.d + j) =
                make_float4(sum[t] * a.scale, sum[t + 1] * a.scale, sum[t + 2] * a.scale, sum[t + 3] * a.scale);
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (j + u >= i && j + u < a.d) a.A[(int64_t)i * a.d + j + u] = sum[t + u] * a.scale;
          }
        }
#pragma unroll
        for (int t = 0; t < 128; ++t) {
          const int j = j0 + t;
          if (j > i && j < a.d) a.A[(int64_t)j * a.d + i] = sum[t] * a.scale;
        }
      } else {
#pragma unroll
        for (int t = 0; t < 128; ++t) {
          const int j = j0 + t;
          if (j >= i && j < a.d) a.part[(int64_t)w.split * a.d * a.d + (int64_t)i * a.d + j] = sum[t];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) tmem_dealloc(tbase, TMEM_COLS);
  if (threadIdx.x == 0 && failed && p.L[failed_layer].err) atomicOr(p.L[failed_layer].err, GIFT_DEV_TIMEOUT);
}

unsigned long long g_attr_mask = 0;

}  // namespace

int syrk_tc_tiles(int d) {
  const int nI = d / BM, nJ = (d + BN - 1) / BN;
  int t = 0;
  for (int i = 0; i < nI; ++i) t += nJ - i / 2;
  return t;
}

cudaError_t launch_syrk_tc(const void* X, gift_dtype xdt, int64_t N, int d, float* A, float* part, int splits,
                           uint32_t* err, cudaStream_t s, bool* used) {
  *used = false;
  if (xdt != GIFT_BF16 || d % BM != 0) return cudaSuccess;
  static thread_local SyrkBatch P;
  SyrkLayer& a = P.L[0];
  if (!make_tmap_2d(&a.tmX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)d, 64, 64))
    return cudaSuccess;  // no driver entry point: the CUDA-core syrk runs instead
  cudaError_t e = ensure_smem_attr(syrk_tc_kernel, SMEM_BYTES, &g_attr_mask);
  if (e != cudaSuccess) return e;
  P.n = 1;
  P.splits = splits < 1 ? 1 : splits;
  a.d = d;
  a.tile_begin = 0;
  a.N = N;
  a.rows_per_split = ((N + P.splits - 1) / P.splits + BK - 1) / BK * BK;
  a.scale = (float)(1.0 / (double)N);
  a.A = A;
  a.part = part;
  a.err = err;
  const int items = syrk_tc_tiles(d) * P.splits;
  syrk_tc_kernel<<<std::min(items, kNumSMs), THREADS, SMEM_BYTES, s>>>(P, items);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (P.splits > 1) e = launch_syrk_reduce(part, P.splits, d, A, a.scale, s);
  *used = true;
  return e;
}

cudaError_t launch_syrk_tc_batch(const SyrkJob* jobs, int n, cudaStream_t s, bool* used) {
  for (int l = 0; l < n; ++l) used[l] = false;
  if (n <= 0 || n > kSyrkMaxBatch) return cudaSuccess;
  static thread_local SyrkBatch P;
  int tiles = 0, m = 0;
  for (int l = 0; l < n; ++l) {
    const SyrkJob& J = jobs[l];
    if (J.xdt != GIFT_BF16 || J.d % BM != 0) continue;
    SyrkLayer& a = P.L[m];
    if (!make_tmap_2d(&a.tmX, J.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)J.N, (uint64_t)J.d, 64, 64))
      continue;  // no driver entry point: the CUDA-core syrk runs instead
    a.d = J.d;
    a.tile_begin = tiles;
    a.N = J.N;
    a.rows_per_split = (J.N + BK - 1) / BK * BK;
    a.scale = (float)(1.0 / (double)J.N);
    a.A = J.A;
    a.part = nullptr;
    a.err = J.err;
    tiles += syrk_tc_tiles(J.d);
    used[l] = true;
    ++m;
  }
  if (m == 0) return cudaSuccess;
  cudaError_t e = ensure_smem_attr(syrk_tc_kernel, SMEM_BYTES, &g_attr_mask);
  if (e != cudaSuccess) {
    for (int l = 0; l < n; ++l) used[l] = false;
    return e;
  }
  P.n = m;
  P.splits = 1;
  syrk_tc_kernel<<<std::min(tiles, kNumSMs), THREADS, SMEM_BYTES, s>>>(P, tiles);
  return cudaGetLastError();
}

}  // namespace gift
