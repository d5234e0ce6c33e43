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
// per 64 features.  One CTA per (tile, token split):
//   warp 4     TMA producer (4-stage ring, 48 KB per stage)
//   warp 5     TMEM allocation and the single-thread MMA issue
//   warps 0-3  epilogue: TMEM -> registers -> A (j >= i only, mirrored),
//              or raw partial sums when the token range is split.
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
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t IDESC = umma_idesc_bf16(BM, BN, /*a MN-major*/ 1, /*b MN-major*/ 1);
constexpr uint32_t kWaitLimit = 1u << 22;

struct SyrkArgs {
  int d;
  int64_t N;
  int splits;
  int64_t rows_per_split;
  float scale;
  float* A;       // direct output (splits == 1)
  float* part;    // splits x d x d raw partial sums (splits > 1)
  uint32_t* err;  // optional device status word
};

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

__global__ void __launch_bounds__(192, 1) syrk_tc_kernel(const __grid_constant__ CUtensorMap tmX, SyrkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 1);
  __shared__ int failed;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % a.splits;
  int I, J2;
  tile_of(blockIdx.x / a.splits, a.d, &I, &J2);
  const int64_t n_begin = (int64_t)split * a.rows_per_split;
  int64_t n_end = n_begin + a.rows_per_split;
  if (n_end > a.N) n_end = a.N;
  const int nk = n_end > n_begin ? (int)((n_end - n_begin + BK - 1) / BK) : 0;

  if (threadIdx.x == 0) {
    failed = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      for (int k = 0; k < nk; ++k) {
        const int s = k % STAGES;
        const uint32_t ph = (uint32_t)(k / STAGES) & 1u;
        if (k >= STAGES && !mbar_wait(&empty[s], ph ^ 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        uint8_t* sa = smem + s * STAGE_BYTES;
        uint8_t* sb = sa + A_BYTES;
        const int y = (int)(n_begin + (int64_t)k * BK);
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d(sa, &tmX, &full[s], I * BM, y);
        tma_load_2d(sa + BOX_BYTES, &tmX, &full[s], I * BM + 64, y);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(sb + b * BOX_BYTES, &tmX, &full[s], J2 * BN + b * 64, y);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      for (int k = 0; k < nk; ++k) {
        const int s = k % STAGES;
        const uint32_t ph = (uint32_t)(k / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph, kWaitLimit)) {
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
          umma_bf16(tbase, ad, bd, IDESC, (k > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
    }
  } else {
    // epilogue: thread = output row i, 32 columns per TMEM load
    const bool ok = (nk == 0) || mbar_wait(acc_full, 0, kWaitLimit);
    if (!ok) failed = 1;
    tc_fence_after();
    const int i = I * BM + warp * 32 + lane;
    const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
    for (int cc = 0; cc < BN / 32; ++cc) {
      uint32_t r[32];
      if (nk > 0) {
        tmem_ld32(trow + cc * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) r[t] = 0u;
      }
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int j = J2 * BN + cc * 32 + t;
        if (j < i || j >= a.d) continue;
        const float v = __uint_as_float(r[t]);
        if (a.splits == 1) {
          a.A[(int64_t)i * a.d + j] = v * a.scale;
          if (j != i) a.A[(int64_t)j * a.d + i] = v * a.scale;
        } else {
          a.part[(int64_t)split * a.d * a.d + (int64_t)i * a.d + j] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tbase, TMEM_COLS);
  if (threadIdx.x == 0 && failed && a.err) atomicOr(a.err, GIFT_DEV_TIMEOUT);
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
  CUtensorMap tm;
  if (!make_tmap_2d(&tm, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)d, 64, 64))
    return cudaSuccess;  // no driver entry point: the CUDA-core syrk runs instead
  cudaError_t e = ensure_smem_attr(syrk_tc_kernel, SMEM_BYTES, &g_attr_mask);
  if (e != cudaSuccess) return e;
  SyrkArgs a;
  a.d = d;
  a.N = N;
  a.splits = splits < 1 ? 1 : splits;
  a.rows_per_split = ((N + a.splits - 1) / a.splits + BK - 1) / BK * BK;
  a.scale = (float)(1.0 / (double)N);
  a.A = A;
  a.part = part;
  a.err = err;
  const int items = syrk_tc_tiles(d) * a.splits;
  syrk_tc_kernel<<<items, 192, SMEM_BYTES, s>>>(tm, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.splits > 1) e = launch_syrk_reduce(part, a.splits, d, A, a.scale, s);
  *used = true;
  return e;
}

}  // namespace gift
