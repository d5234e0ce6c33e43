// Y = A Q on the tcgen05 tensor cores for the subspace iteration of the
// factor refresh (review page, section V.E / Algorithm 1: refresh of the
// rank-32 input-side factor).  A (d x d) and Q (d x m, m <= 64) are fp32;
// both are split into bf16 hi + lo so that
//   A Q ~ A_hi [Q_hi | Q_lo] + A_lo [Q_hi | Q_lo]     (~2^-16 relative)
// with fp32 accumulation in TMEM.  The split copies are written by
// split_a_kernel (A) and by the orthonormalisation (Q, as a [d][128] bf16
// operand: columns 0..63 the hi parts, 64..127 the lo parts).  This serves
// the iteration products, whose rounding only perturbs the sampled subspace;
// the Rayleigh-Ritz product stays on the fp32 CUDA-core kernel.
//
// One CTA per (128-row tile, k-slice, layer); 4-stage TMA ring of
// {A_hi, A_lo [128 rows][64 k], Q split [64 k][128]} = 48 KB per stage;
// warp 4 issues TMA, warp 5 the MMAs (M=128, N=128, K=16), warps 0-3 add the
// hi and lo column halves and store the k-slice of Y.
#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {
namespace {

constexpr int kM = 128, kK = 64, kStages = 4;
constexpr int kABytes = kM * kK * 2;            // 16 KB per bf16 A box
constexpr int kQBox = kK * 64 * 2;              // 8 KB: [64 k][64 n] bf16
constexpr int kStageBytes = 2 * kABytes + 2 * kQBox;
constexpr int kSmem = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kIdesc = umma_idesc_bf16(128, 128, 0, 1);  // A K-major, B MN-major
constexpr uint32_t kWaitLimit = 1u << 22;

struct alignas(64) SkLayer {
  CUtensorMap tmAh, tmAl;  // bf16 [d][d], box [128][64]
  CUtensorMap tmQ;         // bf16 [d][128], box [64][64]
  float* Yp;               // ns k-slices of d x m fp32
  int d, ns, kslice, pad;
};
struct SkParams {
  SkLayer L[kSkinnyMaxBatch];
  int m;
};

__global__ void __launch_bounds__(192, 1) skinny_tc_kernel(const __grid_constant__ SkParams p) {
  const SkLayer& L = p.L[blockIdx.z];
  if ((int)blockIdx.x >= L.d / kM || (int)blockIdx.y >= L.ns) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = (uint64_t*)(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kM;
  const int k0 = blockIdx.y * L.kslice;
  const int k1 = min(L.d, k0 + L.kslice);
  const int nk = k1 > k0 ? (k1 - k0 + kK - 1) / kK : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      for (int k = 0; k < nk; ++k) {
        const int s = k % kStages;
        if (k >= kStages && !mbar_wait(&empty[s], ((k / kStages) - 1) & 1u, kWaitLimit)) break;
        uint8_t* st = smem + s * kStageBytes;
        const int kc = k0 + k * kK;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(st, &L.tmAh, &full[s], kc, row0);
        tma_load_2d(st + kABytes, &L.tmAl, &full[s], kc, row0);
        tma_load_2d(st + 2 * kABytes, &L.tmQ, &full[s], 0, kc);
        tma_load_2d(st + 2 * kABytes + kQBox, &L.tmQ, &full[s], 64, kc);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      for (int k = 0; k < nk; ++k) {
        const int s = k % kStages;
        if (!mbar_wait(&full[s], (k / kStages) & 1u, kWaitLimit)) break;
        tc_fence_after();
        const uint32_t ah = sbase + s * kStageBytes, al = ah + kABytes, qb = ah + 2 * kABytes;
#pragma unroll
        for (int kk = 0; kk < kK / 16; ++kk) {
          // B: 16 k-rows of 128 B, the two 64-column halves one box apart
          const uint64_t bd = umma_desc_sw128(qb + kk * 2048, kQBox, 1024);
          umma_bf16(tbase, umma_desc_sw128(ah + kk * 32, 16, 1024), bd, kIdesc, (k | kk) ? 1u : 0u);
          umma_bf16(tbase, umma_desc_sw128(al + kk * 32, 16, 1024), bd, kIdesc, 1u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
    }
  } else {
    const bool ok = nk == 0 || mbar_wait(acc_full, 0, kWaitLimit);
    tc_fence_after();
    const int row = row0 + warp * 32 + lane;
    float y[64];
    if (ok && nk > 0) {
      uint32_t r[32];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + g * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) y[g * 32 + t] = __uint_as_float(r[t]);
      }
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + 64 + g * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) y[g * 32 + t] += __uint_as_float(r[t]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < 64; ++t) y[t] = 0.0f;
    }
    float* out = L.Yp + (int64_t)blockIdx.y * L.d * p.m + (int64_t)row * p.m;
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (c < p.m) out[c] = y[c];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tbase, 128);
}

unsigned long long g_attr = 0;

}  // namespace

cudaError_t launch_skinny_tc(const SkinnyTcJob* jobs, int n, int m, cudaStream_t s) {
  cudaError_t e = ensure_smem_attr(skinny_tc_kernel, kSmem, &g_attr);
  if (e != cudaSuccess) return e;
  for (int base = 0; base < n; base += kSkinnyMaxBatch) {
    const int cnt = n - base < kSkinnyMaxBatch ? n - base : kSkinnyMaxBatch;
    static thread_local SkParams P;
    P.m = m;
    int tiles = 1, nsmax = 1;
    for (int l = 0; l < cnt; ++l) {
      const SkinnyTcJob& J = jobs[base + l];
      SkLayer& L = P.L[l];
      if (!make_tmap_2d(&L.tmAh, J.Ah, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, J.d, J.d, kM, kK) ||
          !make_tmap_2d(&L.tmAl, J.Al, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, J.d, J.d, kM, kK) ||
          !make_tmap_2d(&L.tmQ, J.Qs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, J.d, 128, kK, 64))
        return cudaErrorInvalidValue;
      L.Yp = J.Yp;
      L.d = J.d;
      L.ns = J.ns;
      L.kslice = J.kslice;
      tiles = J.d / kM > tiles ? J.d / kM : tiles;
      nsmax = J.ns > nsmax ? J.ns : nsmax;
    }
    skinny_tc_kernel<<<dim3(tiles, nsmax, cnt), 192, kSmem, s>>>(P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gift
