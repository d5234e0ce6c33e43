// E4M3 codec under a dense d_in x d_in input-side transform, on the tcgen05
// tensor cores (bf16 gradients).
//
// The GIFT review page ("What carries the argument") describes the rank-32
// codec as the last of a chain of simplifications: full two-sided K-FAC
// whitening, then the input side alone at full rank, then rank 32 (Fig. 2
// caption); section IV.A, Eq. (14) writes the input side with the Cholesky
// factor L_A^{-T}.  Those variants whiten with a dense matrix M:
//   encode  W = G M, per-row 128-column blocks, E4M3 codes and fp32 scales
//   decode  G_hat = W_hat M^{-1},  W_hat = value(codes) * scale (per block)
// with M = L^{-T} (Cholesky) or A^{-1/2} (full rank); dense_factor.cu makes
// them.  Both products are dense GEMMs, so both kernels are tensor-core
// bound.  G is exact in bf16.  M arrives as three bf16 parts (M ~ M_hi +
// M_mid + M_lo, ~2^-24 relative): the entries of a whitening transform are
// large next to W = G M (the sum cancels), so the encoder needs M to fp32
// accuracy for its codes; M^{-1} arrives as a hi/lo pair (~2^-17), enough for
// G_hat.  Accumulation is fp32 in TMEM.
//
// Encode: one CTA per 128 x 128 tile of W (one E4M3 block per row), K = d_in
// streamed in 64-column steps by TMA: G [128][64] (K-major) and the three
// parts of M [64][128] (MN-major, two 64-column boxes each), 3-stage ring.  Warp 4 issues
// TMA, warp 5 the MMAs (M=128, N=128, K=16), warps 0-3 own one row each: the
// row's 128 accumulators are its whole block, so the block maximum, the scale
// and the codes need no exchange.
// Decode: one CTA per 128 x 128 tile of G_hat, K = d_in streamed one scale
// block (128 columns) at a time: the codes tile [128][128] and M^{-1} hi/lo
// [128][128].  Codes are exact in bf16, so the converter warps 4-7 widen
// them into the A operand and each block's product T_c = q_c M^{-1}_c lands
// in one of two TMEM accumulators; the epilogue adds s_c T_c in fp32
// registers (the scale differs per row and block, so it is applied after the
// product).  Warp 8 issues TMA, warp 9 the MMAs.
// An upper-triangular M (the Cholesky form: L^{-T} and L^T are both upper
// triangular) lets a tile stop its K loop at its own last column.
#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {
namespace {

constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t kIdesc = umma_idesc_bf16(128, 128, 0, 1);  // A K-major, B MN-major

// ---------------------------------------------------------------- encode
constexpr int kEStages = 3;
constexpr int kEA = 128 * 64 * 2;        // G box [128 rows][64 k], 16 KB
constexpr int kEBox = 64 * 64 * 2;       // M box [64 k][64 n], 8 KB
constexpr int kEStage = kEA + 6 * kEBox; // G + three parts of M (2 boxes each) = 64 KB
constexpr int kESmem = kEStages * kEStage + 1024 + 256;

struct alignas(64) DenseEnc {
  CUtensorMap tmG;   // bf16 [d_out][d_in], box [128][64]
  CUtensorMap tmM[3];  // bf16 [d_in][d_in] hi, mid, lo; box [64][64]
  uint8_t* codes;
  float* scales;
  int d_out, d_in, upper;
};

__global__ void __launch_bounds__(192, 1) dense_encode_tc_kernel(const __grid_constant__ DenseEnc p, uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = (uint64_t*)(smem + kEStages * kEStage);
  uint64_t* empty = full + kEStages;
  uint64_t* acc_full = empty + kEStages;
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 1);
  __shared__ int failed, nonfin;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, row0 = blockIdx.y * 128;
  const int k_end = p.upper ? min(p.d_in, n0 + 128) : p.d_in;
  const int nk = k_end / 64;

  if (threadIdx.x == 0) {
    failed = 0;
    nonfin = 0;
    for (int s = 0; s < kEStages; ++s) {
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
        const int s = k % kEStages;
        if (k >= kEStages && !mbar_wait(&empty[s], ((k / kEStages) - 1) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        uint8_t* st = smem + s * kEStage;
        mbar_arrive_expect_tx(&full[s], kEStage);
        tma_load_2d(st, &p.tmG, &full[s], k * 64, row0);
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          tma_load_2d(st + kEA + 2 * t * kEBox, &p.tmM[t], &full[s], n0, k * 64);
          tma_load_2d(st + kEA + (2 * t + 1) * kEBox, &p.tmM[t], &full[s], n0 + 64, k * 64);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      int k = 0;
      for (; k < nk; ++k) {
        const int s = k % kEStages;
        if (!mbar_wait(&full[s], (k / kEStages) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a = sbase + s * kEStage, b0 = a + kEA;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // B: 16 k-rows of 128 B, the two 64-column halves one box apart
          const uint64_t ad = umma_desc_sw128(a + kk * 32, 16, 1024);
#pragma unroll
          for (int t = 0; t < 3; ++t)
            umma_bf16(tbase, ad, umma_desc_sw128(b0 + 2 * t * kEBox + kk * 2048, kEBox, 1024), kIdesc,
                      (k | kk | t) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      // every issued MMA has completed when acc_full completes, also after a
      // give-up (then nothing is stored); wait for it here too, so that TMEM
      // is released only once no MMA writes it
      umma_commit(acc_full);
      mbar_wait(acc_full, 0, kWaitLimit);
    }
  } else if (warp < 4) {
    // epilogue: thread = one row of the tile = its TMEM lane
    const bool ok = mbar_wait(acc_full, 0, kWaitLimit);
    tc_fence_after();
    const int64_t row = (int64_t)row0 + warp * 32 + lane;
    float w[128];
    const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t r[32];
      tmem_ld32(trow + g * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t) w[g * 32 + t] = __uint_as_float(r[t]);
    }
    if (!ok) failed = 1;
    if (ok && !failed && row < p.d_out) {
      float m0 = 0.0f, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
#pragma unroll
      for (int t = 0; t < 128; t += 4) {
        m0 = fmax_nan(m0, fabsf(w[t]));
        m1 = fmax_nan(m1, fabsf(w[t + 1]));
        m2 = fmax_nan(m2, fabsf(w[t + 2]));
        m3 = fmax_nan(m3, fabsf(w[t + 3]));
      }
      const float amax = fmax_nan(fmax_nan(m0, m1), fmax_nan(m2, m3));
      if (not_finite(amax)) nonfin = 1;
      const float inv = e4m3_inv_scale(amax);
      uint4* dst = reinterpret_cast<uint4*>(p.codes + row * p.d_in + n0);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = q * 16 + e * 4;
          const uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(w[t], inv), __fmul_rn(w[t + 1], inv));
          const uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(w[t + 2], inv), __fmul_rn(w[t + 3], inv));
          c[e] = inv > 0.0f ? (lo | (hi << 16)) : 0u;
        }
        dst[q] = make_uint4(c[0], c[1], c[2], c[3]);
      }
      p.scales[row * (p.d_in / 128) + n0 / 128] = e4m3_scale(amax, inv);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) tmem_dealloc(tbase, 128);
  if (threadIdx.x == 0 && err && (failed || nonfin))
    atomicOr(err, (failed ? GIFT_DEV_TIMEOUT : 0u) | (nonfin ? GIFT_DEV_NONFINITE : 0u));
}

// ---------------------------------------------------------------- decode
constexpr int kDStages = 2;
constexpr int kDCodes = 128 * 128;           // codes box [128 rows][128 k], 16 KB
constexpr int kDBox = 128 * 64 * 2;          // M^{-1} box [128 k][64 n], 16 KB
constexpr int kDStage = kDCodes + 4 * kDBox; // 80 KB
constexpr int kDAbuf = 128 * 128 * 2;        // widened codes: two K-major [128][64] bf16 boxes, 32 KB
constexpr int kDSmem = kDStages * kDStage + 2 * kDAbuf + 1024 + 256;
static_assert(kDSmem <= 232448, "dense decode shared memory");

struct alignas(64) DenseDec {
  CUtensorMap tmC;   // uint8 [d_out][d_in], box [128][128]
  CUtensorMap tmMh;  // bf16 [d_in][d_in], box [128][64]
  CUtensorMap tmMl;
  const float* scales;
  void* G_hat;
  int d_out, d_in, upper, out_f32;
};

// E4M3 pair -> bf16 pair, exact (an E4M3 value has at most 4 significant bits)
GIFT_DEV uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  const float2 f = e4m3x2_to_f32x2(v);
  return pack_bf16x2(f.x, f.y);
}

GIFT_DEV void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__global__ void __launch_bounds__(320, 1) dense_decode_tc_kernel(const __grid_constant__ DenseDec p, uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t abase = sbase + kDStages * kDStage;
  uint64_t* tfull = (uint64_t*)(smem + kDStages * kDStage + 2 * kDAbuf);  // [2] TMA landed
  uint64_t* empty = tfull + kDStages;    // [2] count 2: converter read the codes + MMA commit
  uint64_t* afull = empty + kDStages;    // [2] count 1: widened codes written
  uint64_t* afree = afull + 2;           // [2] count 1: MMA commit
  uint64_t* acc_full = afree + 2;        // [2] count 1: MMA commit
  uint64_t* acc_empty = acc_full + 2;    // [2] count 128: epilogue
  uint64_t* drain = acc_empty + 2;       // count 1: every MMA of this CTA has completed
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  __shared__ int failed, nonfin;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, row0 = blockIdx.y * 128;
  const int nc = p.upper ? min(p.d_in, n0 + 128) / 128 : p.d_in / 128;

  if (threadIdx.x == 0) {
    failed = 0;
    nonfin = 0;
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&empty[s], 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&afree[b], 1);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 8) {
    // ---- TMA producer
    if (lane == 0) {
      for (int c = 0; c < nc; ++c) {
        const int s = c % kDStages;
        if (c >= kDStages && !mbar_wait(&empty[s], ((c / kDStages) - 1) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        uint8_t* st = smem + s * kDStage;
        mbar_arrive_expect_tx(&tfull[s], kDStage);
        tma_load_2d(st, &p.tmC, &tfull[s], c * 128, row0);
        tma_load_2d(st + kDCodes, &p.tmMh, &tfull[s], n0, c * 128);
        tma_load_2d(st + kDCodes + kDBox, &p.tmMh, &tfull[s], n0 + 64, c * 128);
        tma_load_2d(st + kDCodes + 2 * kDBox, &p.tmMl, &tfull[s], n0, c * 128);
        tma_load_2d(st + kDCodes + 3 * kDBox, &p.tmMl, &tfull[s], n0 + 64, c * 128);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---- converters: row t's 128 codes -> bf16 into the K-major A operand
    const int t = threadIdx.x - 128;
    for (int c = 0; c < nc; ++c) {
      const int s = c % kDStages, j = c & 1;
      bool ok = mbar_wait(&tfull[s], (c / kDStages) & 1u, kWaitLimit);
      if (c >= 2) ok = ok && mbar_wait(&afree[j], ((c >> 1) - 1) & 1u, kWaitLimit);
      // every converter thread takes the same exit: the vote is a named barrier
      uint32_t any;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbarrier.red.or.pred p, 1, 128, q;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(any)
          : "r"((uint32_t)!ok)
          : "memory");
      if (any) {
        failed = 1;
        break;
      }
      const uint32_t ctile = sbase + s * kDStage;
      const uint32_t atile = abase + j * kDAbuf;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 v;
        const uint32_t addr = ctile + (uint32_t)t * 128u + (((uint32_t)q ^ ((uint32_t)t & 7u)) << 4);
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[2 * e] = e4m3x2_to_bf16x2((uint16_t)(w4[e] & 0xFFFFu));
          o[2 * e + 1] = e4m3x2_to_bf16x2((uint16_t)(w4[e] >> 16));
        }
        // codes 16 q .. 16 q + 15 -> bf16 chunks 2q, 2q+1 of the row's 256 bytes
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cc = 2 * q + h;  // 16-byte chunk of the 256-byte bf16 row
          const uint32_t dst = atile + (uint32_t)(cc >> 3) * (kDAbuf / 2) + (uint32_t)t * 128u +
                               ((((uint32_t)cc & 7u) ^ ((uint32_t)t & 7u)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[4 * h]), "r"(o[4 * h + 1]),
                       "r"(o[4 * h + 2]), "r"(o[4 * h + 3])
                       : "memory");
        }
      }
      fence_async_shared();
      named_bar(1, 128);
      if (t == 0) {
        mbar_arrive(&afull[j]);
        mbar_arrive(&empty[s]);  // the codes of this stage are read
      }
    }
  } else if (warp == 9) {
    // ---- MMA issuer: T_c = q_c (M^{-1}_hi + M^{-1}_lo)_c into accumulator c % 2
    if (lane == 0) {
      for (int c = 0; c < nc; ++c) {
        const int s = c % kDStages, j = c & 1, b = c & 1;
        bool ok = mbar_wait(&tfull[s], (c / kDStages) & 1u, kWaitLimit) &&
                  mbar_wait(&afull[j], (c >> 1) & 1u, kWaitLimit);
        if (c >= 2) ok = ok && mbar_wait(&acc_empty[b], ((c >> 1) - 1) & 1u, kWaitLimit);
        if (!ok) {
          failed = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a = abase + j * kDAbuf;
        const uint32_t bh = sbase + s * kDStage + kDCodes, bl = bh + 2 * kDBox;
        const uint32_t d = tbase + b * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = umma_desc_sw128(a + (kk >> 2) * (kDAbuf / 2) + (kk & 3) * 32, 16, 1024);
          umma_bf16(d, ad, umma_desc_sw128(bh + kk * 2048, kDBox, 1024), kIdesc, kk ? 1u : 0u);
          umma_bf16(d, ad, umma_desc_sw128(bl + kk * 2048, kDBox, 1024), kIdesc, 1u);
        }
        umma_commit(&empty[s]);
        umma_commit(&afree[j]);
        umma_commit(&acc_full[b]);
      }
      umma_commit(drain);  // TMEM is released only once no MMA writes it
      mbar_wait(drain, 0, kWaitLimit);
    }
  } else {
    // ---- epilogue (warps 0-3): acc += s_c T_c per block, then the row's 128 outputs
    const int64_t row = (int64_t)row0 + warp * 32 + lane;
    const bool live = row < p.d_out;
    const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
    float acc[128];
#pragma unroll
    for (int t = 0; t < 128; ++t) acc[t] = 0.0f;
    bool stop = false;
    for (int c = 0; c < nc && !stop; ++c) {
      const int b = c & 1;
      const float sc = live ? __ldg(p.scales + row * (p.d_in / 128) + c) : 0.0f;
      if (not_finite(sc)) nonfin = 1;
      if (!mbar_wait(&acc_full[b], (c >> 1) & 1u, kWaitLimit)) {
        failed = 1;
        stop = true;
      }
      tc_fence_after();
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t r[32];
        tmem_ld32(trow + b * 128 + g * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[g * 32 + t] = fmaf(sc, __uint_as_float(r[t]), acc[g * 32 + t]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
    if (live && !stop) {
      if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>((float*)p.G_hat + row * p.d_in + n0);
#pragma unroll
        for (int q = 0; q < 32; ++q) dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)p.G_hat + row * p.d_in + n0);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          dst[q] = make_uint4(pack_bf16x2(acc[8 * q], acc[8 * q + 1]), pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]),
                              pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]), pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) tmem_dealloc(tbase, 256);
  if (threadIdx.x == 0 && err && (failed || nonfin))
    atomicOr(err, (failed ? GIFT_DEV_TIMEOUT : 0u) | (nonfin ? GIFT_DEV_NONFINITE : 0u));
}

unsigned long long g_enc_attr = 0, g_dec_attr = 0;

}  // namespace

cudaError_t launch_dense_encode(const void* G, int d_out, int d_in, const uint16_t* M_split, bool upper,
                                uint8_t* codes, float* scales, uint32_t* err, cudaStream_t s) {
  static thread_local DenseEnc P;
  if (!make_tmap_2d(&P.tmG, G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)d_out, (uint64_t)d_in, 128, 64))
    return cudaErrorInvalidValue;
  for (int t = 0; t < 3; ++t)
    if (!make_tmap_2d(&P.tmM[t], M_split + (int64_t)t * d_in * d_in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                      (uint64_t)d_in, (uint64_t)d_in, 64, 64))
      return cudaErrorInvalidValue;
  P.codes = codes;
  P.scales = scales;
  P.d_out = d_out;
  P.d_in = d_in;
  P.upper = upper ? 1 : 0;
  cudaError_t e = ensure_smem_attr(dense_encode_tc_kernel, kESmem, &g_enc_attr);
  if (e != cudaSuccess) return e;
  dense_encode_tc_kernel<<<dim3(d_in / 128, (d_out + 127) / 128), 192, kESmem, s>>>(P, err);
  return cudaGetLastError();
}

cudaError_t launch_dense_decode(const uint8_t* codes, const float* scales, int d_out, int d_in,
                                const uint16_t* Minv_split, bool upper, void* G_hat, gift_dtype out_dt,
                                uint32_t* err, cudaStream_t s) {
  static thread_local DenseDec P;
  const uint16_t* Mh = Minv_split;
  const uint16_t* Ml = Minv_split + (int64_t)d_in * d_in;
  if (!make_tmap_2d(&P.tmC, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)d_out, (uint64_t)d_in, 128, 128) ||
      !make_tmap_2d(&P.tmMh, Mh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)d_in, (uint64_t)d_in, 128, 64) ||
      !make_tmap_2d(&P.tmMl, Ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)d_in, (uint64_t)d_in, 128, 64))
    return cudaErrorInvalidValue;
  P.scales = scales;
  P.G_hat = G_hat;
  P.d_out = d_out;
  P.d_in = d_in;
  P.upper = upper ? 1 : 0;
  P.out_f32 = out_dt == GIFT_F32 ? 1 : 0;
  cudaError_t e = ensure_smem_attr(dense_decode_tc_kernel, kDSmem, &g_dec_attr);
  if (e != cudaSuccess) return e;
  dense_decode_tc_kernel<<<dim3(d_in / 128, (d_out + 127) / 128), 320, kDSmem, s>>>(P, err);
  return cudaGetLastError();
}

}  // namespace gift
