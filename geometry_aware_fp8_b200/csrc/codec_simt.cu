// Whitened E4M3 codec on the CUDA cores (fp32 arithmetic), any rank <= 32.
//
// GIFT review page, "What carries the argument": W = G M before the FP8
// quantiser, G_hat = W_hat M^{-1} after it, with
//   M^{-+1} = a I + U diag(c) U^T   (a = rho^{-+1/2},
//                                    c_k = (lambda_k+rho)^{-+1/2} - a).
// One CTA owns one row of G; its warps take the row's 128-element scale
// blocks in turn (warp w: blocks w, w + 8, ...), and each lane holds four
// consecutive elements of a block.  Pass 1 forms each warp's share of
// P = g U (32 partial dot products per lane), reduces it across the lanes
// with a 31-shuffle transpose (lane k ends with coefficient k) and across the
// warps in warp order through shared memory; pass 2 forms w = a g +
// (P o c) U^T, the block maximum with five shuffles, and the codes.  This
// kernel serves fp32 gradients and ranks other than 32; the tensor-core
// kernel (codec_tc.cu) serves bf16 gradients at rank 32.
#include "common.cuh"
#include "internal.h"
#include "rowops.cuh"

namespace gift {
namespace {

constexpr int kWarps = 8;  // per CTA; one CTA per row

// P (32 coefficients) of the row from each warp's per-lane partial sums: the
// lanes by transpose, the warps in warp order; every thread returns with
// pc[k] = P_k c_k.  `part` and `pc_s` are reused row after row.
GIFT_DEV void row_projection(float (&P)[32], const float* c_s, float (*part)[32], float* pc_s, float (&pc)[32],
                             int warp, int lane) {
  part[warp][lane] = reduce_transpose32(P, lane);
  __syncthreads();
  if (warp == 0) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += part[w][lane];
    pc_s[lane] = s * c_s[lane];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 32; ++k) pc[k] = pc_s[k];
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) whiten_encode_simt_kernel(
    const T* __restrict__ G, int64_t d_out, int64_t d_in, const float* __restrict__ U,
    const float* __restrict__ lambda, const float* __restrict__ rho, int rank, uint8_t* __restrict__ codes,
    float* __restrict__ scales, uint32_t* err) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  __shared__ float part[kWarps][32];
  __shared__ float pc_s[32];
  transform_coeffs(lambda, rho, rank, false, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = (rank & 3) == 0;
  const int64_t nb = d_in / kBlock;
  bool bad = false;
  for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
    const T* g = G + row * d_in;
    float P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = 0.0f;
    for (int64_t b = warp; b < nb; b += kWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      float v[4];
      load4<T>(g + j0, v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
#pragma unroll
        for (int k = 0; k < 32; ++k) P[k] = fmaf(v[e], u[k], P[k]);
      }
    }
    float pc[32];
    row_projection(P, c_s, part, pc_s, pc, warp, lane);
    for (int64_t b = warp; b < nb; b += kWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      float v[4];
      load4<T>(g + j0, v);
      float w[4];
      float m = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) acc = fmaf(pc[k], u[k], acc);
        w[e] = fmaf(a, v[e], acc);
        m = fmax_nan(m, fabsf(w[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
      bad |= not_finite(m);
      uint32_t q = 0u;
      const float inv = e4m3_inv_scale(m);
      if (inv > 0.0f) {
        uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(w[0], inv), __fmul_rn(w[1], inv));
        uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(w[2], inv), __fmul_rn(w[3], inv));
        q = lo | (hi << 16);
      }
      *reinterpret_cast<uint32_t*>(codes + row * d_in + j0) = q;
      if (lane == 0) scales[row * nb + b] = e4m3_scale(m, inv);
    }
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) whiten_decode_simt_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales, int64_t d_out, int64_t d_in,
    const float* __restrict__ U, const float* __restrict__ lambda, const float* __restrict__ rho, int rank,
    T* __restrict__ out, uint32_t* err) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  __shared__ float part[kWarps][32];
  __shared__ float pc_s[32];
  transform_coeffs(lambda, rho, rank, true, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = (rank & 3) == 0;
  const int64_t nb = d_in / kBlock;
  bool bad = false;
  for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
    float P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = 0.0f;
    for (int64_t b = warp; b < nb; b += kWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(codes + row * d_in + j0));
      const float s = __ldg(scales + row * nb + b);
      float2 lo = e4m3x2_to_f32x2((uint16_t)(q & 0xFFFF)), hi = e4m3x2_to_f32x2((uint16_t)(q >> 16));
      const float v[4] = {lo.x * s, lo.y * s, hi.x * s, hi.y * s};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
#pragma unroll
        for (int k = 0; k < 32; ++k) P[k] = fmaf(v[e], u[k], P[k]);
      }
    }
    float pc[32];
    row_projection(P, c_s, part, pc_s, pc, warp, lane);
    for (int64_t b = warp; b < nb; b += kWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(codes + row * d_in + j0));
      const float s = __ldg(scales + row * nb + b);
      bad |= not_finite(s);
      float2 lo = e4m3x2_to_f32x2((uint16_t)(q & 0xFFFF)), hi = e4m3x2_to_f32x2((uint16_t)(q >> 16));
      const float v[4] = {lo.x * s, lo.y * s, hi.x * s, hi.y * s};
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) acc = fmaf(pc[k], u[k], acc);
        o[e] = fmaf(a, v[e], acc);
      }
      store4<T>(out + row * d_in + j0, o);
    }
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

// Decode-and-sum of the codes of several data-parallel ranks (the per-rank
// gradients g^(r) of Eq. (1) on the review page): every rank codes its own
// gradient with the shared factor, the codes and scales are all-gathered, and
// each rank forms alpha sum_r T^{-1}(W_hat_r) = alpha T^{-1}(sum_r W_hat_r)
// (T is linear, so the inverse transform is applied once, to the sum).
// Same row layout as the decoder above; W_hat is summed over the parts in
// part order in fp32.
constexpr int kMaxParts = 64;
struct SumParts {
  const uint8_t* codes[kMaxParts];
  const float* scales[kMaxParts];
  int n;
};

GIFT_DEV void load_sum4(const SumParts& sp, int64_t row, int64_t d_in, int64_t nb, int64_t b, int64_t j0,
                        float (&v)[4], bool& bad) {
  v[0] = v[1] = v[2] = v[3] = 0.0f;
  for (int r = 0; r < sp.n; ++r) {
    const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(sp.codes[r] + row * d_in + j0));
    const float s = __ldg(sp.scales[r] + row * nb + b);
    bad |= not_finite(s);
    const float2 lo = e4m3x2_to_f32x2((uint16_t)(q & 0xFFFF)), hi = e4m3x2_to_f32x2((uint16_t)(q >> 16));
    v[0] = fmaf(lo.x, s, v[0]);
    v[1] = fmaf(lo.y, s, v[1]);
    v[2] = fmaf(hi.x, s, v[2]);
    v[3] = fmaf(hi.y, s, v[3]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) whiten_decode_sum_simt_kernel(
    const __grid_constant__ SumParts sp, int64_t d_out, int64_t d_in, const float* __restrict__ U,
    const float* __restrict__ lambda, const float* __restrict__ rho, int rank, float alpha, T* __restrict__ out,
    uint32_t* err) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  __shared__ float part[kWarps][32];
  __shared__ float pc_s[32];
  transform_coeffs(lambda, rho, rank, true, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = (rank & 3) == 0;
  const int64_t nb = d_in / kBlock;
  bool bad = false;
  for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
    float P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = 0.0f;
    if (rank > 0) {
      for (int64_t b = warp; b < nb; b += kWarps) {
        const int64_t j0 = b * kBlock + lane * 4;
        float v[4];
        load_sum4(sp, row, d_in, nb, b, j0, v, bad);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float u[32];
          u_row(U, j0 + e, rank, vec, u);
#pragma unroll
          for (int k = 0; k < 32; ++k) P[k] = fmaf(v[e], u[k], P[k]);
        }
      }
    }
    float pc[32];
    row_projection(P, c_s, part, pc_s, pc, warp, lane);
    for (int64_t b = warp; b < nb; b += kWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      float v[4];
      load_sum4(sp, row, d_in, nb, b, j0, v, bad);
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float acc = 0.0f;
        if (rank > 0) {
          float u[32];
          u_row(U, j0 + e, rank, vec, u);
#pragma unroll
          for (int k = 0; k < 32; ++k) acc = fmaf(pc[k], u[k], acc);
        }
        o[e] = alpha * fmaf(a, v[e], acc);
      }
      store4<T>(out + row * d_in + j0, o);
    }
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

// One CTA per row, capped at a few waves of resident CTAs (rows are then
// taken in a grid-stride loop).
int grid_rows(int64_t d_out) {
  const int64_t cap = (int64_t)kNumSMs * 16;
  return (int)(d_out < cap ? d_out : cap);
}

}  // namespace

cudaError_t launch_whiten_encode_simt(const void* G, gift_dtype dt, int64_t d_out, int64_t d_in, const float* U,
                                      const float* lambda, const float* rho, int rank, uint8_t* codes,
                                      float* scales, uint32_t* err, cudaStream_t s) {
  const int grid = grid_rows(d_out);
  if (dt == GIFT_BF16)
    whiten_encode_simt_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(
        (const __nv_bfloat16*)G, d_out, d_in, U, lambda, rho, rank, codes, scales, err);
  else
    whiten_encode_simt_kernel<float><<<grid, kWarps * 32, 0, s>>>((const float*)G, d_out, d_in, U, lambda, rho,
                                                                   rank, codes, scales, err);
  return cudaGetLastError();
}

cudaError_t launch_whiten_decode_simt(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                                      const float* U, const float* lambda, const float* rho, int rank,
                                      void* G_hat, gift_dtype dt, uint32_t* err, cudaStream_t s) {
  const int grid = grid_rows(d_out);
  if (dt == GIFT_BF16)
    whiten_decode_simt_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(codes, scales, d_out, d_in, U, lambda,
                                                                          rho, rank, (__nv_bfloat16*)G_hat, err);
  else
    whiten_decode_simt_kernel<float><<<grid, kWarps * 32, 0, s>>>(codes, scales, d_out, d_in, U, lambda, rho,
                                                                  rank, (float*)G_hat, err);
  return cudaGetLastError();
}

cudaError_t launch_decode_sum(const uint8_t* const* codes, const float* const* scales, int n_parts, int64_t d_out,
                              int64_t d_in, const float* U, const float* lambda, const float* rho, int rank,
                              float alpha, void* G_hat, gift_dtype dt, uint32_t* err, cudaStream_t s) {
  if (n_parts > kMaxParts) return cudaErrorInvalidValue;
  SumParts sp;
  sp.n = n_parts;
  for (int r = 0; r < n_parts; ++r) {
    sp.codes[r] = codes[r];
    sp.scales[r] = scales[r];
  }
  const int grid = grid_rows(d_out);
  if (dt == GIFT_BF16)
    whiten_decode_sum_simt_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(sp, d_out, d_in, U, lambda, rho, rank,
                                                                              alpha, (__nv_bfloat16*)G_hat, err);
  else
    whiten_decode_sum_simt_kernel<float><<<grid, kWarps * 32, 0, s>>>(sp, d_out, d_in, U, lambda, rho, rank, alpha,
                                                                      (float*)G_hat, err);
  return cudaGetLastError();
}

}  // namespace gift
