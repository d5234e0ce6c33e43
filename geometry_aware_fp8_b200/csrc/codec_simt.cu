// Whitened E4M3 codec on the CUDA cores (fp32 arithmetic), any rank <= 32.
//
// GIFT review page, "What carries the argument": W = G M before the FP8
// quantiser, G_hat = W_hat M^{-1} after it, with
//   M^{-+1} = a I + U diag(c) U^T   (a = rho^{-+1/2},
//                                    c_k = (lambda_k+rho)^{-+1/2} - a).
// One warp owns one row of G; each lane holds four consecutive elements of
// every 128-element block, so one warp step covers exactly one scale block.
// Pass 1 forms P = g U (32 partial dot products per lane, then a butterfly
// reduction); pass 2 forms w = a g + (P o c) U^T, the block maximum with
// five shuffles, and the codes.  This kernel serves fp32 gradients and any
// rank; the tensor-core kernel (codec_tc.cu) serves bf16 gradients.
#include "common.cuh"
#include "internal.h"

namespace gift {
namespace {

constexpr int kWarps = 8;

template <typename T>
GIFT_DEV void load4(const T* p, float (&v)[4]);
template <>
GIFT_DEV void load4<float>(const float* p, float (&v)[4]) {
  float4 f = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
template <>
GIFT_DEV void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
  uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
}
template <typename T>
GIFT_DEV void store4(T* p, const float (&v)[4]);
template <>
GIFT_DEV void store4<float>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
GIFT_DEV void store4<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// Butterfly sum of the 32 per-lane partial projections.
GIFT_DEV void project_row_reduce(float (&P)[32]) {
#pragma unroll
  for (int k = 0; k < 32; ++k) P[k] = warp_sum(P[k]);
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) whiten_encode_simt_kernel(
    const T* __restrict__ G, int64_t d_out, int64_t d_in, const float* __restrict__ U,
    const float* __restrict__ lambda, const float* __restrict__ rho, int rank, uint8_t* __restrict__ codes,
    float* __restrict__ scales) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  transform_coeffs(lambda, rho, rank, false, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int lane = threadIdx.x & 31;
  const int64_t nb = d_in / kBlock;
  for (int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); row < d_out;
       row += (int64_t)gridDim.x * kWarps) {
    const T* g = G + row * d_in;
    float P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = 0.0f;
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t j0 = b * kBlock + lane * 4;
      float v[4];
      load4<T>(g + j0, v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* u = U + (j0 + e) * rank;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < rank) P[k] = fmaf(v[e], __ldg(u + k), P[k]);
      }
    }
    project_row_reduce(P);
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] *= c_s[k];
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t j0 = b * kBlock + lane * 4;
      float v[4];
      load4<T>(g + j0, v);
      float w[4];
      float m = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* u = U + (j0 + e) * rank;
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < rank) acc = fmaf(P[k], __ldg(u + k), acc);
        w[e] = fmaf(a, v[e], acc);
        m = fmaxf(m, fabsf(w[e]));
      }
      m = warp_max(m);
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
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) whiten_decode_simt_kernel(
    const uint8_t* __restrict__ codes, const float* __restrict__ scales, int64_t d_out, int64_t d_in,
    const float* __restrict__ U, const float* __restrict__ lambda, const float* __restrict__ rho, int rank,
    T* __restrict__ out) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  transform_coeffs(lambda, rho, rank, true, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int lane = threadIdx.x & 31;
  const int64_t nb = d_in / kBlock;
  for (int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); row < d_out;
       row += (int64_t)gridDim.x * kWarps) {
    float P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = 0.0f;
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t j0 = b * kBlock + lane * 4;
      const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(codes + row * d_in + j0));
      const float s = __ldg(scales + row * nb + b);
      float2 lo = e4m3x2_to_f32x2((uint16_t)(q & 0xFFFF)), hi = e4m3x2_to_f32x2((uint16_t)(q >> 16));
      float v[4] = {lo.x * s, lo.y * s, hi.x * s, hi.y * s};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* u = U + (j0 + e) * rank;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < rank) P[k] = fmaf(v[e], __ldg(u + k), P[k]);
      }
    }
    project_row_reduce(P);
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] *= c_s[k];
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t j0 = b * kBlock + lane * 4;
      const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(codes + row * d_in + j0));
      const float s = __ldg(scales + row * nb + b);
      float2 lo = e4m3x2_to_f32x2((uint16_t)(q & 0xFFFF)), hi = e4m3x2_to_f32x2((uint16_t)(q >> 16));
      float v[4] = {lo.x * s, lo.y * s, hi.x * s, hi.y * s};
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float* u = U + (j0 + e) * rank;
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < rank) acc = fmaf(P[k], __ldg(u + k), acc);
        o[e] = fmaf(a, v[e], acc);
      }
      store4<T>(out + row * d_in + j0, o);
    }
  }
}

int grid_rows(int64_t d_out) {
  int64_t need = (d_out + kWarps - 1) / kWarps;
  int64_t cap = (int64_t)kNumSMs * 8;
  return (int)(need < cap ? need : cap);
}

}  // namespace

cudaError_t launch_whiten_encode_simt(const void* G, gift_dtype dt, int64_t d_out, int64_t d_in, const float* U,
                                      const float* lambda, const float* rho, int rank, uint8_t* codes,
                                      float* scales, cudaStream_t s) {
  const int grid = grid_rows(d_out);
  if (dt == GIFT_BF16)
    whiten_encode_simt_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(
        (const __nv_bfloat16*)G, d_out, d_in, U, lambda, rho, rank, codes, scales);
  else
    whiten_encode_simt_kernel<float><<<grid, kWarps * 32, 0, s>>>((const float*)G, d_out, d_in, U, lambda, rho,
                                                                   rank, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_whiten_decode_simt(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                                      const float* U, const float* lambda, const float* rho, int rank,
                                      void* G_hat, gift_dtype dt, cudaStream_t s) {
  const int grid = grid_rows(d_out);
  if (dt == GIFT_BF16)
    whiten_decode_simt_kernel<__nv_bfloat16><<<grid, kWarps * 32, 0, s>>>(codes, scales, d_out, d_in, U, lambda,
                                                                          rho, rank, (__nv_bfloat16*)G_hat);
  else
    whiten_decode_simt_kernel<float><<<grid, kWarps * 32, 0, s>>>(codes, scales, d_out, d_in, U, lambda, rho,
                                                                  rank, (float*)G_hat);
  return cudaGetLastError();
}

}  // namespace gift
