// One-step round-trip error of the codec (Tables I-II of the GIFT paper:
// relative reconstruction error of the FP8 round trip against the
// full-precision gradient):  ||G_hat - G||_F / ||G||_F, and the same error in
// whitened coordinates, ||(G_hat - G) M||_F / ||G M||_F.
//
// Two launches with a fixed reduction tree, so the result is bit-identical
// from run to run: per-CTA fp64 partial sums (each thread strides over
// 8-element vectors in a fixed order), then one CTA adds the partials in
// index order.  The grid size depends only on the element count.
#include "common.cuh"
#include "internal.h"
#include "rowops.cuh"

namespace gift {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxParts = 1184;  // 8 CTAs per SM

inline int parts_for(int64_t n_elems) {
  int64_t vecs = n_elems / 8;
  int64_t need = (vecs + kThreads * 4 - 1) / (kThreads * 4);
  if (need < 1) need = 1;
  return (int)(need < kMaxParts ? need : kMaxParts);
}

template <typename T>
GIFT_DEV void load8(const T* p, float (&v)[8]);
template <>
GIFT_DEV void load8<float>(const float* p, float (&v)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p)), b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
GIFT_DEV void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 a = __ldcs(reinterpret_cast<const uint4*>(p));
  uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16lo(w[i]);
    v[2 * i + 1] = bf16hi(w[i]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) err_partial_kernel(const T* __restrict__ G, const T* __restrict__ Gh,
                                                               int64_t n_vecs, double* __restrict__ part) {
  double dd = 0.0, gg = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n_vecs; i += (int64_t)gridDim.x * kThreads) {
    float g[8], h[8];
    load8<T>(G + i * 8, g);
    load8<T>(Gh + i * 8, h);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      double gd = (double)g[e];
      double df = (double)h[e] - gd;  // exact in fp64
      dd = fma(df, df, dd);
      gg = fma(gd, gd, gg);
    }
  }
  __shared__ double s_dd[kThreads], s_gg[kThreads];
  s_dd[threadIdx.x] = dd;
  s_gg[threadIdx.x] = gg;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      s_dd[threadIdx.x] += s_dd[threadIdx.x + o];
      s_gg[threadIdx.x] += s_gg[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = s_dd[0];
    part[2 * blockIdx.x + 1] = s_gg[0];
  }
}

__global__ void __launch_bounds__(kThreads) err_final_kernel(const double* __restrict__ part, int nparts,
                                                             double* __restrict__ out) {
  __shared__ double s_dd[kThreads], s_gg[kThreads];
  double dd = 0.0, gg = 0.0;
  for (int i = threadIdx.x; i < nparts; i += kThreads) {
    dd += part[2 * i];
    gg += part[2 * i + 1];
  }
  s_dd[threadIdx.x] = dd;
  s_gg[threadIdx.x] = gg;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      s_dd[threadIdx.x] += s_dd[threadIdx.x + o];
      s_gg[threadIdx.x] += s_gg[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[0] = sqrt(s_dd[0]) / sqrt(s_gg[0]);
    out[1] = s_dd[0];
    out[2] = s_gg[0];
  }
}

// ---- error in whitened coordinates ----
// Per row of G (x = g) and of the difference (y = g_hat - g), with the
// codec's transform M = a I + U diag(c) U^T (a = rho^{-1/2}, c_k =
// (lambda_k + rho)^{-1/2} - a): p = x U, then (x M)_j = a x_j + sum_k p_k c_k
// U_jk, squared and summed in fp64.  One CTA owns a row (grid-stride); its
// warps take the row's 128-element blocks in turn and a lane holds four
// consecutive elements; p is reduced across the lanes by transpose and across
// the warps in warp order, so the partial of every CTA is deterministic.
constexpr int kRowWarps = 8;

inline int white_parts(int64_t d_out) { return (int)(d_out < kMaxParts ? d_out : kMaxParts); }

template <typename T>
__global__ void __launch_bounds__(kRowWarps * 32) white_partial_kernel(
    const T* __restrict__ G, const T* __restrict__ Gh, int64_t d_out, int64_t d_in, const float* __restrict__ U,
    const float* __restrict__ lambda, const float* __restrict__ rho, int rank, double* __restrict__ part) {
  __shared__ float c_s[32];
  __shared__ float a_s;
  __shared__ float pg_part[kRowWarps][32], py_part[kRowWarps][32];
  __shared__ float pg_s[32], py_s[32];
  transform_coeffs(lambda, rho, rank, false, c_s, &a_s, threadIdx.x);
  __syncthreads();
  const float a = a_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = (rank & 3) == 0;
  const int64_t nb = d_in / kBlock;
  double yy = 0.0, gg = 0.0;
  for (int64_t row = blockIdx.x; row < d_out; row += gridDim.x) {
    const T* g = G + row * d_in;
    const T* h = Gh + row * d_in;
    float pg[32], py[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) pg[k] = py[k] = 0.0f;
    for (int64_t b = warp; b < nb; b += kRowWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      float x[4], z[4];
      load4<T>(g + j0, x);
      load4<T>(h + j0, z);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
        const float y = z[e] - x[e];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          pg[k] = fmaf(x[e], u[k], pg[k]);
          py[k] = fmaf(y, u[k], py[k]);
        }
      }
    }
    pg_part[warp][lane] = reduce_transpose32(pg, lane);
    py_part[warp][lane] = reduce_transpose32(py, lane);
    __syncthreads();
    if (warp == 0) {
      float sg = 0.0f, sy = 0.0f;
#pragma unroll
      for (int w = 0; w < kRowWarps; ++w) {
        sg += pg_part[w][lane];
        sy += py_part[w][lane];
      }
      pg_s[lane] = sg * c_s[lane];
      py_s[lane] = sy * c_s[lane];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      pg[k] = pg_s[k];
      py[k] = py_s[k];
    }
    for (int64_t b = warp; b < nb; b += kRowWarps) {
      const int64_t j0 = b * kBlock + lane * 4;
      float x[4], z[4];
      load4<T>(g + j0, x);
      load4<T>(h + j0, z);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float u[32];
        u_row(U, j0 + e, rank, vec, u);
        float wg = 0.0f, wy = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          wg = fmaf(pg[k], u[k], wg);
          wy = fmaf(py[k], u[k], wy);
        }
        wg = fmaf(a, x[e], wg);
        wy = fmaf(a, z[e] - x[e], wy);
        gg = fma((double)wg, (double)wg, gg);
        yy = fma((double)wy, (double)wy, yy);
      }
    }
    __syncthreads();  // the exchange arrays are reused by the next row
  }
  __shared__ double s_yy[kRowWarps * 32], s_gg[kRowWarps * 32];
  s_yy[threadIdx.x] = yy;
  s_gg[threadIdx.x] = gg;
  __syncthreads();
  for (int o = kRowWarps * 16; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      s_yy[threadIdx.x] += s_yy[threadIdx.x + o];
      s_gg[threadIdx.x] += s_gg[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = s_yy[0];
    part[2 * blockIdx.x + 1] = s_gg[0];
  }
}

}  // namespace

size_t error_ws_bytes(int64_t n_elems) { return (size_t)parts_for(n_elems) * 2 * sizeof(double); }

cudaError_t launch_roundtrip_error(const void* G, const void* G_hat, gift_dtype dt, int64_t n_elems, double* out,
                                   void* ws, cudaStream_t s) {
  const int parts = parts_for(n_elems);
  double* part = (double*)ws;
  const int64_t n_vecs = n_elems / 8;
  if (dt == GIFT_BF16)
    err_partial_kernel<__nv_bfloat16><<<parts, kThreads, 0, s>>>((const __nv_bfloat16*)G,
                                                                 (const __nv_bfloat16*)G_hat, n_vecs, part);
  else
    err_partial_kernel<float><<<parts, kThreads, 0, s>>>((const float*)G, (const float*)G_hat, n_vecs, part);
  err_final_kernel<<<1, kThreads, 0, s>>>(part, parts, out);
  return cudaGetLastError();
}

size_t whitened_error_ws_bytes(int64_t d_out) { return (size_t)white_parts(d_out) * 2 * sizeof(double); }

cudaError_t launch_whitened_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out, int64_t d_in,
                                  const float* U, const float* lambda, const float* rho, int rank, double* out,
                                  void* ws, cudaStream_t s) {
  const int parts = white_parts(d_out);
  double* part = (double*)ws;
  if (dt == GIFT_BF16)
    white_partial_kernel<__nv_bfloat16><<<parts, kRowWarps * 32, 0, s>>>(
        (const __nv_bfloat16*)G, (const __nv_bfloat16*)G_hat, d_out, d_in, U, lambda, rho, rank, part);
  else
    white_partial_kernel<float><<<parts, kRowWarps * 32, 0, s>>>((const float*)G, (const float*)G_hat, d_out, d_in,
                                                                 U, lambda, rho, rank, part);
  err_final_kernel<<<1, kThreads, 0, s>>>(part, parts, out);
  return cudaGetLastError();
}

}  // namespace gift
