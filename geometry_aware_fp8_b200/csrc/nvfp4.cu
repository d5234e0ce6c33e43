// NVFP4 codec for Euclidean layers (M = I): E2M1 codes two per byte, E4M3
// scales per 16 elements, one fp32 tensor scale (abstract of the GIFT paper:
// NVFP4 is the second low-precision format the method is applied to).
//
// The tensor scale needs amax over the whole tensor before any block can be
// coded, so encoding is two streaming passes: nvfp4_amax_kernel folds |G| into
// one word (atomicMax on the bits of a non-negative float, which orders like
// the float), nvfp4_quant_kernel codes every block of 16 from it, and
// nvfp4_finalize_kernel turns the word into S_t = amax / (6 * 448) in place.
// One thread owns one block of 16: 32 (bf16) or 64 (fp32) contiguous bytes in,
// 8 bytes of codes and 1 scale byte out.  Bound by HBM.
#include "common.cuh"
#include "internal.h"

namespace gift {
namespace {

GIFT_DEV void load16(const __nv_bfloat16* p, float* v) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  const uint4 a = __ldcs(q), b = __ldcs(q + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16lo(w[i]);
    v[2 * i + 1] = bf16hi(w[i]);
  }
}
GIFT_DEV void load16(const float* p, float* v) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 f = __ldcs(q + i);
    v[4 * i] = f.x;
    v[4 * i + 1] = f.y;
    v[4 * i + 2] = f.z;
    v[4 * i + 3] = f.w;
  }
}
GIFT_DEV void store16(__nv_bfloat16* p, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  uint4* q = reinterpret_cast<uint4*>(p);
  __stcs(q, make_uint4(w[0], w[1], w[2], w[3]));
  __stcs(q + 1, make_uint4(w[4], w[5], w[6], w[7]));
}
GIFT_DEV void store16(float* p, const float* v) {
  float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) __stcs(q + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
}

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads) nvfp4_amax_kernel(const T* __restrict__ G, int64_t n_blocks,
                                                              uint32_t* __restrict__ amax_bits) {
  float m = 0.0f;
  for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < n_blocks; b += (int64_t)gridDim.x * kThreads) {
    float v[16];
    load16(G + b * 16, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmax_nan(m, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
  // a NaN maximum has the largest bit pattern of all, so it survives the max
  if ((threadIdx.x & 31) == 0 && (m > 0.0f || m != m)) atomicMax(amax_bits, __float_as_uint(m));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) nvfp4_quant_kernel(const T* __restrict__ G, int64_t n_blocks,
                                                               const uint32_t* __restrict__ amax_bits,
                                                               uint2* __restrict__ codes, uint8_t* __restrict__ sb) {
  const float S_t = nvfp4_tensor_scale(__uint_as_float(__ldg(amax_bits)));
  for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < n_blocks; b += (int64_t)gridDim.x * kThreads) {
    float v[16];
    load16(G + b * 16, v);
    uint8_t s;
    const uint2 c = nvfp4_block16(v, S_t, &s);
    __stcs(codes + b, c);
    sb[b] = s;
  }
}

// amax bits -> S_t, in place (one thread); a non-finite amax(W) is reported
__global__ void nvfp4_finalize_kernel(float* tensor_scale, uint32_t* err) {
  const float amax = __uint_as_float(*reinterpret_cast<const uint32_t*>(tensor_scale));
  *tensor_scale = nvfp4_tensor_scale(amax);
  if (err && not_finite(amax)) atomicOr(err, GIFT_DEV_NONFINITE);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) nvfp4_decode_kernel(const uint2* __restrict__ codes,
                                                                const uint8_t* __restrict__ sb,
                                                                const float* __restrict__ tensor_scale,
                                                                int64_t n_blocks, T* __restrict__ out, uint32_t* err) {
  const float S_t = __ldg(tensor_scale);
  if (blockIdx.x == 0 && threadIdx.x == 0 && err && not_finite(S_t)) atomicOr(err, GIFT_DEV_NONFINITE);
  for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < n_blocks; b += (int64_t)gridDim.x * kThreads) {
    float v[16];
    nvfp4_block16_values(__ldcs(codes + b), sb[b], v);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], S_t);
    store16(out + b * 16, v);
  }
}

int grid_for(int64_t n_blocks) {
  const int64_t need = (n_blocks + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)kNumSMs * 8;
  return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

cudaError_t launch_nvfp4_amax(const void* G, gift_dtype dt, int64_t n_blocks, float* tensor_scale, cudaStream_t s) {
  const int g = grid_for(n_blocks);
  uint32_t* bits = reinterpret_cast<uint32_t*>(tensor_scale);
  if (dt == GIFT_BF16)
    nvfp4_amax_kernel<<<g, kThreads, 0, s>>>((const __nv_bfloat16*)G, n_blocks, bits);
  else
    nvfp4_amax_kernel<<<g, kThreads, 0, s>>>((const float*)G, n_blocks, bits);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_quant(const void* G, gift_dtype dt, int64_t n_blocks, const float* tensor_scale,
                               uint8_t* codes, uint8_t* sb, cudaStream_t s) {
  const int g = grid_for(n_blocks);
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(tensor_scale);
  if (dt == GIFT_BF16)
    nvfp4_quant_kernel<<<g, kThreads, 0, s>>>((const __nv_bfloat16*)G, n_blocks, bits, (uint2*)codes, sb);
  else
    nvfp4_quant_kernel<<<g, kThreads, 0, s>>>((const float*)G, n_blocks, bits, (uint2*)codes, sb);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_finalize(float* tensor_scale, uint32_t* err, cudaStream_t s) {
  nvfp4_finalize_kernel<<<1, 1, 0, s>>>(tensor_scale, err);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_decode(const uint8_t* codes, const uint8_t* sb, const float* tensor_scale, int64_t n_blocks,
                                void* out, gift_dtype dt, uint32_t* err, cudaStream_t s) {
  const int g = grid_for(n_blocks);
  if (dt == GIFT_BF16)
    nvfp4_decode_kernel<<<g, kThreads, 0, s>>>((const uint2*)codes, sb, tensor_scale, n_blocks, (__nv_bfloat16*)out,
                                               err);
  else
    nvfp4_decode_kernel<<<g, kThreads, 0, s>>>((const uint2*)codes, sb, tensor_scale, n_blocks, (float*)out, err);
  return cudaGetLastError();
}

}  // namespace gift
