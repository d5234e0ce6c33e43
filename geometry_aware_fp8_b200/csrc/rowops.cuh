// Row-wise helpers shared by the CUDA-core kernels that walk a row of G in
// 128-element blocks, four consecutive elements per lane: vector loads and
// stores of the elements, rows of U, and the transpose reduction that hands
// lane k the warp's sum of coefficient k.
#pragma once

#include "common.cuh"

namespace gift {
namespace {

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

// Row j of U (rank values, zero beyond): 16-byte loads when the rows are
// 16-byte aligned (U itself is: the C ABI checks it; rank % 4 == 0 keeps
// every row so).
GIFT_DEV void u_row(const float* __restrict__ U, int64_t j, int rank, bool vec, float (&u)[32]) {
  const float* p = U + j * rank;
  if (vec) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (4 * q < rank) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(p) + q);
        u[4 * q] = f.x; u[4 * q + 1] = f.y; u[4 * q + 2] = f.z; u[4 * q + 3] = f.w;
      } else {
        u[4 * q] = u[4 * q + 1] = u[4 * q + 2] = u[4 * q + 3] = 0.0f;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) u[k] = k < rank ? __ldg(p + k) : 0.0f;
  }
}

// Sum of v[k] over the 32 lanes, delivered to lane k: at each of five steps a
// lane keeps the half of its values whose index bit matches its lane bit and
// adds the partner's copy of that half (31 shuffles in all).
GIFT_DEV float reduce_transpose32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

}  // namespace
}  // namespace gift
