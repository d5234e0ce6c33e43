// Euclidean per-block E4M3 codec (M = I): the comparison arm of the GIFT
// round-trip study (Tables I-II) and the path of every layer that the
// selective deployment leaves unwhitened (section V.C, Fig. 4).
//
// Pure streaming work, bound by HBM: 2 (bf16) or 4 (fp32) bytes in, 1 byte
// plus 4/128 bytes out per element.  Eight threads own one 128-element block,
// 16 elements each, the block maximum is three xor-shuffles, and the grid is a
// multiple of the SM count that strides over all blocks.  A thread's elements
// are pieces of 16 bytes of the gradient (8 bf16 or 4 fp32) spaced by the
// eight threads' pieces, so each warp-wide 16-byte load or store of G or
// G_hat covers whole 32-byte sectors (a thread owning 16 consecutive bf16
// values would write every sector in two halves, from two instructions).
#include "common.cuh"
#include "internal.h"

namespace gift {
namespace {

// The 16 elements of thread `sub` in a 128-element block: kPieces pieces of
// kPiece elements (16 bytes of T); piece k starts at element
// kPiece sub + 8 kPiece k, and holds v[kPiece k .. kPiece (k + 1) - 1].
// The codes of those elements (1 byte each) sit at the same offsets.
template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kPiece = 8;
  struct Raw {
    uint4 a, b;
  };
  static GIFT_DEV Raw load_raw(const __nv_bfloat16* blk, int sub) {
    return Raw{__ldcs(reinterpret_cast<const uint4*>(blk + 8 * sub)),
               __ldcs(reinterpret_cast<const uint4*>(blk + 64 + 8 * sub))};
  }
  static GIFT_DEV void unpack(const Raw& r, float (&v)[16]) {
    const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16lo(w[i]);
      v[2 * i + 1] = bf16hi(w[i]);
    }
  }
  static GIFT_DEV void load(const __nv_bfloat16* blk, int sub, float (&v)[16]) { unpack(load_raw(blk, sub), v); }
  static GIFT_DEV void store(__nv_bfloat16* blk, int sub, const float (&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    __stcs(reinterpret_cast<uint4*>(blk + 8 * sub), make_uint4(w[0], w[1], w[2], w[3]));
    __stcs(reinterpret_cast<uint4*>(blk + 64 + 8 * sub), make_uint4(w[4], w[5], w[6], w[7]));
  }
  // codes word i (4 codes) holds v[4 i .. 4 i + 3]
  static GIFT_DEV void store_codes(uint8_t* blk, int sub, uint4 q) {
    __stcs(reinterpret_cast<uint2*>(blk + 8 * sub), make_uint2(q.x, q.y));
    __stcs(reinterpret_cast<uint2*>(blk + 64 + 8 * sub), make_uint2(q.z, q.w));
  }
  static GIFT_DEV uint4 load_codes(const uint8_t* blk, int sub) {
    const uint2 a = __ldcs(reinterpret_cast<const uint2*>(blk + 8 * sub));
    const uint2 b = __ldcs(reinterpret_cast<const uint2*>(blk + 64 + 8 * sub));
    return make_uint4(a.x, a.y, b.x, b.y);
  }
};

template <>
struct Vec16<float> {
  static constexpr int kPiece = 4;
  struct Raw {
    float4 f[4];
  };
  static GIFT_DEV Raw load_raw(const float* blk, int sub) {
    Raw r;
#pragma unroll
    for (int k = 0; k < 4; ++k) r.f[k] = __ldcs(reinterpret_cast<const float4*>(blk + 4 * sub + 32 * k));
    return r;
  }
  static GIFT_DEV void unpack(const Raw& r, float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[4 * k] = r.f[k].x;
      v[4 * k + 1] = r.f[k].y;
      v[4 * k + 2] = r.f[k].z;
      v[4 * k + 3] = r.f[k].w;
    }
  }
  static GIFT_DEV void load(const float* blk, int sub, float (&v)[16]) { unpack(load_raw(blk, sub), v); }
  static GIFT_DEV void store(float* blk, int sub, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      __stcs(reinterpret_cast<float4*>(blk + 4 * sub + 32 * k), make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]));
  }
  static GIFT_DEV void store_codes(uint8_t* blk, int sub, uint4 q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) __stcs(reinterpret_cast<unsigned int*>(blk + 4 * sub + 32 * k), w[k]);
  }
  static GIFT_DEV uint4 load_codes(const uint8_t* blk, int sub) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = __ldcs(reinterpret_cast<const unsigned int*>(blk + 4 * sub + 32 * k));
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// Quantise 16 values of one block given its reciprocal scale; returns the codes packed in a uint4.
GIFT_DEV uint4 quantize16(const float (&v)[16], float inv) {
  uint32_t w[4];
  if (inv > 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv));
      uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv));
      w[i] = lo | (hi << 16);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = 0u;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Dequantise the 16 codes of a thread (word i = codes of v[4 i .. 4 i + 3]).
GIFT_DEV void dequant16(uint4 q, float s, float (&v)[16]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = e4m3x2_to_f32x2((uint16_t)(w[i] & 0xFFFF));
    const float2 c = e4m3x2_to_f32x2((uint16_t)(w[i] >> 16));
    v[4 * i] = a.x * s;
    v[4 * i + 1] = a.y * s;
    v[4 * i + 2] = c.x * s;
    v[4 * i + 3] = c.y * s;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) euclid_encode_kernel(const T* __restrict__ G, uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales, int64_t n_blocks,
                                                            uint32_t* err) {
  const int sub = threadIdx.x & 7;
  bool bad = false;
  const int64_t groups_per_grid = (int64_t)gridDim.x * (blockDim.x >> 3);
  // the loop bound is the warp's first block, so all 32 lanes take every
  // iteration together and meet at the shuffles; lanes past the end idle
  for (int64_t base = (int64_t)blockIdx.x * (blockDim.x >> 3) + ((threadIdx.x >> 5) << 2); base < n_blocks;
       base += groups_per_grid) {
    const int64_t b = base + ((threadIdx.x & 31) >> 3);
    const bool act = b < n_blocks;
    // lanes past the end load (and discard) the warp's first block: no branch before the shuffles
    const int64_t e0 = (act ? b : base) * kBlock;  // the block's first element
    float v[16];
    Vec16<T>::load(G + e0, sub, v);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmax_nan(m, fabsf(v[i]));
    m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
    m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, 4));
    if (!act) continue;
    bad |= not_finite(m);
    const float inv = e4m3_inv_scale(m);
    Vec16<T>::store_codes(codes + e0, sub, quantize16(v, inv));
    if (sub == 0) scales[b] = e4m3_scale(m, inv);
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

template <typename T>
__global__ void __launch_bounds__(256) euclid_decode_kernel(const uint8_t* __restrict__ codes,
                                                            const float* __restrict__ scales, T* __restrict__ out,
                                                            int64_t n_blocks, uint32_t* err) {
  const int sub = threadIdx.x & 7;
  bool bad = false;
  const int64_t groups_per_grid = (int64_t)gridDim.x * (blockDim.x >> 3);
  for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 3) + (threadIdx.x >> 3); b < n_blocks;
       b += groups_per_grid) {
    const int64_t e0 = b * kBlock;  // the block's first element
    const uint4 q = Vec16<T>::load_codes(codes + e0, sub);
    const float s = __ldg(scales + b);
    bad |= not_finite(s);
    float v[16];
    dequant16(q, s, v);
    Vec16<T>::store(out + e0, sub, v);
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

// Grouped form: many layers in one launch.  A block index b of the
// concatenated layers is mapped to its layer through the prefix sums of the
// layers' block counts (kept in shared memory): the encoder searches once per
// thread and stream and then advances (each stream's block index only grows),
// the decoder searches per block.
constexpr int kGroupMax = 64;

struct EuclidGroup {
  const void* src[kGroupMax];   // encode: G; decode: codes
  void* dst[kGroupMax];         // encode: codes; decode: G_hat
  float* scales[kGroupMax];
  int64_t prefix[kGroupMax + 1];  // prefix[i] = first block of layer i
  int n;
  uint32_t* err;                  // device status word (nullable)
};

GIFT_DEV int find_layer(const int64_t* pre, int n, int64_t b) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}
// the layer of block b, given the layer of an earlier block of this thread
GIFT_DEV int advance_layer(const int64_t* pre, int n, int l, int64_t b) {
  while (l + 1 < n && b >= pre[l + 1]) ++l;
  return l;
}

// kEncU blocks per thread group per iteration: every block's loads are issued
// (as raw 16-byte words) before any is used, so each thread keeps kEncU x 32
// bytes (bf16) in flight.  Stream u of a thread group takes blocks
// first + u G, first + (u + kEncU) G, ... and keeps its own layer cursor.
constexpr int kEncU = 4;
template <typename T>
__global__ void __launch_bounds__(256) euclid_encode_group_kernel(const __grid_constant__ EuclidGroup g) {
  __shared__ int64_t pre[kGroupMax + 1];
  for (int i = threadIdx.x; i <= g.n; i += blockDim.x) pre[i] = g.prefix[i];
  __syncthreads();
  const int sub = threadIdx.x & 7;
  const int64_t total = pre[g.n];
  const int64_t G = (int64_t)gridDim.x * (blockDim.x >> 3);
  // per warp: blocks base .. base + 3 (the loop bound is the warp's first
  // block, so all 32 lanes take every iteration together and meet at the
  // shuffles; lanes past the end idle)
  const int64_t wfirst = (int64_t)blockIdx.x * (blockDim.x >> 3) + ((threadIdx.x >> 5) << 2);
  const int64_t first = wfirst + ((threadIdx.x & 31) >> 3);
  int lc[kEncU];
#pragma unroll
  for (int u = 0; u < kEncU; ++u) lc[u] = first + u * G < total ? find_layer(pre, g.n, first + u * G) : 0;
  bool bad = false;
  for (int64_t base = wfirst; base < total; base += kEncU * G) {
    const bool has0 = base + ((threadIdx.x & 31) >> 3) < total;
    // lanes past the end work on the warp's first block and discard it: no
    // branch before the shuffles
    const int64_t b0 = has0 ? base + ((threadIdx.x & 31) >> 3) : base;
    int64_t e[kEncU];
    bool has[kEncU];
    typename Vec16<T>::Raw raw[kEncU];
    // stream 0 follows b0 even on idle lanes (b0 only grows), so its cursor
    // always names the layer of a block that exists
    lc[0] = advance_layer(pre, g.n, lc[0], b0);
#pragma unroll
    for (int u = 0; u < kEncU; ++u) {
      const int64_t b = b0 + u * G;
      has[u] = has0 && b < total;
      if (u > 0 && has[u]) lc[u] = advance_layer(pre, g.n, lc[u], b);
      // a stream past the end loads (and discards) stream 0's block
      const int l = has[u] ? lc[u] : lc[0];
      e[u] = ((has[u] ? b : b0) - pre[l]) * kBlock;  // the block's first element
      raw[u] = Vec16<T>::load_raw((const T*)g.src[l] + e[u], sub);
    }
#pragma unroll
    for (int u = 0; u < kEncU; ++u) {
      float v[16];
      Vec16<T>::unpack(raw[u], v);
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmax_nan(m, fabsf(v[i]));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (!has[u]) continue;  // after the shuffles
      const int l = lc[u];
      bad |= not_finite(m);
      const float inv = e4m3_inv_scale(m);
      Vec16<T>::store_codes((uint8_t*)g.dst[l] + e[u], sub, quantize16(v, inv));
      if (sub == 0) g.scales[l][e[u] / kBlock] = e4m3_scale(m, inv);
    }
  }
  report_bits(g.err, bad, GIFT_DEV_NONFINITE);
}

template <typename T>
__global__ void __launch_bounds__(256) euclid_decode_group_kernel(const __grid_constant__ EuclidGroup g) {
  __shared__ int64_t pre[kGroupMax + 1];
  for (int i = threadIdx.x; i <= g.n; i += blockDim.x) pre[i] = g.prefix[i];
  __syncthreads();
  const int sub = threadIdx.x & 7;
  const int64_t total = pre[g.n];
  const int64_t G = (int64_t)gridDim.x * (blockDim.x >> 3);
  bool bad = false;
  // kDecU blocks per thread group per iteration, all loads issued first (6
  // measured faster than 4 or 8 on the stack)
  constexpr int kDecU = 6;
  for (int64_t b0 = (int64_t)blockIdx.x * (blockDim.x >> 3) + (threadIdx.x >> 3); b0 < total; b0 += kDecU * G) {
    uint4 qv[kDecU];
    float sv[kDecU];
    int lv[kDecU];
    int64_t lbv[kDecU];
#pragma unroll
    for (int u = 0; u < kDecU; ++u) {
      const int64_t b = b0 + u * G;
      qv[u] = make_uint4(0, 0, 0, 0);
      sv[u] = 0.0f;
      lv[u] = 0;
      lbv[u] = 0;
      if (b < total) {
        lv[u] = find_layer(pre, g.n, b);
        lbv[u] = b - pre[lv[u]];
        qv[u] = Vec16<T>::load_codes((const uint8_t*)g.src[lv[u]] + lbv[u] * kBlock, sub);
        sv[u] = __ldg(g.scales[lv[u]] + lbv[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kDecU; ++u) {
      if (b0 + u * G >= total) continue;
      bad |= not_finite(sv[u]);
      float v[16];
      dequant16(qv[u], sv[u], v);
      Vec16<T>::store((T*)g.dst[lv[u]] + lbv[u] * kBlock, sub, v);
    }
  }
  report_bits(g.err, bad, GIFT_DEV_NONFINITE);
}

inline int grid_for(int64_t n_blocks) {
  // 8 blocks per 256-thread CTA; up to 8 resident CTAs per SM.
  int64_t need = (n_blocks + 31) / 32;  // four blocks of work per group
  int64_t cap = (int64_t)kNumSMs * 8;
  if (need < 1) need = 1;
  return (int)(need < cap ? need : cap);
}

}  // namespace

cudaError_t launch_euclid_encode(const void* G, gift_dtype dt, int64_t n_blocks, uint8_t* codes, float* scales,
                                 uint32_t* err, cudaStream_t s) {
  if (n_blocks == 0) return cudaSuccess;
  const int grid = grid_for(n_blocks);
  if (dt == GIFT_BF16)
    euclid_encode_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)G, codes, scales, n_blocks, err);
  else
    euclid_encode_kernel<float><<<grid, 256, 0, s>>>((const float*)G, codes, scales, n_blocks, err);
  return cudaGetLastError();
}

cudaError_t launch_euclid_decode(const uint8_t* codes, const float* scales, int64_t n_blocks, void* G_hat,
                                 gift_dtype dt, uint32_t* err, cudaStream_t s) {
  if (n_blocks == 0) return cudaSuccess;
  const int grid = grid_for(n_blocks);
  if (dt == GIFT_BF16)
    euclid_decode_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(codes, scales, (__nv_bfloat16*)G_hat, n_blocks, err);
  else
    euclid_decode_kernel<float><<<grid, 256, 0, s>>>(codes, scales, (float*)G_hat, n_blocks, err);
  return cudaGetLastError();
}

// Grid of a grouped launch: as many CTAs as stay resident (one wave), found once
// per kernel with the occupancy calculator.
// slot: one cached count per kernel (the kernels share one pointer type).
template <typename K>
int group_grid(K kernel, int slot, int64_t n_blocks) {
  static int resident[4] = {0, 0, 0, 0};
  if (resident[slot] == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 4;
    resident[slot] = per_sm * kNumSMs;
  }
  const int res = resident[slot];
  int64_t need = (n_blocks + 31) / 32;
  if (need < 1) need = 1;
  return (int)(need < res ? need : res);
}

cudaError_t launch_euclid_group(const EuclidLayer* layers, int n, gift_dtype dt, bool encode, uint32_t* err,
                               cudaStream_t s) {
  for (int base = 0; base < n; base += kGroupMax) {
    const int cnt = n - base < kGroupMax ? n - base : kGroupMax;
    EuclidGroup g;
    g.n = cnt;
    g.err = err;
    int64_t tot = 0;
    for (int i = 0; i < cnt; ++i) {
      const EuclidLayer& L = layers[base + i];
      g.src[i] = L.src;
      g.dst[i] = L.dst;
      g.scales[i] = L.scales;
      g.prefix[i] = tot;
      tot += L.n_blocks;
    }
    g.prefix[cnt] = tot;
    if (tot == 0) continue;
    if (encode) {
      if (dt == GIFT_BF16) {
        auto k = euclid_encode_group_kernel<__nv_bfloat16>;
        k<<<group_grid(k, 0, tot), 256, 0, s>>>(g);
      } else {
        auto k = euclid_encode_group_kernel<float>;
        k<<<group_grid(k, 1, tot), 256, 0, s>>>(g);
      }
    } else {
      if (dt == GIFT_BF16) {
        auto k = euclid_decode_group_kernel<__nv_bfloat16>;
        k<<<group_grid(k, 2, tot), 256, 0, s>>>(g);
      } else {
        auto k = euclid_decode_group_kernel<float>;
        k<<<group_grid(k, 3, tot), 256, 0, s>>>(g);
      }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gift
