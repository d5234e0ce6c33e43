// Shared device helpers for the GIFT sm_100a kernels: number-format
// conversions through the hardware cvt instructions, warp reductions, and
// thin inline-PTX wrappers for mbarriers, TMA and tcgen05.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/gift.h"

#define GIFT_DEV __device__ __forceinline__

namespace gift {

constexpr int kBlock = GIFT_E4M3_BLOCK;   // elements per E4M3 scale
constexpr float kE4M3Max = 448.0f;
constexpr int kNumSMs = 148;

// ---------------------------------------------------------------------------
// Scalar loads of the two gradient storage types as fp32.
// ---------------------------------------------------------------------------
GIFT_DEV float to_f32(float x) { return x; }
GIFT_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

GIFT_DEV void store_from_f32(float* p, float v) { *p = v; }
GIFT_DEV void store_from_f32(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// bf16 pair packed in a 32-bit word -> two floats (exact: bf16 is the top half of fp32)
GIFT_DEV float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
GIFT_DEV float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two floats -> bf16x2 with round-to-nearest-even, x0 in the low half
GIFT_DEV uint32_t pack_bf16x2(float x0, float x1) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  return r;
}

// two floats -> f16x2 with round-to-nearest-even, x0 in the low half
GIFT_DEV uint32_t pack_f16x2(float x0, float x1) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  return r;
}

// Instruction descriptor for kind::f16 with f16 A/B, fp32 D (see umma_idesc_bf16).
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// E4M3 through the hardware converters (round to nearest even, saturating to
// +-448; the sign of zero follows the input).  The first operand of the PTX
// cvt lands in the high byte, so x1 is passed first to put x0 in byte 0.
// ---------------------------------------------------------------------------
GIFT_DEV uint16_t f32x2_to_e4m3x2(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// two E4M3 bytes (byte 0 = first element) -> two floats, exact
GIFT_DEV float2 e4m3x2_to_f32x2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

// E2M1 pair -> one byte (x0 in the low nibble), RNE saturating to +-6
GIFT_DEV uint8_t f32x2_to_e2m1x2(float x0, float x1) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(x1), "f"(x0));
  return (uint8_t)r;
}

// E2M1 pair byte -> two floats, exact
GIFT_DEV float2 e2m1x2_to_f32x2(uint8_t v) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"((uint32_t)v));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

GIFT_DEV float e4m3_to_f32(uint8_t v) { return e4m3x2_to_f32x2((uint16_t)v).x; }

// ---------------------------------------------------------------------------
// NVFP4 block of 16 (abstract of the GIFT paper: NVFP4 as the second format),
// decisions in fp32: tensor scale S_t = amax(W) / (6 * 448); the block's scale
// code sb = E4M3(amax_b / fp32(6 S_t)) (IEEE division, RNE, saturating);
// element codes E2M1(w * fp32(1 / fp32(value(sb) * S_t))).  A block whose
// scale decodes to 0, or whose reciprocal overflows fp32, gets sb = 0 and all
// codes 0.  Codes come back packed two per byte, element 2i in the low nibble.
// ---------------------------------------------------------------------------
constexpr float kNvfp4TensorDiv = 6.0f * 448.0f;

GIFT_DEV float nvfp4_tensor_scale(float amax_t) { return __fdiv_rn(amax_t, kNvfp4TensorDiv); }

GIFT_DEV uint2 nvfp4_block16(const float* w, float S_t, uint8_t* sb_out) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(w[i]));
  const float denom = __fmul_rn(6.0f, S_t);
  const float ratio = denom > 0.0f ? __fdiv_rn(amax, denom) : 0.0f;
  uint8_t sb = (uint8_t)(f32x2_to_e4m3x2(ratio, 0.0f) & 0xFFu);
  const float dq = __fmul_rn(e4m3_to_f32(sb), S_t);
  const float inv = dq > 0.0f ? __frcp_rn(dq) : 0.0f;
  const bool live = dq > 0.0f && !isinf(inv);
  uint32_t c[2] = {0u, 0u};
  if (live) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      c[i >> 2] |= (uint32_t)f32x2_to_e2m1x2(__fmul_rn(w[2 * i], inv), __fmul_rn(w[2 * i + 1], inv)) << (8 * (i & 3));
  } else {
    sb = 0;
  }
  *sb_out = sb;
  return make_uint2(c[0], c[1]);
}

// The 16 values of an NVFP4 block divided by S_t: value(code) * value(sb), exact
// (E2M1 x E4M3 has at most 6 significant bits).
GIFT_DEV void nvfp4_block16_values(uint2 codes, uint8_t sb, float* v) {
  const float s = e4m3_to_f32(sb);
  const uint32_t c[2] = {codes.x, codes.y};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = e2m1x2_to_f32x2((uint8_t)(c[i >> 2] >> (8 * (i & 3))));
    v[2 * i] = f.x * s;
    v[2 * i + 1] = f.y * s;
  }
}

// Reciprocal scale of one E4M3 block: 448/amax (IEEE fp32 division).  A block
// whose amax is 0, or so small that 448/amax overflows fp32, is flushed:
// the function returns 0, and the caller writes scale 0 and codes 0x00.
GIFT_DEV float e4m3_inv_scale(float amax) {
  if (!(amax > 0.0f)) return 0.0f;
  const float inv = __fdiv_rn(kE4M3Max, amax);
  return isinf(inv) ? 0.0f : inv;
}
GIFT_DEV float e4m3_scale(float amax, float inv) { return inv > 0.0f ? __fdiv_rn(amax, kE4M3Max) : 0.0f; }

// ---------------------------------------------------------------------------
// Non-finite inputs.  Block maxima are taken with max.NaN, which returns NaN
// when either operand is NaN (fmaxf would drop it), so a block holding a NaN
// or an infinity has a non-finite maximum; such a block is coded as a
// flushed block (scale 0, codes 0x00) and GIFT_DEV_NONFINITE is reported.
// ---------------------------------------------------------------------------
GIFT_DEV float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
GIFT_DEV bool not_finite(float x) { return !(fabsf(x) <= 3.402823466e38f); }

// OR `bits` into *err from every thread whose `bad` is set.  Not a warp
// collective: callers may have lanes that already left their loops.
GIFT_DEV void report_bits(uint32_t* err, bool bad, uint32_t bits) {
  if (bad && err) atomicOr(err, bits);
}

// ---------------------------------------------------------------------------
// Warp reductions
// ---------------------------------------------------------------------------
GIFT_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
GIFT_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
GIFT_DEV double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Transform coefficients from (lambda, rho), computed in fp64 and rounded once:
//   encode: a = rho^{-1/2}, c_k = (lambda_k + rho)^{-1/2} - rho^{-1/2}
//   decode: a = rho^{+1/2}, c_k = (lambda_k + rho)^{+1/2} - rho^{+1/2}
// Padded with zeros up to 32 coefficients.  rank == 0 gives a = 1, c = 0.
// ---------------------------------------------------------------------------
GIFT_DEV void transform_coeffs(const float* lambda, const float* rho, int rank, bool inverse,
                               float* c_out /* 32 */, float* a_out, int tid) {
  if (rank == 0) {
    if (tid < 32) c_out[tid] = 0.0f;
    if (tid == 0) *a_out = 1.0f;
    return;
  }
  double r = (double)__ldg(rho);
  double a = inverse ? sqrt(r) : 1.0 / sqrt(r);
  if (tid < 32) {
    float c = 0.0f;
    if (tid < rank) {
      double l = (double)__ldg(lambda + tid) + r;
      double v = inverse ? sqrt(l) : 1.0 / sqrt(l);
      c = (float)(v - a);
    }
    c_out[tid] = c;
  }
  if (tid == 0) *a_out = (float)a;
}

// ---------------------------------------------------------------------------
// mbarrier / TMA / tcgen05 wrappers (sm_100a)
// ---------------------------------------------------------------------------
GIFT_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

GIFT_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
GIFT_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
GIFT_DEV void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

GIFT_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
GIFT_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
GIFT_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after `limit` polls (each try_wait itself blocks for
// a hardware-defined interval) and returns false, so no kernel can spin
// forever on a barrier that never completes.
GIFT_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = (1u << 24)) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 2-D tiled TMA load global -> shared, completion on an mbarrier.
GIFT_DEV void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

GIFT_DEV void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// tcgen05: TMEM allocation (whole warp), MMA (one thread), commit, loads.
GIFT_DEV void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
GIFT_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
GIFT_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
GIFT_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
GIFT_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate)
GIFT_DEV void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A is K-major in TMEM, row i
// in lane i, two 16-bit elements per 32-bit column (the lower K in the low half).
GIFT_DEV void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once all prior tcgen05 ops of this thread complete.
GIFT_DEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

GIFT_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 16 consecutive columns: thread i of the warp gets row
// (lane base + i), columns [col, col+16).
GIFT_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 32 lanes x 32 bit, 32 consecutive columns.
GIFT_DEV void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 32 lanes x 32 bit, 8 consecutive columns: thread i of the warp writes row
// (lane base + i), columns [col, col+8).
GIFT_DEV void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
GIFT_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for tcgen05 (sm_100 layout):
// bits 0-13 start>>4, 16-29 leading byte offset>>4, 32-45 stride byte
// offset>>4, 46-47 version = 1, 61-63 swizzle mode (2 = 128-byte swizzle).
GIFT_DEV uint64_t umma_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D.
// a_mn / b_mn: operand is MN-major (1) instead of K-major (0).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                     // D format fp32
         | (1u << 7)                   // A bf16
         | (1u << 10)                  // B bf16
         | ((uint32_t)a_mn << 15)      // A major
         | ((uint32_t)b_mn << 16)      // B major
         | ((uint32_t)(N >> 3) << 17)  // N / 8
         | ((uint32_t)(M >> 4) << 24); // M / 16
}

}  // namespace gift
