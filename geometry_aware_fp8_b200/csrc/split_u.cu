// The U split of the tensor-core codec for many layers in one launch
// (gift_split_u_many).  An implementation format, not part of the method:
// row i of part 0 is [bf16(U_i) | bf16(U_i - bf16(U_i))], row i of part 1 is
// [f16(U_i) | f16((U_i - f16(U_i)) 2^11)], all round to nearest even; these
// are the parts that gift_split_u writes for one layer and that the codec's
// converter warps form in shared memory when no split is given (the GPU
// tests check the three against each other and against the definition).
#include "common.cuh"
#include "internal.h"

namespace gift {
namespace {

constexpr float kLoScaleF16 = 2048.0f;  // 2^11: the f16 lo part's scale
constexpr int kSplitMaxLayers = 512;

struct SplitBatch {
  const float* U[kSplitMaxLayers];
  uint16_t* out[kSplitMaxLayers];
  int64_t d_in[kSplitMaxLayers];
  int block_begin[kSplitMaxLayers];  // first block of each layer, increasing
  int n;
};
static_assert(sizeof(SplitBatch) <= 32760, "kernel parameter space");

// One thread per U row (32 fp32 values).
__global__ void __launch_bounds__(128) split_u_many_kernel(const __grid_constant__ SplitBatch p) {
  int lo = 0, hi = p.n - 1;  // the last layer whose first block is <= blockIdx.x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.block_begin[mid] <= (int)blockIdx.x)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int64_t d_in = p.d_in[lo];
  const int64_t i = (int64_t)((int)blockIdx.x - p.block_begin[lo]) * blockDim.x + threadIdx.x;
  if (i >= d_in) return;
  const float4* src = reinterpret_cast<const float4*>(p.U[lo] + i * 32);
  float u[32];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = __ldg(src + q);
    u[4 * q] = v.x;
    u[4 * q + 1] = v.y;
    u[4 * q + 2] = v.z;
    u[4 * q + 3] = v.w;
  }
  uint32_t bh[16], bl[16], fh[16], fl[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float b0 = __bfloat162float(__float2bfloat16_rn(u[2 * k]));
    const float b1 = __bfloat162float(__float2bfloat16_rn(u[2 * k + 1]));
    bh[k] = pack_bf16x2(b0, b1);
    bl[k] = pack_bf16x2(u[2 * k] - b0, u[2 * k + 1] - b1);
    const float g0 = __half2float(__float2half_rn(u[2 * k]));
    const float g1 = __half2float(__float2half_rn(u[2 * k + 1]));
    fh[k] = pack_f16x2(g0, g1);
    fl[k] = pack_f16x2((u[2 * k] - g0) * kLoScaleF16, (u[2 * k + 1] - g1) * kLoScaleF16);
  }
  uint4* b = reinterpret_cast<uint4*>(p.out[lo] + i * 64);
  uint4* f = reinterpret_cast<uint4*>(p.out[lo] + (d_in + i) * 64);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    b[q] = make_uint4(bh[4 * q], bh[4 * q + 1], bh[4 * q + 2], bh[4 * q + 3]);
    b[4 + q] = make_uint4(bl[4 * q], bl[4 * q + 1], bl[4 * q + 2], bl[4 * q + 3]);
    f[q] = make_uint4(fh[4 * q], fh[4 * q + 1], fh[4 * q + 2], fh[4 * q + 3]);
    f[4 + q] = make_uint4(fl[4 * q], fl[4 * q + 1], fl[4 * q + 2], fl[4 * q + 3]);
  }
}

}  // namespace

cudaError_t launch_split_u_many(const float* const* U, uint16_t* const* U_split, const int64_t* d_in, int n,
                                cudaStream_t s) {
  static thread_local SplitBatch P;
  int l = 0;
  while (l < n) {
    int m = 0;
    int64_t blocks = 0;
    for (; l < n && m < kSplitMaxLayers; ++l) {
      if (d_in[l] <= 0) continue;
      const int64_t nb = (d_in[l] + 127) / 128;
      if (m > 0 && blocks + nb > (int64_t)1 << 30) break;  // the next launch takes it
      P.U[m] = U[l];
      P.out[m] = U_split[l];
      P.d_in[m] = d_in[l];
      P.block_begin[m] = (int)blocks;
      blocks += nb;
      ++m;
    }
    if (m == 0) continue;
    P.n = m;
    split_u_many_kernel<<<(unsigned)blocks, 128, 0, s>>>(P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gift
