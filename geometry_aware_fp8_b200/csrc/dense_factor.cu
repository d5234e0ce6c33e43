// Dense input-side transforms for the variants GIFT is simplified from
// (review page, "What carries the argument"; Fig. 2 caption: full-rank
// input-side whitening; section IV.A, Eq. (14): the Cholesky form L_A^{-T}).
// From A = X^T X / N (d x d, fp32), all arithmetic in fp64:
//   Cholesky:     A = L L^T,  M = L^{-T},   M^{-1} = L^T       (upper triangular)
//   full rank:    M = A^{-1/2},             M^{-1} = A^{1/2}   (symmetric)
// Outputs M and M^{-1} in fp32, M as three bf16 parts (hi, mid, lo) and
// M^{-1} as a bf16 hi/lo pair: the operands of the dense tensor-core codec
// (dense_tc.cu).
//
// Cholesky is blocked by 64: per block column p, one CTA factors the diagonal
// block and inverts its factor (fp64, shared memory), the blocks below are
// solved against it, and the trailing lower triangle is updated
// (A_ij -= L_ip L_jp^T, one CTA per 64 x 64 block).  L^{-1} is formed block
// row by block row: X_ii = L_ii^{-1}, X_ij = -L_ii^{-1} sum_{k=j}^{i-1} L_ik X_kj.
// The inverse square root is the coupled Newton-Schulz iteration (Higham,
// "Functions of Matrices", section 6.7): Y_0 = A / c, Z_0 = I with c = ||A||_F,
//   T = (3 I - Z Y) / 2,  Y <- Y T,  Z <- T Z,
// Y -> (A/c)^{1/2}, Z -> (A/c)^{-1/2}; once a step with max |T - I| below
// 1e-8 has been applied (the iteration converges quadratically, so the
// result is then at rounding level), later iterations copy their operands
// through unchanged.
// Products are a register-tiled fp64 GEMM on the CUDA cores (128 x 128 tile,
// 8 x 8 outputs per thread).
#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {
namespace {

constexpr int kNB = 64;          // Cholesky / inverse block
constexpr int kFT = 256;         // threads of the block kernels
constexpr int kBlockSmem = 2 * kNB * (kNB + 1) * 8;  // dynamic shared memory of the block kernels
constexpr double kNsTol = 1e-8;  // Newton-Schulz: max |T - I| of the last applied step
constexpr int kNsMaxIter = 60;

// ---- fp64 copies and reductions ----
__global__ void to_f64_kernel(const float* __restrict__ A, double* __restrict__ B, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    B[i] = (double)A[i];
}

// sum of squares of A64 into *out (fixed order: per-block partials, then one block)
__global__ void sumsq_partial_kernel(const double* __restrict__ A, int64_t n, double* __restrict__ part) {
  double s = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    s = fma(A[i], A[i], s);
  s = warp_sum(s);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    part[blockIdx.x] = t;
  }
}

// Y = A / c, Z = I with c = sqrt(sum part) (one value, every thread recomputes it in the same order)
__global__ void ns_init_kernel(const double* __restrict__ A, const double* __restrict__ part, int nparts, int d,
                               double* __restrict__ Y, double* __restrict__ Z, double* __restrict__ cval,
                               int* __restrict__ done, uint32_t* err) {
  double s = 0.0;
  for (int i = 0; i < nparts; ++i) s += part[i];
  const double c = sqrt(s);
  const int64_t n = (int64_t)d * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    Y[i] = A[i] / c;
    Z[i] = (i / d == i % d) ? 1.0 : 0.0;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *cval = c;
    *done = 0;
    if (!(c > 0.0) || !isfinite(c)) {
      *done = 1;
      if (err) atomicOr(err, GIFT_DEV_NONFINITE);
    }
  }
}

// ---- register-tiled fp64 GEMM: C = alpha A B + beta I (row-major d x d) ----
// Skip mode (Newton-Schulz after convergence): if *done, C = copy_src instead.
// track: max |C - I| over the tile folded into *dev (bits of a non-negative double).
constexpr int kGT = 128, kGK = 8;
__global__ void __launch_bounds__(256) dgemm_kernel(const double* __restrict__ A, const double* __restrict__ B,
                                                    double* __restrict__ C, int d, double alpha, double beta,
                                                    const int* __restrict__ done, const double* __restrict__ copy_src,
                                                    unsigned long long* __restrict__ dev) {
  const int r0 = blockIdx.y * kGT, c0 = blockIdx.x * kGT;
  const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;  // 16 x 16 threads, 8 x 8 outputs each
  if (done && *done) {
    if (copy_src) {
      for (int e = threadIdx.x; e < kGT * kGT; e += 256) {
        const int r = r0 + e / kGT, c = c0 + e % kGT;
        if (r < d && c < d) C[(int64_t)r * d + c] = copy_src[(int64_t)r * d + c];
      }
    }
    return;
  }
  __shared__ double As[kGK][kGT + 2];
  __shared__ double Bs[kGK][kGT + 2];
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < d; k0 += kGK) {
    for (int e = threadIdx.x; e < kGT * kGK; e += 256) {
      const int r = e / kGK, k = e % kGK;  // A tile: rows r0.., cols k0..
      const int gr = r0 + r, gk = k0 + k;
      As[k][r] = (gr < d && gk < d) ? A[(int64_t)gr * d + gk] : 0.0;
      const int kb = e / kGT, c = e % kGT;  // B tile: rows k0.., cols c0..
      const int gkb = k0 + kb, gc = c0 + c;
      Bs[kb][c] = (gkb < d && gc < d) ? B[(int64_t)gkb * d + gc] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kGK; ++k) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[k][tr + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[k][tc + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double mx = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + tr + 16 * i;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + tc + 16 * j;
      if (r < d && c < d) {
        const double v = alpha * acc[i][j] + (r == c ? beta : 0.0);
        C[(int64_t)r * d + c] = v;
        if (dev) mx = fmax(mx, fabs(v - (r == c ? 1.0 : 0.0)));
      }
    }
  }
  if (dev) {
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    for (int o = 2; o < 32; o <<= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) atomicMax(dev, (unsigned long long)__double_as_longlong(mx));
  }
}

// after an applied step: stop once its max |T - I| was below tol (or not
// finite: give up, the output kernel reports it); reset the tracker
__global__ void ns_check_kernel(unsigned long long* dev, int* done) {
  const double v = __longlong_as_double((long long)*dev);
  if (v < kNsTol || !isfinite(v)) *done = 1;
  *dev = 0ull;
}

// ---- blocked Cholesky ----
// Diagonal block p: unblocked right-looking factorisation in shared memory,
// then its inverse by forward substitution.  A non-positive pivot (A not
// positive definite to fp64 precision) is reported and replaced by the
// smallest positive pivot scale, so the factor stays finite.
__global__ void __launch_bounds__(kFT) chol_diag_kernel(double* __restrict__ A, int d, int p,
                                                        double* __restrict__ Dinv, uint32_t* err) {
  extern __shared__ double dsm[];  // two [64][65] fp64 tiles (kBlockSmem bytes)
  double (*S)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm);
  double (*Iv)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm + kNB * (kNB + 1));
  __shared__ int bad;
  const int o = p * kNB;
  if (threadIdx.x == 0) bad = 0;
  for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
    const int i = e / kNB, j = e % kNB;
    S[i][j] = j <= i ? A[(int64_t)(o + i) * d + o + j] : 0.0;
  }
  __syncthreads();
  for (int j = 0; j < kNB; ++j) {
    if (threadIdx.x == 0) {
      double v = S[j][j];
      if (!(v > 0.0)) {
        bad = isfinite(v) ? (bad | 1) : (bad | 2);
        v = 1e-300;
      }
      S[j][j] = sqrt(v);
    }
    __syncthreads();
    const double ljj = S[j][j];
    for (int i = j + 1 + threadIdx.x; i < kNB; i += kFT) S[i][j] /= ljj;
    __syncthreads();
    for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
      const int i = e / kNB, k = e % kNB;
      if (k > j && i >= k) S[i][k] -= S[i][j] * S[k][j];
    }
    __syncthreads();
  }
  // inverse of the lower-triangular S: column c solved by thread c
  if (threadIdx.x < kNB) {
    const int c = threadIdx.x;
    for (int i = 0; i < kNB; ++i) {
      double v = (i == c) ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) v -= S[i][k] * Iv[k][c];
      Iv[i][c] = i >= c ? v / S[i][i] : 0.0;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
    const int i = e / kNB, j = e % kNB;
    A[(int64_t)(o + i) * d + o + j] = j <= i ? S[i][j] : 0.0;
    Dinv[(int64_t)p * kNB * kNB + e] = Iv[i][j];
  }
  if (threadIdx.x == 0 && err && bad)
    atomicOr(err, ((bad & 1) ? GIFT_DEV_RANK_DEFICIENT : 0u) | ((bad & 2) ? GIFT_DEV_NONFINITE : 0u));
}

// 64 x 64 block product acc = sum over a 64-long k of L[i][k] R[k][j] with both
// operands in shared memory; thread (tr, tc) owns rows tr + 16 a, cols tc + 16 b.
GIFT_DEV void block_mma(const double (*L)[kNB + 1], const double (*R)[kNB + 1], double (&acc)[4][4], int tr, int tc) {
#pragma unroll 8
  for (int k = 0; k < kNB; ++k) {
    double a[4], b[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) a[x] = L[tr + 16 * x][k];
#pragma unroll
    for (int y = 0; y < 4; ++y) b[y] = R[k][tc + 16 * y];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
  }
}

// Blocks below the diagonal: L_ip = A_ip L_pp^{-T} = A_ip (Dinv_p)^T, in place.
__global__ void __launch_bounds__(kFT) chol_panel_kernel(double* __restrict__ A, int d, int p,
                                                         const double* __restrict__ Dinv) {
  extern __shared__ double dsm[];  // two [64][65] fp64 tiles (kBlockSmem bytes)
  double (*Ab)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm);
  double (*Dt)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm + kNB * (kNB + 1));
  const int i = p + 1 + blockIdx.x, o = p * kNB;
  for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
    const int r = e / kNB, c = e % kNB;
    Ab[r][c] = A[(int64_t)(i * kNB + r) * d + o + c];
    Dt[c][r] = Dinv[(int64_t)p * kNB * kNB + e];
  }
  __syncthreads();
  const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;
  double acc[4][4] = {};
  block_mma(Ab, Dt, acc, tr, tc);
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) A[(int64_t)(i * kNB + tr + 16 * x) * d + o + tc + 16 * y] = acc[x][y];
}

// Trailing update: A_ij -= L_ip L_jp^T for p < j <= i (one CTA per block).
__global__ void __launch_bounds__(kFT) chol_update_kernel(double* __restrict__ A, int d, int p) {
  extern __shared__ double dsm[];  // two [64][65] fp64 tiles (kBlockSmem bytes)
  double (*Li)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm);
  double (*Ljt)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm + kNB * (kNB + 1));
  const int nr = d / kNB - p - 1;
  // block index -> (i, j), i >= j, in the remaining lower triangle
  int b = blockIdx.x, ii = 0;
  while (b >= ii + 1) {
    b -= ii + 1;
    ++ii;
  }
  if (ii >= nr) return;
  const int i = p + 1 + ii, j = p + 1 + b, o = p * kNB;
  for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
    const int r = e / kNB, c = e % kNB;
    Li[r][c] = A[(int64_t)(i * kNB + r) * d + o + c];
    Ljt[c][r] = A[(int64_t)(j * kNB + r) * d + o + c];
  }
  __syncthreads();
  const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;
  double acc[4][4] = {};
  block_mma(Li, Ljt, acc, tr, tc);
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) A[(int64_t)(i * kNB + tr + 16 * x) * d + j * kNB + tc + 16 * y] -= acc[x][y];
}

// Block row i of X = L^{-1}: CTA j < i forms X_ij = -Dinv_i sum_{k=j}^{i-1} L_ik X_kj,
// CTA i writes X_ii = Dinv_i.
__global__ void __launch_bounds__(kFT) trinv_row_kernel(const double* __restrict__ L, double* __restrict__ X, int d,
                                                        int i, const double* __restrict__ Dinv) {
  extern __shared__ double dsm[];  // two [64][65] fp64 tiles (kBlockSmem bytes)
  double (*P)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm);
  double (*Q)[kNB + 1] = reinterpret_cast<double (*)[kNB + 1]>(dsm + kNB * (kNB + 1));
  const int j = blockIdx.x;
  if (j == i) {
    for (int e = threadIdx.x; e < kNB * kNB; e += kFT)
      X[(int64_t)(i * kNB + e / kNB) * d + j * kNB + e % kNB] = Dinv[(int64_t)i * kNB * kNB + e];
    return;
  }
  const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;
  double acc[4][4] = {};
  for (int k = j; k < i; ++k) {
    __syncthreads();
    for (int e = threadIdx.x; e < kNB * kNB; e += kFT) {
      const int r = e / kNB, c = e % kNB;
      P[r][c] = L[(int64_t)(i * kNB + r) * d + k * kNB + c];
      Q[r][c] = X[(int64_t)(k * kNB + r) * d + j * kNB + c];
    }
    __syncthreads();
    block_mma(P, Q, acc, tr, tc);
  }
  __syncthreads();
  // P = Dinv_i, Q = acc
  for (int e = threadIdx.x; e < kNB * kNB; e += kFT) P[e / kNB][e % kNB] = Dinv[(int64_t)i * kNB * kNB + e];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) Q[tr + 16 * x][tc + 16 * y] = acc[x][y];
  __syncthreads();
  double out[4][4] = {};
  block_mma(P, Q, out, tr, tc);
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) X[(int64_t)(i * kNB + tr + 16 * x) * d + j * kNB + tc + 16 * y] = -out[x][y];
}

// bf16 parts of x: parts = 2 (hi, lo) or 3 (hi, mid, lo), each the bf16
// rounding of what the earlier parts leave; written at split[t * n + i].
GIFT_DEV void write_bf16_parts(float x, int parts, uint16_t* __restrict__ split, int64_t n, int64_t i) {
  float rest = x;
  for (int t = 0; t < parts; ++t) {
    const __nv_bfloat16 b = __float2bfloat16_rn(rest);
    split[t * n + i] = __bfloat16_as_ushort(b);
    rest -= __bfloat162float(b);
  }
}

// ---- outputs: fp32 and the bf16 parts of a d x d matrix ----
// mode 0: out[r][c] = s * S[r][c];  mode 1: out[r][c] = s * S[c][r] for r <= c, else 0
// (the transpose of a lower-triangular source).  32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) dense_out_kernel(const double* __restrict__ S, int d, int mode,
                                                        const double* __restrict__ scale, int scale_pow,
                                                        float* __restrict__ out, uint16_t* __restrict__ split,
                                                        int parts, uint32_t* err) {
  __shared__ double T[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  double s = 1.0;
  if (scale) s = scale_pow > 0 ? sqrt(*scale) : 1.0 / sqrt(*scale);
  for (int y = ty; y < 32; y += 8) {
    // mode 1 reads the transposed tile (rows c0.., cols r0..) coalesced
    const int rr = mode ? c0 + y : r0 + y, cc = mode ? r0 + tx : c0 + tx;
    T[y][tx] = (rr < d && cc < d) ? S[(int64_t)rr * d + cc] : 0.0;
  }
  __syncthreads();
  bool bad = false;
  for (int y = ty; y < 32; y += 8) {
    const int r = r0 + y, c = c0 + tx;
    if (r >= d || c >= d) continue;
    double v = mode ? (r <= c ? T[tx][y] : 0.0) : T[y][tx];
    v *= s;
    const float f = (float)v;
    bad |= not_finite(f);
    out[(int64_t)r * d + c] = f;
    write_bf16_parts(f, parts, split, (int64_t)d * d, (int64_t)r * d + c);
  }
  report_bits(err, bad, GIFT_DEV_NONFINITE);
}

// fp32 M -> its bf16 parts (for a transform made elsewhere)
__global__ void dense_split_kernel(const float* __restrict__ M, int64_t n, int parts, uint16_t* __restrict__ split) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    write_bf16_parts(M[i], parts, split, n, i);
}

constexpr int kPartBlocks = 256;

}  // namespace

size_t dense_factor_ws_bytes(int64_t d, int kind) {
  const size_t m = (size_t)d * d * sizeof(double);
  if (kind == GIFT_DENSE_CHOLESKY) return 2 * m + (size_t)d * kNB * sizeof(double);
  // Newton-Schulz: A, Y, Z, T, P, plus partial sums, c, done, tracker
  return 5 * m + kPartBlocks * sizeof(double) + 64;
}

cudaError_t launch_dense_factor(const float* A, int d, int kind, float* M, float* M_inv, uint16_t* M_split,
                                uint16_t* M_inv_split, void* ws, uint32_t* err, cudaStream_t s) {
  const int64_t n = (int64_t)d * d;
  double* A64 = (double*)ws;
  const int ew = kNumSMs * 8;
  to_f64_kernel<<<ew, 256, 0, s>>>(A, A64, n);
  const dim3 og((d + 31) / 32, (d + 31) / 32);
  if (kind == GIFT_DENSE_CHOLESKY) {
    static unsigned long long masks[4] = {};
    cudaError_t e;
    if ((e = ensure_smem_attr(chol_diag_kernel, kBlockSmem, &masks[0])) != cudaSuccess ||
        (e = ensure_smem_attr(chol_panel_kernel, kBlockSmem, &masks[1])) != cudaSuccess ||
        (e = ensure_smem_attr(chol_update_kernel, kBlockSmem, &masks[2])) != cudaSuccess ||
        (e = ensure_smem_attr(trinv_row_kernel, kBlockSmem, &masks[3])) != cudaSuccess)
      return e;
    double* X = A64 + n;
    double* Dinv = X + n;
    const int nb = d / kNB;
    for (int p = 0; p < nb; ++p) {
      chol_diag_kernel<<<1, kFT, kBlockSmem, s>>>(A64, d, p, Dinv, err);
      if (p + 1 < nb) {
        chol_panel_kernel<<<nb - p - 1, kFT, kBlockSmem, s>>>(A64, d, p, Dinv);
        const int r = nb - p - 1;
        chol_update_kernel<<<r * (r + 1) / 2, kFT, kBlockSmem, s>>>(A64, d, p);
      }
    }
    for (int i = 0; i < nb; ++i) trinv_row_kernel<<<i + 1, kFT, kBlockSmem, s>>>(A64, X, d, i, Dinv);
    // M = (L^{-1})^T, M^{-1} = L^T
    dense_out_kernel<<<og, 256, 0, s>>>(X, d, 1, nullptr, 0, M, M_split, 3, err);
    dense_out_kernel<<<og, 256, 0, s>>>(A64, d, 1, nullptr, 0, M_inv, M_inv_split, 2, err);
    return cudaGetLastError();
  }
  double* Y = A64 + n;
  double* Z = Y + n;
  double* T = Z + n;
  double* P = T + n;
  double* part = P + n;
  double* cval = part + kPartBlocks;
  int* done = (int*)(cval + 1);
  unsigned long long* dev = (unsigned long long*)(cval + 2);
  sumsq_partial_kernel<<<kPartBlocks, 256, 0, s>>>(A64, n, part);
  ns_init_kernel<<<ew, 256, 0, s>>>(A64, part, kPartBlocks, d, Y, Z, cval, done, err);
  cudaMemsetAsync(dev, 0, sizeof(unsigned long long), s);
  const dim3 gg((d + kGT - 1) / kGT, (d + kGT - 1) / kGT);
  for (int it = 0; it < kNsMaxIter; ++it) {
    // T = 1.5 I - 0.5 Z Y (tracks max |T - I|), then Y <- Y T, Z <- T Z
    dgemm_kernel<<<gg, 256, 0, s>>>(Z, Y, T, d, -0.5, 1.5, done, nullptr, dev);
    dgemm_kernel<<<gg, 256, 0, s>>>(Y, T, P, d, 1.0, 0.0, done, Y, nullptr);
    dgemm_kernel<<<gg, 256, 0, s>>>(T, Z, Y, d, 1.0, 0.0, done, Z, nullptr);  // Y buffer takes T Z
    ns_check_kernel<<<1, 1, 0, s>>>(dev, done);
    // rotate: (Y, Z) <- (P, old-Y buffer)
    double* y = P;
    double* z = Y;
    P = Z;
    Y = y;
    Z = z;
  }
  // M = Z c^{-1/2} = A^{-1/2},  M^{-1} = Y c^{1/2} = A^{1/2}
  dense_out_kernel<<<og, 256, 0, s>>>(Z, d, 0, cval, -1, M, M_split, 3, err);
  dense_out_kernel<<<og, 256, 0, s>>>(Y, d, 0, cval, +1, M_inv, M_inv_split, 2, err);
  return cudaGetLastError();
}

cudaError_t launch_dense_split(const float* M, int d, int parts, uint16_t* split, cudaStream_t s) {
  dense_split_kernel<<<kNumSMs * 8, 256, 0, s>>>(M, (int64_t)d * d, parts, split);
  return cudaGetLastError();
}

}  // namespace gift
