// Factor refresh of the GIFT input-side factor (review page, section V.E /
// Algorithm 1: the factor A is recomputed every K steps; rank 32 from
// section V.B / Table II):
//
//   A = X^T X / N                                  (syrk, upper tiles mirrored)
//   Omega = +-1 from SplitMix64, Q = orth(Omega)   (counter-based, seeded)
//   repeat iters:  Q = orth(A Q)                   (skinny product + Cholesky-QR2)
//   B = Q^T A Q, B = V diag(theta) V^T (Jacobi), lambda = theta[0:r],
//   U = Q V[:, 0:r], rho = (trace A - sum lambda) / (d - r)
//
// Everything runs on the device on one stream; no host round trip.  Small
// dense steps (m x m Cholesky, Jacobi, sort) run in one CTA in fp64 shared
// memory; Gram matrices are reduced in fp64 with a fixed order so results
// are bit-identical from run to run.
#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {

cudaError_t launch_syrk_tc(const void* X, gift_dtype xdt, int64_t N, int d, float* A, float* part, int splits,
                           uint32_t* err, cudaStream_t s, bool* used);
int syrk_tc_tiles(int d);

namespace {

constexpr int kRT = 256;
constexpr double kCholTol = 1e-10;     // pivot / max diagonal below this: column dropped
constexpr double kJacobiTol = 1e-14;   // off(B) / ||B||_F at convergence
constexpr int kJacobiMaxSweeps = 40;

// Per-layer view of one refresh problem; the small-matrix kernels take a
// batch of these and pick their layer with blockIdx.z, so the refreshes of
// many layers run side by side (one CTA per layer for the fp64 steps).
constexpr int kMaxBatch = 64;
struct RefLayer {
  const float* A;   // d x d
  __nv_bfloat16* Ah;  // bf16 hi / lo split of A (tensor-core products), or null
  __nv_bfloat16* Al;
  __nv_bfloat16* Qs;  // d x 128 bf16 [Q_hi | Q_lo] operand, or null
  float* buf[3];    // [0] Q (d x m), [1] Y (ns k-slices of d x m), [2] T (d x m)
  double* gram;     // parts x m x m fp64 partial Gram matrices
  double* Lf;       // Cholesky factor (m x m) + reciprocal diagonal (m)
  double* Vs;       // m x r sorted Ritz vectors
  float* U;
  float* lambda;
  float* rho;
  uint32_t* st;
  uint64_t seed;
  int d, ns, parts, kslice;
};
struct RefBatch {
  RefLayer L[kMaxBatch];
  int n, m, r;
};
enum { kBufQ = 0, kBufY = 1, kBufT = 2 };

GIFT_DEV uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ---------------------------------------------------------------------------
// A = X^T X / N on CUDA cores: 64 x 64 output tiles of the upper triangle,
// 32-row chunks of X staged in shared memory, 4 x 4 outputs per thread.
// Off-diagonal tiles are written twice (tile and its mirror).
// ---------------------------------------------------------------------------
template <typename T>
GIFT_DEV void load8f(const T* p, float* dst);
template <>
GIFT_DEV void load8f<float>(const float* p, float* dst) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  dst[0] = a.x; dst[1] = a.y; dst[2] = a.z; dst[3] = a.w; dst[4] = b.x; dst[5] = b.y; dst[6] = b.z; dst[7] = b.w;
}
template <>
GIFT_DEV void load8f<__nv_bfloat16>(const __nv_bfloat16* p, float* dst) {
  uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = bf16lo(w[i]);
    dst[2 * i + 1] = bf16hi(w[i]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kRT) syrk_simt_kernel(const T* __restrict__ X, int64_t N, int d,
                                                        float* __restrict__ A, float scale) {
  // tile index -> (I, J), J >= I
  const int nt = d / 64;
  int t = blockIdx.x, I = 0;
  while (t >= nt - I) {
    t -= nt - I;
    ++I;
  }
  const int J = I + t;
  __shared__ float Xi[32][64 + 4];
  __shared__ float Xj[32][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  for (int64_t n0 = 0; n0 < N; n0 += 32) {
    const int64_t n = n0 + lr;
    if (n < N) {
      load8f<T>(X + n * d + I * 64 + lc, &Xi[lr][lc]);
      load8f<T>(X + n * d + J * 64 + lc, &Xj[lr][lc]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) Xi[lr][lc + e] = Xj[lr][lc + e] = 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a[e] = Xi[k][ty * 4 + e];
        b[e] = Xj[k][tx * 4 + e];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = I * 64 + ty * 4 + p, j = J * 64 + tx * 4 + q;
      const float v = acc[p][q] * scale;
      A[(int64_t)i * d + j] = v;
      if (I != J) A[(int64_t)j * d + i] = v;
    }
}

// Sum of split-K partials (entries j >= i) into the full symmetric A.
__global__ void syrk_reduce_kernel(const float* __restrict__ part, int splits, int d, float* __restrict__ A,
                                   float scale) {
  const int64_t dd = (int64_t)d * d;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < dd; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / d), j = (int)(e % d);
    if (j < i) continue;  // the lower triangle is written as the mirror
    float v = 0.0f;
    for (int s = 0; s < splits; ++s) v += part[s * dd + e];
    v *= scale;
    A[e] = v;
    if (j != i) A[(int64_t)j * d + i] = v;
  }
}

// Omega[i][j] = +1 if the top bit of splitmix64(seed ^ (i*m + j)) is 0, else -1.
__global__ void omega_kernel(const __grid_constant__ RefBatch b) {
  const RefLayer& L = b.L[blockIdx.z];
  float* Y = L.buf[kBufQ];
  const int64_t n = (int64_t)L.d * b.m;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t h = splitmix64(L.seed ^ (uint64_t)e);
    Y[e] = (h >> 63) ? -1.0f : 1.0f;
  }
  if (L.Qs) {  // split operand: +-1 is exact in bf16, lo parts and padding are 0
    const int m = b.m;
    const int64_t n2 = (int64_t)L.d * 128;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n2; e += (int64_t)gridDim.x * blockDim.x) {
      const int64_t row = e >> 7;
      const int c = (int)(e & 127);
      float v = 0.0f;
      if (c < m) v = (splitmix64(L.seed ^ (uint64_t)(row * m + c)) >> 63) ? -1.0f : 1.0f;
      L.Qs[e] = __float2bfloat16_rn(v);
    }
  }
}

// Ah = bf16(A), Al = bf16(A - Ah), elementwise (the tensor-core operands).
__global__ void split_a_kernel(const __grid_constant__ RefBatch b) {
  const RefLayer& L = b.L[blockIdx.z];
  if (!L.Ah) return;
  const int64_t n4 = (int64_t)L.d * L.d / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(L.A) + e);
    const float v[4] = {a.x, a.y, a.z, a.w};
    float h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
      l[i] = v[i] - h[i];
    }
    reinterpret_cast<uint2*>(L.Ah)[e] = make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
    reinterpret_cast<uint2*>(L.Al)[e] = make_uint2(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]));
  }
}

// Y = A Q (d x d times d x m, m <= 64), fp32 on the CUDA cores.  128 x 8 CW
// output tiles (CW = 6 for m <= 48, else 8; columns >= m idle) on 128
// threads, 8 x CW outputs per thread (two 16-byte A reads and CW / 2 8-byte Q
// reads of shared memory per 8 CW fmaf: the kernel is bound by shared-memory
// issue, not by the FMA pipe); the k range of a CTA is walked in steps of 16
// through two shared-memory buffers, the next step's A and Q values
// prefetched into registers while the current one is used.  Each output is
// one fmaf chain in increasing k over its slice; the k range is split into
// `ns` slices written to Yp[slice] (fixed order), which consumers add in
// index order.
constexpr int kSkK = 32;   // k-slice granularity
constexpr int kSkStep = 16;
constexpr int kSkThreads = 128;

template <int CW>
__global__ void __launch_bounds__(kSkThreads) skinny_kernel(const __grid_constant__ RefBatch b, int src, int dst) {
  constexpr int NC = 8 * CW;                        // tile columns
  constexpr int QPT = kSkStep * NC / kSkThreads;    // Q values a thread stages per step
  static_assert(QPT * kSkThreads == kSkStep * NC, "Q staging");
  static_assert(CW % 2 == 0, "8-byte Q reads");
  const RefLayer& Lr = b.L[blockIdx.z];
  const int d = Lr.d, m = b.m, kslice = Lr.kslice;
  if ((int)blockIdx.x >= d / 128 || (int)blockIdx.y >= Lr.ns) return;
  const float* __restrict__ A = Lr.A;
  const float* __restrict__ Q = Lr.buf[src];
  float* __restrict__ Yp = Lr.buf[dst];
  __shared__ __align__(16) float As[2][kSkStep][128 + 4];  // As[k][row]
  __shared__ __align__(16) float Qs[2][kSkStep][NC];
  const int row0 = blockIdx.x * 128;
  const int k_begin = blockIdx.y * kslice;
  const int k_end = min(d, k_begin + kslice);
  const int ty = threadIdx.x >> 3, tx = threadIdx.x & 7;  // rows 8 ty.., columns CW tx..
  // loaders: A row t, k 0 .. 15 of the step; Q row k = t / 8, columns QPT (t % 8) ..
  const int ar = threadIdx.x;
  const int qk = threadIdx.x >> 3, qc = (threadIdx.x & 7) * QPT;
  float acc[8][CW];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < CW; ++c) acc[a][c] = 0.0f;
  float4 ra[4];
  float rq[QPT];
  auto fetch = [&](int k0) {
    const float4* src4 = reinterpret_cast<const float4*>(A + (int64_t)(row0 + ar) * d + k0);
#pragma unroll
    for (int q = 0; q < 4; ++q) ra[q] = __ldg(src4 + q);
    const float* qrow = Q + (int64_t)(k0 + qk) * m;
#pragma unroll
    for (int c = 0; c < QPT; ++c) rq[c] = qc + c < m ? __ldg(qrow + qc + c) : 0.0f;
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      As[buf][4 * q + 0][ar] = ra[q].x;
      As[buf][4 * q + 1][ar] = ra[q].y;
      As[buf][4 * q + 2][ar] = ra[q].z;
      As[buf][4 * q + 3][ar] = ra[q].w;
    }
#pragma unroll
    for (int c = 0; c < QPT; ++c) Qs[buf][qk][qc + c] = rq[c];
  };
  int buf = 0;
  if (k_begin < k_end) {
    fetch(k_begin);
    stash(0);
  }
  __syncthreads();
  for (int k0 = k_begin; k0 < k_end; k0 += kSkStep) {
    const bool more = k0 + kSkStep < k_end;
    if (more) fetch(k0 + kSkStep);
#pragma unroll
    for (int kk = 0; kk < kSkStep; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      float qv[CW];
#pragma unroll
      for (int c = 0; c < CW; c += 2) {
        const float2 q2 = *reinterpret_cast<const float2*>(&Qs[buf][kk][tx * CW + c]);
        qv[c] = q2.x;
        qv[c + 1] = q2.y;
      }
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < CW; ++c) acc[a][c] = fmaf(av[a], qv[c], acc[a][c]);
    }
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
  float* out = Yp + (int64_t)blockIdx.y * d * m;
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      const int col = tx * CW + c;
      if (col < m) out[(int64_t)(row0 + ty * 8 + a) * m + col] = acc[a][c];
    }
}

// Y[0..n) += Y[s n .. (s+1) n) for s = 1..ns-1, in slice order.
__global__ void fold_slices_kernel(const __grid_constant__ RefBatch b, int which) {
  const RefLayer& L = b.L[blockIdx.z];
  const int ns = L.ns;
  if (ns < 2) return;
  float* __restrict__ Y = L.buf[which];
  const int64_t n = (int64_t)L.d * b.m;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float v = Y[e];
    for (int s = 1; s < ns; ++s) v += Y[s * n + e];
    Y[e] = v;
  }
}

// part[p] = Ya[rows of p]^T Yb[rows of p] (m x m, fp64), 256 rows per part
// staged in shared memory 64 rows at a time; thread (ti, tj) of a 16 x 16 grid
// owns the 4 x 4 block of entries (4 ti.., 4 tj..).  Parts of 256 rows keep
// the partials few (d / 256), so the one-CTA consumers sum little.
constexpr int kGramRows = 256;

template <int TM>  // outputs per thread and dimension: 16 TM >= m columns of the tile
__global__ void __launch_bounds__(kRT) gram_partial_kernel(const __grid_constant__ RefBatch bt, int wa, int wb) {
  constexpr int W = 16 * TM;        // tile columns (48 or 64)
  constexpr int E = 64 * W / kRT;   // entries of a 64-row tile per thread
  static_assert(E * kRT == 64 * W, "tile entries per thread");
  const RefLayer& Lr = bt.L[blockIdx.z];
  const int d = Lr.d, m = bt.m;
  if ((int)blockIdx.x >= Lr.parts) return;
  const float* __restrict__ Ya = Lr.buf[wa];
  const float* __restrict__ Yb = Lr.buf[wb];
  double* __restrict__ part = Lr.gram;
  __shared__ __align__(16) float Sa[64][W];
  __shared__ __align__(16) float Sb[64][W];
  const int p = blockIdx.x;
  const int ti = threadIdx.x >> 4, tj = threadIdx.x & 15;
  double acc[TM][TM];
#pragma unroll
  for (int a = 0; a < TM; ++a)
#pragma unroll
    for (int b = 0; b < TM; ++b) acc[a][b] = 0.0;
  // A thread's E entries of each 64-row tile, loaded into registers all at
  // once (one memory latency per tile), the next tile's while this one is
  // multiplied.
  float ra[E], rb[E];
  auto fetch = [&](int r0) {
    const int rows = min(64, d - r0);
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int e = threadIdx.x + k * kRT, rr = e / W, c = e % W;
      const bool in = rr < rows && c < m;
      ra[k] = in ? __ldg(Ya + (int64_t)(r0 + rr) * m + c) : 0.0f;
      rb[k] = in ? __ldg(Yb + (int64_t)(r0 + rr) * m + c) : 0.0f;
    }
  };
  const int rbeg = p * kGramRows, rend = min(d, rbeg + kGramRows);
  if (rbeg < rend) fetch(rbeg);
  for (int r0 = rbeg; r0 < rend; r0 += 64) {
    __syncthreads();
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const int e = threadIdx.x + k * kRT;
      Sa[e / W][e % W] = ra[k];
      Sb[e / W][e % W] = rb[k];
    }
    __syncthreads();
    if (r0 + 64 < rend) fetch(r0 + 64);
#pragma unroll 4
    for (int rr = 0; rr < 64; ++rr) {
      double a4[TM], b4[TM];
      if constexpr (TM == 4) {
        const float4 va = *reinterpret_cast<const float4*>(&Sa[rr][ti * 4]);
        const float4 vb = *reinterpret_cast<const float4*>(&Sb[rr][tj * 4]);
        a4[0] = va.x; a4[1] = va.y; a4[2] = va.z; a4[3] = va.w;
        b4[0] = vb.x; b4[1] = vb.y; b4[2] = vb.z; b4[3] = vb.w;
      } else {
#pragma unroll
        for (int a = 0; a < TM; ++a) {
          a4[a] = Sa[rr][ti * TM + a];
          b4[a] = Sb[rr][tj * TM + a];
        }
      }
#pragma unroll
      for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int b = 0; b < TM; ++b) acc[a][b] = fma(a4[a], b4[b], acc[a][b]);
    }
  }
  const int mm = m * m;
#pragma unroll
  for (int a = 0; a < TM; ++a)
#pragma unroll
    for (int b = 0; b < TM; ++b) {
      const int i = ti * TM + a, j = tj * TM + b;
      if (i < m && j < m) part[(int64_t)p * mm + i * m + j] = acc[a][b];
    }
}

// Fixed-order sum of the Gram partials of entry e (loads issued ahead).
GIFT_DEV double sum_parts(const double* __restrict__ part, int nparts, int mm, int e) {
  double g = 0.0;
#pragma unroll 8
  for (int p = 0; p < nparts; ++p) g += __ldg(part + (int64_t)p * mm + e);
  return g;
}

constexpr int kST = 1024;  // threads of the single-CTA small-matrix kernels

// Cholesky factor L of the summed Gram matrix (fp64, outer-product form):
// at step j every thread updates its fixed lower-triangle entries (i, k),
// k > j, by G[i][k] -= G[i][j] G[k][j] / G[j][j]; one barrier per column.
// A pivot below kCholTol of the largest diagonal entry drops column j
// (L[:, j] = e_j, flagged), so that column of Q comes out zero.
// Output: Lout = X (m x m, row-major, lower triangle), the inverse of L in
// the sense of the forward substitution that qr_apply_kernel applies to every
// row:  x_i = inv_i (e_i - sum_{k<i} L[i][k] x_k),  inv_i = 1/L[i][i] (0 for a
// dropped column, whose row of X is then zero), followed by inv (m).
__global__ void __launch_bounds__(kST) chol_kernel(const __grid_constant__ RefBatch bt) {
  const RefLayer& Lr = bt.L[blockIdx.z];
  const double* __restrict__ part = Lr.gram;
  const int nparts = Lr.parts, m = bt.m;
  double* __restrict__ Lout = Lr.Lf;
  uint32_t* __restrict__ dev_status = Lr.st;
  extern __shared__ double sm[];
  const int ld = 65;
  double* G = sm;  // m x m
  __shared__ double piv[64];
  __shared__ double mxd;
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < m * m; e += kST) {
    const double g = sum_parts(part, nparts, m * m, e);
    if (!isfinite(g)) bad = 1;
    G[(e / m) * ld + e % m] = g;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    double mx = 0.0;
    for (int i = threadIdx.x; i < m; i += 32) mx = fmax(mx, G[i * ld + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (threadIdx.x == 0) mxd = mx;
  }
  // this thread's lower-triangle entries (i, k), k <= i (at most 3 for m <= 64)
  int ei[3], ek[3], ne = 0;
  {
    int e = threadIdx.x, i = 0;
    for (int q = 0; q < 3; ++q, e += kST) {
      while (i < m && e >= (i + 1) * (i + 2) / 2) ++i;
      if (i < m) {
        ei[ne] = i;
        ek[ne] = e - i * (i + 1) / 2;
        ++ne;
      }
    }
  }
  __syncthreads();
  const double tol = kCholTol * mxd;
  for (int j = 0; j < m; ++j) {
    const double pj = G[j * ld + j];
    const bool ok = pj > tol;
    if (threadIdx.x == 0) piv[j] = ok ? pj : 0.0;
    if (ok) {
      const double inv = 1.0 / pj;
      for (int q = 0; q < ne; ++q) {
        const int i = ei[q], k = ek[q];
        if (k > j) G[i * ld + k] -= G[i * ld + j] * G[k * ld + j] * inv;
      }
    }
    __syncthreads();
  }
  // L[i][j] = G[i][j] / sqrt(piv_j) below the diagonal (in place; the
  // diagonal is not needed below: inv carries it)
  __shared__ double inv[64];
  if (threadIdx.x < m) inv[threadIdx.x] = piv[threadIdx.x] > 0.0 ? 1.0 / sqrt(piv[threadIdx.x]) : 0.0;
  for (int e = threadIdx.x; e < m * m; e += kST) {
    const int i = e / m, j = e % m;
    const double pj = piv[j];
    if (i > j) G[i * ld + j] = pj > 0.0 ? G[i * ld + j] / sqrt(pj) : 0.0;
  }
  // Z = unscaled rows of X, right-looking: Z starts as I; once row k is final
  // (after step k-1), every row i > k takes Z[i] -= L[i][k] inv_k Z[k]
  // (entries j <= k).  X[i] = inv_i Z[i].  One barrier per k.
  double* Z = sm + 64 * ld;
  for (int e = threadIdx.x; e < m * m; e += kST) Z[(e / m) * ld + e % m] = (e / m == e % m) ? 1.0 : 0.0;
  __syncthreads();
  for (int k = 0; k + 1 < m; ++k) {
    const double ik = inv[k];
    for (int e = threadIdx.x; e < (m - 1 - k) * (k + 1); e += kST) {
      const int i = k + 1 + e / (k + 1), j = e % (k + 1);
      Z[i * ld + j] -= G[i * ld + k] * ik * Z[k * ld + j];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < m * m; e += kST) {
    const int i = e / m, j = e % m;
    Lout[e] = j <= i ? inv[i] * Z[i * ld + j] : 0.0;
  }
  if (threadIdx.x < m) Lout[m * m + threadIdx.x] = inv[threadIdx.x];
  if (threadIdx.x == 0 && dev_status) {
    uint32_t f = 0;
    for (int j = 0; j < m; ++j)
      if (!(piv[j] > 0.0)) f |= GIFT_DEV_RANK_DEFICIENT;
    if (bad) f |= GIFT_DEV_NONFINITE;
    if (f) atomicOr(dev_status, f);
  }
}

// Qo = Yi R^{-1} with R = L^T, i.e. every row q = X y with X the
// substitution inverse written by chol_kernel (fp64 products, fp32 out).
// A CTA keeps X in shared memory and walks 32-row tiles of Yi; thread
// (i, rg) computes column i of rows rg, rg + 4, ..., rg + 28 of the tile.
// With dst == Q the bf16 [hi | lo] operand of the tensor-core product is
// written too (columns m..63 zero).
// fp64 shared memory of qr_apply_kernel: the m x m factor and one 32-row tile of
// Y, both as doubles (Y converted once per element, not once per product)
constexpr size_t kQrSmem = (64 * 65 + 32 * 65) * sizeof(double);

__global__ void __launch_bounds__(kRT) qr_apply_kernel(const __grid_constant__ RefBatch bt, int src, int dst) {
  const RefLayer& Lr = bt.L[blockIdx.z];
  const int d = Lr.d, m = bt.m;
  const float* __restrict__ Yi = Lr.buf[src];
  const double* __restrict__ X = Lr.Lf;
  float* __restrict__ Qo = Lr.buf[dst];
  __nv_bfloat16* __restrict__ Qs = dst == kBufQ ? Lr.Qs : nullptr;
  extern __shared__ double qsm[];
  double* Xs = qsm;            // [64][65]
  double* Yd = qsm + 64 * 65;  // [32][65]
  if ((int64_t)blockIdx.x * 32 >= d) return;
  for (int e = threadIdx.x; e < m * m; e += kRT) Xs[(e / m) * 65 + e % m] = X[e];
  const int i = threadIdx.x & 63, rg = threadIdx.x >> 6;
  for (int64_t t0 = (int64_t)blockIdx.x * 32; t0 < d; t0 += (int64_t)gridDim.x * 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * m; e += kRT) Yd[(e / m) * 65 + e % m] = (double)Yi[t0 * m + e];
    __syncthreads();
    double acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.0;
    if (i < m) {
      for (int j = 0; j <= i; ++j) {
        const double x = Xs[i * 65 + j];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fma(x, Yd[(rg + 4 * u) * 65 + j], acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t row = t0 + rg + 4 * u;
      const float q = (float)acc[u];
      if (i < m) Qo[row * m + i] = q;
      if (Qs) {
        const float hi = __bfloat162float(__float2bfloat16_rn(q));
        Qs[row * 128 + i] = __float2bfloat16_rn(hi);
        Qs[row * 128 + 64 + i] = __float2bfloat16_rn(q - hi);
      }
    }
  }
}

// Rayleigh-Ritz on B = Q^T (A Q): fp64 Jacobi in parallel round-robin order.
// Each round computes the rotations of the disjoint pairs, then every thread
// updates whole 2x2 blocks: block (a, b) of B' = J^T B J needs only the four
// entries of pairs a and b, and V' = V J is updated two entries at a time.
// Eigenvalues are sorted descending; lambda, rho and the sorted eigenvectors
// (Vs, m x r) are written.
__global__ void __launch_bounds__(kST) rr_kernel(const __grid_constant__ RefBatch bt) {
  const RefLayer& Lr = bt.L[blockIdx.z];
  const double* __restrict__ part = Lr.gram;
  const int nparts = Lr.parts, m = bt.m, r = bt.r, d = Lr.d;
  const float* __restrict__ A = Lr.A;
  double* __restrict__ Vs = Lr.Vs;
  float* __restrict__ lambda = Lr.lambda;
  float* __restrict__ rho = Lr.rho;
  uint32_t* __restrict__ dev_status = Lr.st;
  extern __shared__ double sm[];
  const int ld = 65;
  double* Bb0 = sm;
  double* Bb1 = sm + 64 * ld;
  double* Vb0 = sm + 2 * 64 * ld;
  double* Vb1 = sm + 3 * 64 * ld;
  __shared__ int pp[32], pq[32];
  __shared__ double pc[32], ps[32];
  __shared__ double red[kST / 32];
  __shared__ int order[64];
  __shared__ int stop;
  for (int e = threadIdx.x; e < m * m; e += kST) {
    Bb0[(e / m) * ld + e % m] = sum_parts(part, nparts, m * m, e);
    Vb0[(e / m) * ld + e % m] = (e / m == e % m) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < m * m; e += kST) {  // symmetrise
    const int i = e / m, j = e % m;
    if (i < j) {
      const double v = 0.5 * (Bb0[i * ld + j] + Bb0[j * ld + i]);
      Bb0[i * ld + j] = v;
      Bb0[j * ld + i] = v;
    }
  }
  __syncthreads();
  double* B = Bb0;
  double* Bn = Bb1;
  double* V = Vb0;
  double* Vn = Vb1;
  const int mp = m + (m & 1);  // even count for the round-robin tournament
  const int npairs = mp / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the tournament's pairs, round by round (p < q; q == m marks the dummy
  // partner of an odd m), and this thread's fixed work items: 2 x 2 block
  // (ba, bb) of B and up to two (row k, pair b) items of V
  __shared__ unsigned char tab_p[63][32], tab_q[63][32];
  for (int e = threadIdx.x; e < (mp - 1) * npairs; e += kST) {
    const int round = e / npairs, a = e % npairs;
    auto pos = [&](int k) { return k == 0 ? 0 : 1 + (k - 1 + round) % (mp - 1); };
    int p = pos(a), q = pos(mp - 1 - a);
    if (p > q) {
      const int t = p;
      p = q;
      q = t;
    }
    tab_p[round][a] = (unsigned char)p;
    tab_q[round][a] = (unsigned char)q;
  }
  const int nb = npairs * npairs, nv = m * npairs;
  const int ba = threadIdx.x / npairs, bb = threadIdx.x % npairs;
  const int v0 = threadIdx.x, v1 = threadIdx.x + kST;
  const int vk0 = v0 / npairs, vb0 = v0 % npairs, vk1 = v1 / npairs, vb1 = v1 % npairs;
  for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
    // convergence: off(B)^2 <= tol^2 ||B||_F^2
    double off = 0.0, tot = 0.0;
    for (int e = threadIdx.x; e < m * m; e += kST) {
      const double b = B[(e / m) * ld + e % m];
      tot += b * b;
      if (e / m != e % m) off += b * b;
    }
    off = warp_sum(off);
    tot = warp_sum(tot);
    if (lane == 0) red[warp] = off;
    __syncthreads();
    if (threadIdx.x == 0) {
      double o = 0.0;
      for (int w = 0; w < kST / 32; ++w) o += red[w];
      red[0] = o;
    }
    __syncthreads();
    const double off_all = red[0];
    __syncthreads();
    if (lane == 0) red[warp] = tot;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int w = 0; w < kST / 32; ++w) t += red[w];
      stop = (off_all <= kJacobiTol * kJacobiTol * t) ? 1 : 0;
    }
    __syncthreads();
    if (stop) break;
    for (int round = 0; round < mp - 1; ++round) {
      if (threadIdx.x < npairs) {
        const int a = threadIdx.x;
        const int p = tab_p[round][a], q = tab_q[round][a];
        // The rotation's tangent t only has to shrink B[p][q]: it is taken
        // in fp32 from the fp64 entries (a factor ~1e-7 of B[p][q] remains,
        // removed by the next sweep), so the fp64 divisions and square root
        // leave the round's critical path.  The rotation itself, c = (1 +
        // t^2)^{-1/2} and s = t c, is fp64, so B and V stay exact
        // orthogonal transforms to fp64 rounding.
        double c = 1.0, s = 0.0;
        if (q < m) {
          const float bpq = (float)B[p * ld + q];
          const float dqp = (float)(B[q * ld + q] - B[p * ld + p]);
          if (bpq != 0.0f) {
            const float theta = dqp / (2.0f * bpq);
            float t;
            if (fabsf(theta) > 1e18f)
              t = 0.5f / theta;
            else
              t = copysignf(1.0f, theta) / (fabsf(theta) + sqrtf(fmaf(theta, theta, 1.0f)));
            const double td = (double)t;
            c = rsqrt(fma(td, td, 1.0));
            s = td * c;
          }
        }
        pp[a] = p;
        pq[a] = q;
        pc[a] = c;
        ps[a] = s;
      }
      __syncthreads();
      // new row/column p = c p - s q, q = s p + c q
      if (threadIdx.x < nb) {
        const int a = ba, b = bb;
        const int pa = pp[a], qa = pq[a], pb = pp[b], qb = pq[b];
        const double ca = pc[a], sa = ps[a], cb = pc[b], sb = ps[b];
        const bool ha = qa < m, hb = qb < m;
        const double b00 = B[pa * ld + pb];
        const double b01 = hb ? B[pa * ld + qb] : 0.0;
        const double b10 = ha ? B[qa * ld + pb] : 0.0;
        const double b11 = (ha && hb) ? B[qa * ld + qb] : 0.0;
        const double r00 = ca * b00 - sa * b10, r01 = ca * b01 - sa * b11;
        const double r10 = sa * b00 + ca * b10, r11 = sa * b01 + ca * b11;
        Bn[pa * ld + pb] = cb * r00 - sb * r01;
        if (hb) Bn[pa * ld + qb] = sb * r00 + cb * r01;
        if (ha) Bn[qa * ld + pb] = cb * r10 - sb * r11;
        if (ha && hb) Bn[qa * ld + qb] = sb * r10 + cb * r11;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int w = u ? v1 : v0;
        if (w >= nv) continue;
        const int k = u ? vk1 : vk0, b = u ? vb1 : vb0;
        const int pb = pp[b], qb = pq[b];
        const double cb = pc[b], sb = ps[b];
        const double vp = V[k * ld + pb];
        if (qb < m) {
          const double vq = V[k * ld + qb];
          Vn[k * ld + pb] = cb * vp - sb * vq;
          Vn[k * ld + qb] = sb * vp + cb * vq;
        } else {
          Vn[k * ld + pb] = vp;
        }
      }
      __syncthreads();
      double* t = B;
      B = Bn;
      Bn = t;
      t = V;
      V = Vn;
      Vn = t;
    }
  }
  // sort eigenvalues descending (ties by index).  A NaN sorts as -inf, so the
  // comparison is a total order and `order` is a permutation whatever B holds
  // (a non-finite input gives NaN eigenvalues, reported as GIFT_DEV_NONFINITE;
  // with NaN compared as is, every index took rank 0 and `order` kept stale
  // shared-memory contents, which the gathers below then used as indices).
  if (threadIdx.x < m) {
    const int i = threadIdx.x;
    const double bi = B[i * ld + i];
    const double ti = isnan(bi) ? -INFINITY : bi;
    int rank_i = 0;
    for (int j = 0; j < m; ++j) {
      const double bj = B[j * ld + j];
      const double tj = isnan(bj) ? -INFINITY : bj;
      if (tj > ti || (tj == ti && j < i)) ++rank_i;
    }
    order[rank_i] = i;
  }
  // trace(A) in a fixed order
  double tr = 0.0;
  for (int i = threadIdx.x; i < d; i += kST) tr += (double)A[(int64_t)i * d + i];
  tr = warp_sum(tr);
  __syncthreads();
  if (lane == 0) red[warp] = tr;
  __syncthreads();
  for (int e = threadIdx.x; e < m * r; e += kST) {
    const int j = e / r, k = e % r;
    Vs[e] = V[j * ld + order[k]];
  }
  if (threadIdx.x == 0) {
    double trace = 0.0;
    for (int w = 0; w < kST / 32; ++w) trace += red[w];
    double sum = 0.0;
    for (int k = 0; k < r; ++k) sum += B[order[k] * ld + order[k]];
    const double l1 = B[order[0] * ld + order[0]];
    double rh = (trace - sum) / (double)(d - r);
    uint32_t f = 0;
    const double floor = ldexp(l1, -24);
    if (!(rh > floor)) {
      rh = floor;
      f |= GIFT_DEV_RHO_FLOORED;
    }
    if (!isfinite(rh) || !isfinite(sum)) f |= GIFT_DEV_NONFINITE;
    *rho = (float)rh;
    if (f && dev_status) atomicOr(dev_status, f);
  }
  for (int k = threadIdx.x; k < r; k += kST) lambda[k] = (float)B[order[k] * ld + order[k]];
}

// U = Q Vs (d x m times m x r), fp64 accumulation.
__global__ void form_u_kernel(const __grid_constant__ RefBatch bt) {
  const RefLayer& Lr = bt.L[blockIdx.z];
  const float* __restrict__ Q = Lr.buf[kBufQ];
  const double* __restrict__ Vs = Lr.Vs;
  float* __restrict__ U = Lr.U;
  const int m = bt.m, r = bt.r;
  const int64_t n = (int64_t)Lr.d * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / r;
    const int k = (int)(e % r);
    double acc = 0.0;
    for (int j = 0; j < m; ++j) acc = fma((double)Q[row * m + j], Vs[j * r + k], acc);
    U[e] = (float)acc;
  }
}

constexpr size_t kCholSmem = 2 * 64 * 65 * sizeof(double);
constexpr size_t kRRSmem = 4 * 64 * 65 * sizeof(double);

// k-slices of the skinny product: enough CTAs to cover the SMs twice
inline int skinny_slices(int d) {
  const int tiles = d / 128;
  int ns = (2 * kNumSMs + tiles - 1) / tiles;
  const int max_ns = d / (4 * kSkK);
  if (ns > max_ns) ns = max_ns;
  return ns < 1 ? 1 : ns;
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

void refresh_plan(int64_t N, int64_t d, int rank, int oversample, bool a_out_given, RefreshPlan* p,
                  bool no_split) {
  p->N = N;
  p->d = d;
  p->rank = rank;
  p->m = rank + oversample;
  p->iters = 0;
  p->seed = 0;
  p->gram_parts = (int)((d + kGramRows - 1) / kGramRows);
  p->skinny_slices = no_split ? 1 : skinny_slices((int)d);
  // split-K over tokens so that the triangle of 128 x 256 tiles fills the SMs
  const int64_t tiles = syrk_tc_tiles((int)d);
  int splits = 1;
  while (!no_split && splits < 16 && tiles * splits < kNumSMs && N / (splits * 2) >= 1024) splits *= 2;
  p->syrk_splits = splits;
  const size_t dm = (size_t)d * p->m * sizeof(float);
  size_t off = 0;
  p->off_A = off;
  if (!a_out_given) off += align256((size_t)d * d * sizeof(float));
  p->off_Q = off;
  off += align256(dm);
  p->off_Y = off;
  off += align256(dm * p->skinny_slices);
  p->off_T = off;
  off += align256(dm);
  p->off_gram = off;
  off += align256((size_t)p->gram_parts * p->m * p->m * sizeof(double));
  p->off_small = off;
  off += align256(2 * 64 * 64 * sizeof(double));
  p->off_syrk = off;
  if (splits > 1) off += align256((size_t)splits * d * d * sizeof(float));
  p->tc_skinny = !no_split;
  p->off_Ah = p->off_Al = p->off_Qs = off;
  if (p->tc_skinny) {
    p->off_Ah = off;
    off += align256((size_t)d * d * 2);
    p->off_Al = off;
    off += align256((size_t)d * d * 2);
    p->off_Qs = off;
    off += align256((size_t)d * 128 * 2);
  }
  p->total = off;
}

cudaError_t launch_refresh_batch(const RefreshPlan* plans, const RefreshIO* io, int n, cudaStream_t s) {
  static unsigned long long chol_attr = 0, rr_attr = 0, qr_attr = 0;
  cudaError_t e = ensure_smem_attr(chol_kernel, (int)kCholSmem, &chol_attr);
  if (e != cudaSuccess) return e;
  if ((e = ensure_smem_attr(rr_kernel, (int)kRRSmem, &rr_attr)) != cudaSuccess) return e;
  if ((e = ensure_smem_attr(qr_apply_kernel, (int)kQrSmem, &qr_attr)) != cudaSuccess) return e;
  if (n <= 0) return cudaSuccess;
  const int m = plans[0].m, r = plans[0].rank, iters = plans[0].iters;
  for (int base = 0; base < n; base += kMaxBatch) {
    const int cnt = n - base < kMaxBatch ? n - base : kMaxBatch;
    static thread_local RefBatch B;
    B.n = cnt;
    B.m = m;
    B.r = r;
    int dmax = 0, nsmax = 1, pmax = 1;
    // R1: A = X^T X / N for every layer of the batch in one tensor-core launch
    // (bf16 X); otherwise one launch per layer below
    static thread_local SyrkJob sj[kMaxBatch];
    for (int l = 0; l < cnt; ++l) {
      const RefreshPlan& p = plans[base + l];
      const RefreshIO& o = io[base + l];
      sj[l] = SyrkJob{o.X, o.xdt, p.N, (int)p.d, o.A_out ? o.A_out : (float*)((char*)o.ws + p.off_A), o.dev_status};
    }
    static thread_local bool batched[kMaxBatch];
    if ((e = launch_syrk_tc_batch(sj, cnt, s, batched)) != cudaSuccess) return e;
    for (int l = 0; l < cnt; ++l) {
      const RefreshPlan& p = plans[base + l];
      const RefreshIO& o = io[base + l];
      char* w = (char*)o.ws;
      const int d = (int)p.d;
      float* A = o.A_out ? o.A_out : (float*)(w + p.off_A);
      bool used_tc = batched[l];
      if (!used_tc)
        e = launch_syrk_tc(o.X, o.xdt, p.N, d, A, (float*)(w + p.off_syrk), p.syrk_splits, o.dev_status, s,
                           &used_tc);
      if (e != cudaSuccess) return e;
      if (!used_tc) {
        const int nt = d / 64;
        const int tiles = nt * (nt + 1) / 2;
        const float scale = (float)(1.0 / (double)p.N);
        if (o.xdt == GIFT_BF16)
          syrk_simt_kernel<__nv_bfloat16><<<tiles, kRT, 0, s>>>((const __nv_bfloat16*)o.X, p.N, d, A, scale);
        else
          syrk_simt_kernel<float><<<tiles, kRT, 0, s>>>((const float*)o.X, p.N, d, A, scale);
      }
      RefLayer& L = B.L[l];
      L.A = A;
      L.buf[kBufQ] = (float*)(w + p.off_Q);
      L.buf[kBufY] = (float*)(w + p.off_Y);
      L.buf[kBufT] = (float*)(w + p.off_T);
      L.gram = (double*)(w + p.off_gram);
      L.Lf = (double*)(w + p.off_small);
      L.Vs = L.Lf + 64 * 64 + 64;  // after m*m + m doubles (m <= 64)
      L.Ah = p.tc_skinny ? (__nv_bfloat16*)(w + p.off_Ah) : nullptr;
      L.Al = p.tc_skinny ? (__nv_bfloat16*)(w + p.off_Al) : nullptr;
      L.Qs = p.tc_skinny ? (__nv_bfloat16*)(w + p.off_Qs) : nullptr;
      L.U = o.U;
      L.lambda = o.lambda;
      L.rho = o.rho;
      L.st = o.dev_status;
      L.seed = p.seed;
      L.d = d;
      L.ns = p.skinny_slices;
      L.parts = p.gram_parts;
      L.kslice = (d / L.ns + kSkK - 1) / kSkK * kSkK;
      dmax = d > dmax ? d : dmax;
      nsmax = L.ns > nsmax ? L.ns : nsmax;
      pmax = L.parts > pmax ? L.parts : pmax;
    }
    const int64_t dm = (int64_t)dmax * m;
    const int ew_blocks = (int)((dm + kRT - 1) / kRT < 2 * kNumSMs ? (dm + kRT - 1) / kRT : 2 * kNumSMs);
    // qr_apply: two 32-row tiles per CTA (the m x m factor is loaded once per CTA)
    const int qr_blocks = (dmax / 32 + 1) / 2;
    const dim3 g_ew(ew_blocks, 1, cnt), g_skinny(dmax / 128, nsmax, cnt), g_gram(pmax, 1, cnt), g_one(1, 1, cnt),
        g_qr(qr_blocks, 1, cnt);
    // one Cholesky-QR pass: dst = src R^{-1} with src^T src = R^T R
    auto cholqr_pass = [&](int src, int dst) {
      if (m <= 48)
        gram_partial_kernel<3><<<g_gram, kRT, 0, s>>>(B, src, src);
      else
        gram_partial_kernel<4><<<g_gram, kRT, 0, s>>>(B, src, src);
      chol_kernel<<<g_one, kST, kCholSmem, s>>>(B);
      qr_apply_kernel<<<g_qr, kRT, kQrSmem, s>>>(B, src, dst);
    };
    // A Q into Y, k-slices folded into slice 0: fp32 CUDA cores, or for the
    // iteration products (tc) the tensor cores on the bf16 split operands
    const bool tc = plans[base].tc_skinny;
    int tc_tiles = 0;
    for (int l = 0; l < cnt; ++l) tc_tiles += B.L[l].d / 128;
    static thread_local SkinnyTcJob sk[kMaxBatch];
    int tc_nsmax = 1;
    for (int l = 0; l < cnt && tc; ++l) {
      const RefLayer& L = B.L[l];
      int ns = (2 * kNumSMs + tc_tiles - 1) / tc_tiles;
      if (ns > L.ns) ns = L.ns;
      if (ns > L.d / 256) ns = L.d / 256 > 0 ? L.d / 256 : 1;
      sk[l] = SkinnyTcJob{L.Ah, L.Al, L.Qs, L.buf[kBufY], L.d, ns, (L.d / ns + 63) / 64 * 64};
      tc_nsmax = ns > tc_nsmax ? ns : tc_nsmax;
    }
    auto skinny_product = [&](bool use_tc) {
      if (use_tc) {
        launch_skinny_tc(sk, cnt, m, s);
        // fold the tensor-core k-slices (their count may differ from the CUDA-core one)
        for (int l = 0; l < cnt; ++l) B.L[l].ns = sk[l].ns;
        if (tc_nsmax > 1) fold_slices_kernel<<<g_ew, kRT, 0, s>>>(B, kBufY);
        for (int l = 0; l < cnt; ++l) B.L[l].ns = plans[base + l].skinny_slices;
      } else {
        if (m <= 48)
          skinny_kernel<6><<<g_skinny, kSkThreads, 0, s>>>(B, kBufQ, kBufY);
        else
          skinny_kernel<8><<<g_skinny, kSkThreads, 0, s>>>(B, kBufQ, kBufY);
        if (nsmax > 1) fold_slices_kernel<<<g_ew, kRT, 0, s>>>(B, kBufY);
      }
    };
    if (tc) split_a_kernel<<<dim3(2 * kNumSMs, 1, cnt), kRT, 0, s>>>(B);
    // R2: randomised subspace iteration.  span(A Omega) = span(A orth(Omega)),
    // so the +-1 start block (exact) is multiplied by A directly; with no
    // iterations it is orthonormalised for the Rayleigh-Ritz step instead.
    omega_kernel<<<g_ew, kRT, 0, s>>>(B);
    if (iters == 0) {
      cholqr_pass(kBufQ, kBufT);
      cholqr_pass(kBufT, kBufQ);
    }
    // Each iteration needs only an orthonormal basis of span(A Q): one
    // Cholesky-QR pass (orthogonal to ~kappa^2 eps in fp64) until the last,
    // whose basis feeds the Rayleigh-Ritz step and gets the second pass
    // (Cholesky-QR2, orthogonal to working precision).
    for (int it = 0; it < iters; ++it) {
      skinny_product(tc);
      if (it + 1 < iters) {
        cholqr_pass(kBufY, kBufQ);
      } else {
        cholqr_pass(kBufY, kBufT);
        cholqr_pass(kBufT, kBufQ);
      }
    }
    // R3/R4: Rayleigh-Ritz, lambda, rho, U (fp32 product: the Ritz values
    // need the accuracy the bf16 split would not give)
    skinny_product(false);
    if (m <= 48)
      gram_partial_kernel<3><<<g_gram, kRT, 0, s>>>(B, kBufQ, kBufY);
    else
      gram_partial_kernel<4><<<g_gram, kRT, 0, s>>>(B, kBufQ, kBufY);
    rr_kernel<<<g_one, kST, kRRSmem, s>>>(B);
    form_u_kernel<<<g_ew, kRT, 0, s>>>(B);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_refresh(const RefreshPlan& p, const void* X, gift_dtype xdt, float* U, float* lambda, float* rho,
                           float* A_out, void* ws, uint32_t* dev_status, cudaStream_t s) {
  const RefreshIO io{X, xdt, U, lambda, rho, A_out, ws, dev_status};
  return launch_refresh_batch(&p, &io, 1, s);
}

// Split-K reduction used by the tensor-core syrk.
cudaError_t launch_syrk_reduce(const float* part, int splits, int d, float* A, float scale, cudaStream_t s) {
  const int64_t dd = (int64_t)d * d;
  int64_t blocks = (dd + kRT - 1) / kRT;
  if (blocks > kNumSMs * 16) blocks = kNumSMs * 16;
  syrk_reduce_kernel<<<(int)blocks, kRT, 0, s>>>(part, splits, d, A, scale);
  return cudaGetLastError();
}

}  // namespace gift
