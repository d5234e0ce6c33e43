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
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace gift {

cudaError_t launch_syrk_tc(const void* X, gift_dtype xdt, int64_t N, int d, float* A, float* part, int splits,
                           uint32_t* err, cudaStream_t s, bool* used);
int syrk_tc_tiles(int d);

namespace {

constexpr int kRT = 256;
constexpr double kCholTol = 1e-10;     // pivot / max diagonal below this: column dropped
constexpr double kJacobiTol = 1e-15;   // off(B) / ||B||_F at convergence
constexpr int kJacobiMaxSweeps = 40;

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
__global__ void omega_kernel(float* __restrict__ Y, int d, int m, uint64_t seed) {
  const int64_t n = (int64_t)d * m;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t h = splitmix64(seed ^ (uint64_t)e);
    Y[e] = (h >> 63) ? -1.0f : 1.0f;
  }
}

// Y = A Q (d x d times d x m, m <= 64), 32 rows of Y per CTA, fp32 in a fixed order.
__global__ void __launch_bounds__(kRT) skinny_kernel(const float* __restrict__ A, const float* __restrict__ Q,
                                                     float* __restrict__ Y, int d, int m) {
  __shared__ float As[32][64 + 4];
  __shared__ float Qs[64][64];
  const int r = threadIdx.x >> 3, cg = (threadIdx.x & 7) * 8;
  const int64_t row0 = (int64_t)blockIdx.x * 32;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  for (int k0 = 0; k0 < d; k0 += 64) {
    {
      const float* src = A + (row0 + r) * d + k0 + cg;
      float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
      As[r][cg + 0] = a.x; As[r][cg + 1] = a.y; As[r][cg + 2] = a.z; As[r][cg + 3] = a.w;
      As[r][cg + 4] = b.x; As[r][cg + 5] = b.y; As[r][cg + 6] = b.z; As[r][cg + 7] = b.w;
    }
    for (int e = threadIdx.x; e < 64 * 64; e += kRT) {
      const int kk = e >> 6, c = e & 63;
      Qs[kk][c] = (c < m) ? __ldg(Q + (int64_t)(k0 + kk) * m + c) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 64; ++kk) {
      const float a = As[r][kk];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = fmaf(a, Qs[kk][cg + c], acc[c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int c = 0; c < 8; ++c)
    if (cg + c < m) Y[(row0 + r) * m + cg + c] = acc[c];
}

// part[p] = Ya[rows of p]^T Yb[rows of p] (m x m, fp64), 64 rows per part.
__global__ void __launch_bounds__(kRT) gram_partial_kernel(const float* __restrict__ Ya,
                                                           const float* __restrict__ Yb, int d, int m,
                                                           double* __restrict__ part) {
  __shared__ float Sa[64][64];
  __shared__ float Sb[64][64];
  const int p = blockIdx.x;
  const int r0 = p * 64;
  const int rows = min(64, d - r0);
  for (int e = threadIdx.x; e < 64 * m; e += kRT) {
    const int rr = e / m, c = e % m;
    Sa[rr][c] = rr < rows ? Ya[(int64_t)(r0 + rr) * m + c] : 0.0f;
    Sb[rr][c] = rr < rows ? Yb[(int64_t)(r0 + rr) * m + c] : 0.0f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < m * m; e += kRT) {
    const int i = e / m, j = e % m;
    double acc = 0.0;
    for (int rr = 0; rr < 64; ++rr) acc = fma((double)Sa[rr][i], (double)Sb[rr][j], acc);
    part[(int64_t)p * m * m + e] = acc;
  }
}

// Sum the Gram partials, Cholesky-factor in fp64 (dropping columns whose
// pivot vanishes), and write R^{-1} (m x m, upper) with dropped columns zeroed.
__global__ void __launch_bounds__(kRT) chol_kernel(const double* __restrict__ part, int nparts, int m,
                                                   double* __restrict__ Rinv, uint32_t* __restrict__ dev_status) {
  extern __shared__ double sm[];
  double* Gs = sm;                  // m x m (lower Cholesky factor in place)
  double* Li = sm + 64 * 65;        // m x m, L^{-1}
  __shared__ int defic[64];
  __shared__ double maxdiag;
  __shared__ int bad;
  const int ld = 65;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < m * m; e += kRT) {
    double g = 0.0;
    for (int p = 0; p < nparts; ++p) g += part[(int64_t)p * m * m + e];
    if (!isfinite(g)) bad = 1;
    Gs[(e / m) * ld + e % m] = g;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double mx = 0.0;
    for (int i = 0; i < m; ++i) mx = fmax(mx, Gs[i * ld + i]);
    maxdiag = mx;
  }
  __syncthreads();
  for (int j = 0; j < m; ++j) {
    if (threadIdx.x == 0) {
      const double piv = Gs[j * ld + j];
      const bool ok = piv > kCholTol * maxdiag;
      defic[j] = ok ? 0 : 1;
      Gs[j * ld + j] = ok ? sqrt(piv) : 1.0;
    }
    __syncthreads();
    const double Ljj = Gs[j * ld + j];
    for (int i = j + 1 + threadIdx.x; i < m; i += kRT) Gs[i * ld + j] = defic[j] ? 0.0 : Gs[i * ld + j] / Ljj;
    __syncthreads();
    const int rem = m - j - 1;
    for (int e = threadIdx.x; e < rem * rem; e += kRT) {
      const int i = j + 1 + e / rem, k = j + 1 + e % rem;
      if (k <= i) Gs[i * ld + k] -= Gs[i * ld + j] * Gs[k * ld + j];
    }
    __syncthreads();
  }
  // L^{-1} column by column (forward substitution), one thread per column
  if (threadIdx.x < m) {
    const int c = threadIdx.x;
    for (int i = 0; i < m; ++i) Li[i * ld + c] = 0.0;
    for (int i = c; i < m; ++i) {
      double x = (i == c) ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) x -= Gs[i * ld + k] * Li[k * ld + c];
      Li[i * ld + c] = x / Gs[i * ld + i];
    }
  }
  __syncthreads();
  // R = L^T, so R^{-1} = (L^{-1})^T; zero dropped columns so those Q columns are 0
  for (int e = threadIdx.x; e < m * m; e += kRT) {
    const int k = e / m, c = e % m;
    Rinv[e] = defic[c] ? 0.0 : Li[c * ld + k];
  }
  if (threadIdx.x == 0 && dev_status) {
    uint32_t f = 0;
    for (int j = 0; j < m; ++j)
      if (defic[j]) f |= GIFT_DEV_RANK_DEFICIENT;
    if (bad) f |= GIFT_DEV_NONFINITE;
    if (f) atomicOr(dev_status, f);
  }
}

// Qo = Yi R^{-1} (row by row, fp64 accumulation), 4 rows per CTA.
__global__ void __launch_bounds__(kRT) qr_apply_kernel(const float* __restrict__ Yi, const double* __restrict__ Rinv,
                                                       float* __restrict__ Qo, int d, int m) {
  __shared__ double Rs[64 * 64];
  __shared__ double Ys[4][64];
  for (int e = threadIdx.x; e < m * m; e += kRT) Rs[e] = Rinv[e];
  const int rr = threadIdx.x >> 6, c = threadIdx.x & 63;
  const int64_t row = (int64_t)blockIdx.x * 4 + rr;
  if (row < d && c < m) Ys[rr][c] = (double)Yi[row * m + c];
  __syncthreads();
  if (row < d && c < m) {
    double acc = 0.0;
    for (int k = 0; k <= c; ++k) acc = fma(Ys[rr][k], Rs[k * m + c], acc);
    Qo[row * m + c] = (float)acc;
  }
}

// Rayleigh-Ritz on B = Q^T (A Q): fp64 Jacobi (parallel round-robin order),
// eigenvalues sorted descending, lambda/rho written, sorted vectors to Vs.
__global__ void __launch_bounds__(kRT) rr_kernel(const double* __restrict__ part, int nparts, int m, int r,
                                                 const float* __restrict__ A, int d, double* __restrict__ Vs,
                                                 float* __restrict__ lambda, float* __restrict__ rho,
                                                 uint32_t* __restrict__ dev_status) {
  extern __shared__ double sm[];
  const int ld = 65;
  double* B = sm;              // m x m
  double* V = sm + 64 * ld;    // m x m
  __shared__ double rc[32], rs[32];
  __shared__ int rp[32], rq[32];
  __shared__ double red[kRT];
  __shared__ int order[64];
  __shared__ int stop;
  for (int e = threadIdx.x; e < m * m; e += kRT) {
    double g = 0.0;
    for (int p = 0; p < nparts; ++p) g += part[(int64_t)p * m * m + e];
    B[(e / m) * ld + e % m] = g;
    V[(e / m) * ld + e % m] = (e / m == e % m) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < m * m; e += kRT) {
    const int i = e / m, j = e % m;
    if (i < j) {
      const double s = 0.5 * (B[i * ld + j] + B[j * ld + i]);
      B[i * ld + j] = s;
      B[j * ld + i] = s;
    }
  }
  __syncthreads();
  const int mp = m + (m & 1);  // even count for the round-robin tournament
  const int npairs = mp / 2;
  for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
    // convergence: off(B)^2 <= tol^2 ||B||_F^2
    double off = 0.0, tot = 0.0;
    for (int e = threadIdx.x; e < m * m; e += kRT) {
      const double b = B[(e / m) * ld + e % m];
      tot += b * b;
      if (e / m != e % m) off += b * b;
    }
    red[threadIdx.x] = off;
    __syncthreads();
    for (int o = kRT / 2; o > 0; o >>= 1) {
      if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
      __syncthreads();
    }
    const double off_all = red[0];
    __syncthreads();
    red[threadIdx.x] = tot;
    __syncthreads();
    for (int o = kRT / 2; o > 0; o >>= 1) {
      if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
      __syncthreads();
    }
    if (threadIdx.x == 0) stop = (off_all <= kJacobiTol * kJacobiTol * red[0]) ? 1 : 0;
    __syncthreads();
    if (stop) break;
    for (int round = 0; round < mp - 1; ++round) {
      if (threadIdx.x < npairs) {
        const int i = threadIdx.x;
        auto pos = [&](int k) { return k == 0 ? 0 : 1 + (k - 1 + round) % (mp - 1); };
        int p = pos(i), q = pos(mp - 1 - i);
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        double c = 1.0, s = 0.0;
        if (q < m) {
          const double bpq = B[p * ld + q];
          if (bpq != 0.0) {
            const double theta = (B[q * ld + q] - B[p * ld + p]) / (2.0 * bpq);
            double t;
            if (fabs(theta) > 1e150)
              t = 0.5 / theta;
            else
              t = copysign(1.0, theta) / (fabs(theta) + sqrt(theta * theta + 1.0));
            c = 1.0 / sqrt(t * t + 1.0);
            s = t * c;
          }
        }
        rc[i] = c;
        rs[i] = s;
        rp[i] = p;
        rq[i] = q;
      }
      __syncthreads();
      // rows: B[p,:], B[q,:]
      for (int e = threadIdx.x; e < npairs * m; e += kRT) {
        const int i = e / m, k = e % m;
        const int p = rp[i], q = rq[i];
        if (q >= m) continue;
        const double c = rc[i], s = rs[i];
        const double bp = B[p * ld + k], bq = B[q * ld + k];
        B[p * ld + k] = c * bp - s * bq;
        B[q * ld + k] = s * bp + c * bq;
      }
      __syncthreads();
      // columns: B[:,p], B[:,q] and V[:,p], V[:,q]
      for (int e = threadIdx.x; e < npairs * m; e += kRT) {
        const int i = e / m, k = e % m;
        const int p = rp[i], q = rq[i];
        if (q >= m) continue;
        const double c = rc[i], s = rs[i];
        const double bp = B[k * ld + p], bq = B[k * ld + q];
        B[k * ld + p] = c * bp - s * bq;
        B[k * ld + q] = s * bp + c * bq;
        const double vp = V[k * ld + p], vq = V[k * ld + q];
        V[k * ld + p] = c * vp - s * vq;
        V[k * ld + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  // sort eigenvalues descending (ties by index)
  if (threadIdx.x < m) {
    const int i = threadIdx.x;
    const double ti = B[i * ld + i];
    int rank_i = 0;
    for (int j = 0; j < m; ++j) {
      const double tj = B[j * ld + j];
      if (tj > ti || (tj == ti && j < i)) ++rank_i;
    }
    order[rank_i] = i;
  }
  // trace(A) in a fixed order
  double tr = 0.0;
  for (int i = threadIdx.x; i < d; i += kRT) tr += (double)A[(int64_t)i * d + i];
  red[threadIdx.x] = tr;
  __syncthreads();
  for (int o = kRT / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  for (int e = threadIdx.x; e < m * r; e += kRT) {
    const int j = e / r, k = e % r;
    Vs[e] = V[j * ld + order[k]];
  }
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int k = 0; k < r; ++k) sum += B[order[k] * ld + order[k]];
    const double l1 = B[order[0] * ld + order[0]];
    double rh = (red[0] - sum) / (double)(d - r);
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
  for (int k = threadIdx.x; k < r; k += kRT) lambda[k] = (float)B[order[k] * ld + order[k]];
}

// U = Q Vs (d x m times m x r), fp64 accumulation.
__global__ void form_u_kernel(const float* __restrict__ Q, const double* __restrict__ Vs, int d, int m, int r,
                              float* __restrict__ U) {
  const int64_t n = (int64_t)d * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / r;
    const int k = (int)(e % r);
    double acc = 0.0;
    for (int j = 0; j < m; ++j) acc = fma((double)Q[row * m + j], Vs[j * r + k], acc);
    U[e] = (float)acc;
  }
}

constexpr size_t kSmallSmem = 2 * 64 * 65 * sizeof(double);

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

void refresh_plan(int64_t N, int64_t d, int rank, int oversample, bool a_out_given, RefreshPlan* p) {
  p->N = N;
  p->d = d;
  p->rank = rank;
  p->m = rank + oversample;
  p->iters = 0;
  p->seed = 0;
  p->gram_parts = (int)((d + 63) / 64);
  // split-K over tokens so that the triangle of 128 x 256 tiles fills the SMs
  const int64_t tiles = syrk_tc_tiles((int)d);
  int splits = 1;
  while (splits < 16 && tiles * splits < kNumSMs && N / (splits * 2) >= 1024) splits *= 2;
  p->syrk_splits = splits;
  size_t off = 0;
  p->off_A = off;
  if (!a_out_given) off += align256((size_t)d * d * sizeof(float));
  p->off_Q = off;
  off += align256((size_t)d * p->m * sizeof(float));
  p->off_Y = off;
  off += align256((size_t)d * p->m * sizeof(float));
  p->off_gram = off;
  off += align256((size_t)p->gram_parts * p->m * p->m * sizeof(double));
  p->off_small = off;
  off += align256(2 * 64 * 64 * sizeof(double));
  p->off_syrk = off;
  if (splits > 1) off += align256((size_t)splits * d * d * sizeof(float));
  p->total = off;
}

static cudaError_t orth_cholqr2(float* Yb, float* tmp, int d, int m, int parts, double* gram, double* Rinv,
                                uint32_t* dev_status, cudaStream_t s) {
  float* in = Yb;
  float* out = tmp;
  for (int pass = 0; pass < 2; ++pass) {
    gram_partial_kernel<<<parts, kRT, 0, s>>>(in, in, d, m, gram);
    chol_kernel<<<1, kRT, kSmallSmem, s>>>(gram, parts, m, Rinv, dev_status);
    qr_apply_kernel<<<(d + 3) / 4, kRT, 0, s>>>(in, Rinv, out, d, m);
    float* t = in;
    in = out;
    out = t;
  }
  return cudaGetLastError();
}

cudaError_t launch_refresh(const RefreshPlan& p, const void* X, gift_dtype xdt, float* U, float* lambda, float* rho,
                           float* A_out, void* ws, uint32_t* dev_status, cudaStream_t s) {
  // the two single-CTA fp64 kernels need 65 KB of dynamic shared memory
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    cudaError_t e1 = cudaFuncSetAttribute(chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallSmem);
    cudaError_t e2 = cudaFuncSetAttribute(rr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallSmem);
    if (e1 != cudaSuccess) return e1;
    if (e2 != cudaSuccess) return e2;
    attr_done.fetch_or(bit);
  }
  char* w = (char*)ws;
  const int d = (int)p.d, m = p.m, r = p.rank;
  float* A = A_out ? A_out : (float*)(w + p.off_A);
  float* B1 = (float*)(w + p.off_Q);
  float* B2 = (float*)(w + p.off_Y);
  double* gram = (double*)(w + p.off_gram);
  double* Rinv = (double*)(w + p.off_small);
  double* Vs = Rinv + 64 * 64;
  const float scale = (float)(1.0 / (double)p.N);

  // R1: A = X^T X / N
  bool used_tc = false;
  cudaError_t e = launch_syrk_tc(X, xdt, p.N, d, A, (float*)(w + p.off_syrk), p.syrk_splits, dev_status, s,
                                 &used_tc);
  if (e != cudaSuccess) return e;
  if (!used_tc) {
    const int nt = d / 64;
    const int tiles = nt * (nt + 1) / 2;
    if (xdt == GIFT_BF16)
      syrk_simt_kernel<__nv_bfloat16><<<tiles, kRT, 0, s>>>((const __nv_bfloat16*)X, p.N, d, A, scale);
    else
      syrk_simt_kernel<float><<<tiles, kRT, 0, s>>>((const float*)X, p.N, d, A, scale);
  }
  // R2: randomised subspace iteration
  omega_kernel<<<(d * m + kRT - 1) / kRT, kRT, 0, s>>>(B1, d, m, p.seed);
  if ((e = orth_cholqr2(B1, B2, d, m, p.gram_parts, gram, Rinv, dev_status, s)) != cudaSuccess) return e;
  for (int it = 0; it < p.iters; ++it) {
    skinny_kernel<<<d / 32, kRT, 0, s>>>(A, B1, B2, d, m);
    if ((e = orth_cholqr2(B2, B1, d, m, p.gram_parts, gram, Rinv, dev_status, s)) != cudaSuccess) return e;
    float* t = B1;
    B1 = B2;
    B2 = t;
  }
  // R3/R4: Rayleigh-Ritz, lambda, rho, U
  skinny_kernel<<<d / 32, kRT, 0, s>>>(A, B1, B2, d, m);
  gram_partial_kernel<<<p.gram_parts, kRT, 0, s>>>(B1, B2, d, m, gram);
  rr_kernel<<<1, kRT, kSmallSmem, s>>>(gram, p.gram_parts, m, r, A, d, Vs, lambda, rho, dev_status);
  form_u_kernel<<<(d * r + kRT - 1) / kRT, kRT, 0, s>>>(B1, Vs, d, m, r, U);
  return cudaGetLastError();
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
