// Internal launch interface between the C-ABI layer (abi.cu) and the kernel
// files.  Every launcher enqueues work on `stream` and returns the launch
// error (cudaSuccess when the launch was accepted).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gift.h"

namespace gift {

// ---- Euclidean per-block E4M3 codec (rank 0): flat arrays of n_blocks*128 ----
// `err` (nullable, device): the caller's status word; kernels OR GIFT_DEV_* bits into it.
cudaError_t launch_euclid_encode(const void* G, gift_dtype dt, int64_t n_blocks, uint8_t* codes,
                                 float* scales, uint32_t* err, cudaStream_t s);
cudaError_t launch_euclid_decode(const uint8_t* codes, const float* scales, int64_t n_blocks, void* G_hat,
                                 gift_dtype dt, uint32_t* err, cudaStream_t s);

// Grouped Euclidean codec: one launch for many rank-0 layers of one dtype.
struct EuclidLayer {
  const void* src;   // encode: G;     decode: codes
  void* dst;         // encode: codes; decode: G_hat
  float* scales;
  int64_t n_blocks;  // d_out * d_in / 128
};
cudaError_t launch_euclid_group(const EuclidLayer* layers, int n, gift_dtype dt, bool encode, uint32_t* err,
                               cudaStream_t s);

// ---- Whitened codec on CUDA cores (any rank <= 32, fp32 or bf16) ----
cudaError_t launch_whiten_encode_simt(const void* G, gift_dtype dt, int64_t d_out, int64_t d_in, const float* U,
                                      const float* lambda, const float* rho, int rank, uint8_t* codes,
                                      float* scales, uint32_t* err, cudaStream_t s);
cudaError_t launch_whiten_decode_simt(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                                      const float* U, const float* lambda, const float* rho, int rank,
                                      void* G_hat, gift_dtype dt, uint32_t* err, cudaStream_t s);

// Decode-and-sum of n_parts code sets (data-parallel ranks), CUDA cores.
constexpr int kDecodeSumMaxParts = 64;
cudaError_t launch_decode_sum(const uint8_t* const* codes, const float* const* scales, int n_parts, int64_t d_out,
                              int64_t d_in, const float* U, const float* lambda, const float* rho, int rank,
                              float alpha, void* G_hat, gift_dtype dt, uint32_t* err, cudaStream_t s);

// ---- Whitened codec on the tensor cores (bf16 G, tcgen05 + TMA) ----
struct TcLayer {
  const void* G;      // bf16 d_out x d_in (encode input)
  void* G_hat;        // bf16 d_out x d_in (decode output)
  uint8_t* codes;
  float* scales;
  const float* U;
  const float* lambda;
  const float* rho;
  int d_out;
  int d_in;
  int rank;
  // 0: E4M3 codes + fp32 scales per 128.  NVFP4 (codes two per byte, E4M3
  // scales per 16 in block_scales, tensor scale in tensor_scale): encode pass 1
  // folds amax(W) into tensor_scale's bits, encode pass 2 writes the codes,
  // decode reads them.
  int fmt = 0;
  uint8_t* block_scales = nullptr;
  float* tensor_scale = nullptr;
  // Optional U split by gift_split_u ([2][d_in][64] 16-bit: bf16 [hi | lo]
  // rows, then f16 [hi | 2^11 lo] rows): the kernels then load it as it is
  // instead of splitting U themselves.  Layers with and without it go to
  // separate launches.
  const uint16_t* U_split = nullptr;
};
constexpr int kFmtE4M3 = 0, kFmtNvfp4Amax = 1, kFmtNvfp4 = 2;
bool tc_codec_available();
// stall_polls > 0 is a test hook: before any work, one thread of every CTA
// waits at most that many polls on a barrier nothing arrives at, gives up,
// and the CTA skips its work and reports GIFT_DEV_TIMEOUT.
// U (d_in x 32 fp32) -> the [2][d_in][64] split the tensor-core codec loads (see TcLayer::U_split).
cudaError_t launch_split_u(const float* U, int64_t d_in, uint16_t* U_split, cudaStream_t s);
cudaError_t launch_split_u_many(const float* const* U, uint16_t* const* U_split, const int64_t* d_in, int n,
                                cudaStream_t s);
cudaError_t launch_whiten_encode_tc(const TcLayer* layers, int n, uint32_t* err, cudaStream_t s,
                                    uint32_t stall_polls = 0);
cudaError_t launch_whiten_decode_tc(const TcLayer* layers, int n, uint32_t* err, cudaStream_t s,
                                    uint32_t stall_polls = 0);
// Cluster size (1, 2 or 4) the tensor-core codec plans for the first launch
// over these layers (-1 if they cannot be planned).  Host-side; queries the
// device's cluster occupancy once per kernel.
int tc_codec_split(const TcLayer* layers, int n, bool encode);

// ---- Round-trip error ----
size_t error_ws_bytes(int64_t n_elems);
// ---- NVFP4, Euclidean (M = I) ----
cudaError_t launch_nvfp4_amax(const void* G, gift_dtype dt, int64_t n_blocks, float* tensor_scale, cudaStream_t s);
cudaError_t launch_nvfp4_quant(const void* G, gift_dtype dt, int64_t n_blocks, const float* tensor_scale,
                               uint8_t* codes, uint8_t* sb, cudaStream_t s);
cudaError_t launch_nvfp4_finalize(float* tensor_scale, uint32_t* err, cudaStream_t s);
cudaError_t launch_nvfp4_decode(const uint8_t* codes, const uint8_t* sb, const float* tensor_scale, int64_t n_blocks,
                                void* out, gift_dtype dt, uint32_t* err, cudaStream_t s);

cudaError_t launch_roundtrip_error(const void* G, const void* G_hat, gift_dtype dt, int64_t n_elems,
                                   double* out, void* ws, cudaStream_t s);
size_t whitened_error_ws_bytes(int64_t d_out);
cudaError_t launch_whitened_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out, int64_t d_in,
                                  const float* U, const float* lambda, const float* rho, int rank, double* out,
                                  void* ws, cudaStream_t s);

// ---- Dense input-side transforms (full-rank and Cholesky variants) ----
size_t dense_factor_ws_bytes(int64_t d, int kind);
cudaError_t launch_dense_factor(const float* A, int d, int kind, float* M, float* M_inv, uint16_t* M_split,
                                uint16_t* M_inv_split, void* ws, uint32_t* err, cudaStream_t s);
cudaError_t launch_dense_split(const float* M, int d, int parts, uint16_t* split, cudaStream_t s);
cudaError_t launch_dense_encode(const void* G, int d_out, int d_in, const uint16_t* M_split, bool upper,
                                uint8_t* codes, float* scales, uint32_t* err, cudaStream_t s);
cudaError_t launch_dense_decode(const uint8_t* codes, const float* scales, int d_out, int d_in,
                                const uint16_t* Minv_split, bool upper, void* G_hat, gift_dtype out_dt,
                                uint32_t* err, cudaStream_t s);

// ---- Factor refresh ----
struct RefreshPlan {
  int64_t N, d;
  int rank, m;          // m = rank + oversample
  int iters;
  uint64_t seed;
  int gram_parts;       // partial Gram blocks
  int syrk_splits;      // split-K partial sums of A
  int skinny_slices;    // k-slices of the A Q product
  bool tc_skinny;       // iteration products on the tensor cores (needs the bf16 splits)
  // workspace carve-up (byte offsets from ws)
  size_t off_A, off_Q, off_Y, off_T, off_gram, off_small, off_syrk, off_Ah, off_Al, off_Qs, total;
};
// no_split: one token range for A and one k-slice for A Q (smallest workspace)
void refresh_plan(int64_t N, int64_t d, int rank, int oversample, bool a_out_given, RefreshPlan* p,
                  bool no_split = false);
cudaError_t launch_refresh(const RefreshPlan& p, const void* X, gift_dtype xdt, float* U, float* lambda,
                           float* rho, float* A_out, void* ws, uint32_t* dev_status, cudaStream_t s);
// ---- A = X^T X / N of many layers in one tensor-core launch (syrk_tc.cu) ----
struct SyrkJob {
  const void* X;
  gift_dtype xdt;
  int64_t N;
  int d;
  float* A;
  uint32_t* err;
};
// Every job with bf16 X and d % 128 == 0 is computed (token range never split,
// so a layer's A does not depend on what it is batched with) and gets
// used[i] = true; the others are left to the caller.  n <= 64.
cudaError_t launch_syrk_tc_batch(const SyrkJob* jobs, int n, cudaStream_t s, bool* used);

// A Q on the tensor cores (bf16 hi/lo split operands), one k-slice per CTA row.
constexpr int kSkinnyMaxBatch = 48;
struct SkinnyTcJob {
  const void* Ah;  // bf16 d x d
  const void* Al;  // bf16 d x d
  const void* Qs;  // bf16 d x 128: [Q_hi (64) | Q_lo (64)]
  float* Yp;       // ns k-slices of d x m fp32
  int d, ns, kslice;
};
cudaError_t launch_skinny_tc(const SkinnyTcJob* jobs, int n, int m, cudaStream_t s);

// Many refreshes in one sequence of launches (same rank, oversample, iters).
struct RefreshIO {
  const void* X;
  gift_dtype xdt;
  float* U;
  float* lambda;
  float* rho;
  float* A_out;
  void* ws;
  uint32_t* dev_status;
};
cudaError_t launch_refresh_batch(const RefreshPlan* plans, const RefreshIO* io, int n, cudaStream_t s);

}  // namespace gift
