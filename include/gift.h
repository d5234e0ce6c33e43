/*
 * gift.h — C ABI of the B200 (sm_100a) GIFT gradient codec.
 *
 * GIFT: Geometry-Informed Low-precision Gradient Communication for LLM
 * Pretraining (arXiv 2607.07494).  Per linear layer, the gradient G
 * (d_out x d_in) is moved into coordinates whitened on its input side by a
 * rank-r approximation of the K-FAC input factor A = X^T X / N, quantised
 * (FP8 E4M3 with one fp32 scale per 128 contiguous elements of a row, or
 * NVFP4), dequantised on the far side and mapped back (review page, "What
 * carries the argument"; abstract).  The rank is 32 (section V.B, Table II);
 * the factor is refreshed every K = 50 steps (section V.E, Algorithm 1).
 *
 * The pages do not print the transform.  This library uses
 *     M      = rho^{-1/2} I + U diag(c)  U^T,  c_k  = (lambda_k+rho)^{-1/2} - rho^{-1/2}
 *     M^{-1} = rho^{+1/2} I + U diag(c') U^T,  c'_k = (lambda_k+rho)^{+1/2} - rho^{+1/2}
 * with (U, lambda) the top-r eigenpairs of A and rho the mean of A's other
 * eigenvalues, i.e. M = (U diag(lambda) U^T + rho I)^{-1/2} for orthonormal U.
 * Encode: W = G M, per-block E4M3.  Decode: G_hat = W_hat M^{-1}.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller, except where
 *    a comment says "host".  The library never allocates device memory:
 *    scratch space is the caller's `ws`, sized by the *_workspace_size calls.
 *  - Layouts are row-major and dense: G, G_hat, codes are d_out x d_in (row
 *    stride d_in elements); scales are d_out x (d_in/128); X is N x d_in;
 *    U is d_in x rank fp32 (row stride rank); A_out is d_in x d_in fp32.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *    and runs entirely on the current device; there is no host round trip,
 *    so refresh -> encode -> decode chains need no synchronisation.
 *  - Host-detectable errors (null pointers, bad enums, shapes, alignment,
 *    workspace too small) return a status before anything is launched and
 *    before any CUDA call, so they can be checked without a GPU.  Launch
 *    failures return GIFT_ERR_CUDA.  Numerical conditions found on the
 *    device are OR-ed into the caller's `dev_status` word (GIFT_DEV_* bits);
 *    no kernel traps.
 *  - rank == 0 selects the Euclidean codec (M = I): U, lambda, rho ignored.
 *  - The library keeps no state between calls except a per-process cache of
 *    device properties; calls are re-entrant.
 */
#ifndef GIFT_H_
#define GIFT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* gift_stream_t;

typedef enum {
  GIFT_OK = 0,
  GIFT_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative or zero size */
  GIFT_ERR_SHAPE = 2,       /* d_in not a multiple of the block, rank too large, ... */
  GIFT_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  GIFT_ERR_WORKSPACE = 4,   /* ws == NULL or ws_bytes below the required size */
  GIFT_ERR_CUDA = 5,        /* a CUDA runtime call or a launch failed */
  GIFT_ERR_UNSUPPORTED = 6  /* the current device is not sm_100 */
} gift_status;

typedef enum { GIFT_F32 = 0, GIFT_BF16 = 1 } gift_dtype;

/* Bits OR-ed into the caller's *dev_status word (device memory, 4-byte
 * aligned; the caller zeroes it, calls only OR bits in).
 *   refresh: RHO_FLOORED, RANK_DEFICIENT, NONFINITE (A, lambda or rho),
 *            TIMEOUT (tensor-core syrk);
 *   encode:  NONFINITE (a block maximum of W, or the NVFP4 tensor maximum,
 *            is NaN or infinite: that block is coded as flushed, scale 0 and
 *            codes 0), TIMEOUT (tensor-core whitened encoder);
 *   decode:  NONFINITE (a block scale, or the NVFP4 tensor scale, is NaN or
 *            infinite), TIMEOUT (tensor-core whitened decoder). */
#define GIFT_DEV_RHO_FLOORED 0x1u    /* rho <= 2^-24 lambda_1: floored to that value */
#define GIFT_DEV_RANK_DEFICIENT 0x2u /* a Cholesky-QR pivot vanished: the sampled
                                        subspace has lower rank; that column is zeroed */
#define GIFT_DEV_NONFINITE 0x4u      /* a non-finite value reached the call's arithmetic */
#define GIFT_DEV_TIMEOUT 0x8u        /* a pipeline wait inside a kernel gave up after its
                                        iteration bound; the outputs of that call are undefined */

#define GIFT_E4M3_BLOCK 128
#define GIFT_NVFP4_BLOCK 16
#define GIFT_MAX_RANK 32             /* encode/decode: 0 <= rank <= 32 */
#define GIFT_MAX_SUBSPACE 64         /* refresh: rank + oversample <= 64 */

const char* gift_status_string(gift_status s);

/* Library version, e.g. 200 for 0.2.0.  GIFT_VERSION is the version this
 * header describes; a caller can compare it with gift_version() at run time
 * (0.2.0: dev_status on every codec call, gift_layer.U_split, gift_split_u,
 * the dense-transform and decode-and-sum calls; 0.2.1: gift_split_u_many). */
#define GIFT_VERSION 201
int gift_version(void);

/* ------------------------------------------------------------------------
 * Factor refresh (section V.E, Algorithm 1: the input-side factor is
 * recomputed every K steps; rank 32 from section V.B).
 *
 *   A = X^T X / N                       (bf16 or fp32 X, fp32 accumulation)
 *   Omega[i][j] = +-1 from SplitMix64(seed ^ (i*m + j)), m = rank+oversample
 *   Q = orth(Omega); repeat `iters` times: Q = orth(A Q)   (Cholesky-QR2)
 *   B = Q^T A Q; (theta, V) = eig(B) descending; lambda = theta[0:rank];
 *   U = Q V[:, 0:rank]; rho = (trace A - sum lambda) / (d_in - rank),
 *   floored at 2^-24 lambda_1 (GIFT_DEV_RHO_FLOORED).
 *
 * X: N x d_in, dtype xdt, 16-byte aligned.  Requires N >= 1,
 * d_in % 128 == 0, 1 <= rank, rank + oversample <= 64 and <= d_in.
 * Outputs: U (d_in x rank fp32), lambda (rank fp32, descending), rho (1 fp32);
 * A_out (d_in x d_in fp32, full symmetric) if non-NULL, else A lives in ws.
 * dev_status may be NULL; bits are OR-ed in (the caller zeroes it).
 * ------------------------------------------------------------------------ */
gift_status gift_refresh_workspace_size(int64_t N, int64_t d_in, int rank, int oversample,
                                        int a_out_given, size_t* bytes /* host */);

gift_status gift_factor_refresh(const void* X, gift_dtype xdt, int64_t N, int64_t d_in, int rank,
                                int oversample, int iters, uint64_t seed, float* U, float* lambda,
                                float* rho, float* A_out, void* ws, size_t ws_bytes,
                                uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Refresh of many layers at once (section V.E, Algorithm 1 refreshes the
 * factors of all whitened layers every K steps).  Same computation per job
 * as gift_factor_refresh; the A = X^T X / N contraction runs per layer and
 * all small fp64 steps of all layers run side by side (one CTA per layer),
 * so the latency of n refreshes is close to that of one.
 * `jobs` is a HOST array of n entries; every job has its own workspace of
 * gift_refresh_workspace_size(N, d_in, rank, oversample, A_out != NULL)
 * bytes.  rank, oversample and iters are shared by all jobs.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* X;          /* N x d_in, dtype xdt */
  int32_t xdt;            /* gift_dtype */
  int32_t reserved;       /* 0 */
  int64_t N;
  int64_t d_in;
  uint64_t seed;
  float* U;               /* d_in x rank */
  float* lambda;          /* rank */
  float* rho;             /* 1 */
  float* A_out;           /* nullable, d_in x d_in */
  void* ws;
  size_t ws_bytes;
  uint32_t* dev_status;   /* nullable */
} gift_refresh_job;

gift_status gift_factor_refresh_many(const gift_refresh_job* jobs /* host */, int n, int rank, int oversample,
                                     int iters, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Factor refresh without any allocation.  The paper has no counterpart: this
 * entry point exists for callers that cannot hand the library a workspace,
 * e.g. code whose device memory is entirely owned by another allocator, or
 * a step that must not call cudaMalloc because it can synchronise the
 * device.  It computes exactly what gift_factor_refresh computes, with its
 * scratch in a fixed array inside the library (present on every GPU that
 * loads libgift, until the process exits; nothing is allocated per call).
 *
 * Same arguments as gift_factor_refresh without ws/ws_bytes, except that
 * A_out is REQUIRED (d_in x d_in fp32, written in full).  Limits:
 * d_in <= 4096 and rank + oversample <= 64 (GIFT_ERR_SHAPE beyond them);
 * the token range is never split, so small layers use fewer SMs than
 * gift_factor_refresh would.
 * Set-up: the first call on each device looks up the array's device address
 * with that device current; make that first call before any stream capture.
 * The address is looked up again when the device's context is no longer the
 * one it was found in (after cudaDeviceReset, for example), so the library
 * may be used across a device reset; such a call is again a first call.
 * Every call on a device shares the one array and leaves its contents
 * behind; no value in it needs to start at zero.  Calls whose executions
 * overlap on the GPU (different streams, or different host threads) race
 * on the array and produce undefined results: serialise them.
 * ------------------------------------------------------------------------ */
gift_status gift_factor_refresh_noalloc(const void* X, gift_dtype xdt, int64_t N, int64_t d_in, int rank,
                                        int oversample, int iters, uint64_t seed, float* U, float* lambda,
                                        float* rho, float* A_out, uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Encode (review page, "What carries the argument": whiten with the
 * input-side factor before FP8 quantisation and communication).
 *
 *   W = G M  (fp32),  per row and per block b of 128 columns:
 *   amax = max |W|;  scales[b] = amax / 448;
 *   codes = E4M3_RNE_satfinite(W * (448 / amax))   (all 0x00 when amax == 0)
 *
 * G: d_out x d_in (GIFT_BF16 or GIFT_F32).  codes: d_out x d_in bytes.
 * scales: d_out x (d_in/128) fp32.  U/lambda/rho as produced by the refresh
 * (rho > 0 and finite); 0 <= rank <= 32.  d_in % 128 == 0, d_out >= 1.
 * dev_status (nullable): GIFT_DEV_NONFINITE, GIFT_DEV_TIMEOUT.
 * ------------------------------------------------------------------------ */
gift_status gift_encode(const void* G, gift_dtype gdt, int64_t d_out, int64_t d_in, const float* U,
                        const float* lambda, const float* rho, int rank, uint8_t* codes,
                        float* scales, uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Decode ("applies the inverse transform afterward").
 *
 *   W_hat = E4M3_value(codes) * scales (per block);  G_hat = W_hat M^{-1},
 *   written as out_dt (bf16 by round-to-nearest-even, or fp32).
 * dev_status (nullable): GIFT_DEV_NONFINITE, GIFT_DEV_TIMEOUT.
 * ------------------------------------------------------------------------ */
gift_status gift_decode(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                        const float* U, const float* lambda, const float* rho, int rank,
                        void* G_hat, gift_dtype out_dt, uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Grouped encode / decode over many layers in as few launches as possible
 * (selective deployment: whitened layers have rank 32, the others rank 0;
 * section V.C, Fig. 3 / Fig. 4).  `layers` is a HOST array of n entries;
 * each entry follows the rules of gift_encode / gift_decode.  Encode reads
 * G and writes codes/scales; decode reads codes/scales and writes G_hat.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* G;       /* encode input */
  void* G_hat;         /* decode output */
  uint8_t* codes;      /* encode output / decode input */
  float* scales;       /* encode output / decode input */
  const float* U;      /* d_in x rank, ignored when rank == 0 */
  const float* lambda; /* rank */
  const float* rho;    /* 1 */
  int64_t d_out;
  int64_t d_in;
  int32_t rank;        /* 0 (Euclidean) or 1..32 */
  int32_t dtype;       /* gift_dtype of G and G_hat */
  /* Optional (NULL: unused): U split once by gift_split_u after the factor
   * refresh.  The tensor-core codec (bf16, rank 32, d_in % 128 == 0) then
   * loads it as it is instead of splitting U in every launch; the results are
   * bit-identical either way.  Must be the split of this layer's current U.
   * Ignored by the other paths (which read U). */
  const uint16_t* U_split;
} gift_layer;

/* ------------------------------------------------------------------------
 * U split for the tensor-core codec (an implementation format, not part of
 * the method): U_split = [2][d_in][64] 16-bit words, device, 16-byte
 * aligned, caller-owned.  Row i of part 0 is [bf16(U_i) | bf16(U_i -
 * bf16(U_i))] (32 + 32 values, round to nearest even), row i of part 1 is
 * [f16(U_i) | f16((U_i - f16(U_i)) 2^11)].  U: d_in x 32 fp32, device,
 * 16-byte aligned.  rank must be 32.  Asynchronous on `stream`.
 * Errors: GIFT_ERR_INVALID_ARG (null pointer, rank != 32, d_in < 1),
 * GIFT_ERR_ALIGN, GIFT_ERR_CUDA.
 * ------------------------------------------------------------------------ */
gift_status gift_split_u(const float* U, int64_t d_in, int rank, uint16_t* U_split, gift_stream_t stream);

/* The same split for every layer of `layers` whose U_split is non-NULL and
 * rank is 32 (others are skipped), in one launch: after a batched factor
 * refresh, one call refreshes the splits of a whole grouped codec's layer
 * array.  Per layer the result is that of gift_split_u (bit-identical).
 * layers: host array of n descriptors (read during the call only); U and
 * U_split as for gift_split_u.  n == 0 is a no-op.
 * Errors: GIFT_ERR_INVALID_ARG (layers NULL with n > 0, n < 0, a U_split
 * layer with U NULL or d_in < 1), GIFT_ERR_ALIGN, GIFT_ERR_CUDA.  Nothing is
 * launched when an argument check fails. */
gift_status gift_split_u_many(const gift_layer* layers, int n, gift_stream_t stream);

/* dev_status (nullable): one word for the whole call, bits as for gift_encode
 * / gift_decode; a TIMEOUT leaves the outputs of every layer undefined. */
gift_status gift_encode_many(const gift_layer* layers /* host */, int n, uint32_t* dev_status,
                             gift_stream_t stream);
gift_status gift_decode_many(const gift_layer* layers /* host */, int n, uint32_t* dev_status,
                             gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Decode-and-sum for data-parallel training (review page, referee report on
 * section II.A, Eq. (1): the per-rank gradients g^(r); abstract: the
 * communication collective is left unchanged).  Every rank codes its own
 * gradient with the shared factor (gift_encode), the codes and scales of
 * all ranks are all-gathered by the caller's collective, and each rank forms
 *
 *   G_hat = alpha * sum_r W_hat_r M^{-1}  =  alpha * (sum_r W_hat_r) M^{-1}
 *
 * (M^{-1} is linear, so it is applied once, to the fp32 sum of the
 * dequantised parts, added in part order).  alpha = 1 gives the sum,
 * 1 / n_parts the mean.  codes / scales: HOST arrays of n_parts DEVICE
 * pointers, each laid out as gift_decode's codes and scales; 1 <= n_parts
 * <= 64.  Other arguments, layouts and alignment as for gift_decode (rank 0:
 * the Euclidean codec, M = I).  Runs on the CUDA cores.
 * dev_status (nullable): GIFT_DEV_NONFINITE (a non-finite scale).
 * ------------------------------------------------------------------------ */
gift_status gift_decode_sum(const uint8_t* const* codes /* host */, const float* const* scales /* host */,
                            int n_parts, int64_t d_out, int64_t d_in, const float* U, const float* lambda,
                            const float* rho, int rank, float alpha, void* G_hat, gift_dtype out_dt,
                            uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Test hook of the codec's failure path (the pages have no counterpart).
 * Launches the tensor-core whitened encoder (encode != 0) or decoder on one
 * layer (bf16, rank 32, d_in <= 8192) with one extra wait before any work:
 * one thread of every CTA waits at most stall_polls polls on a barrier that
 * nothing arrives at, the wait runs out, every CTA skips the layer's work
 * and returns, and GIFT_DEV_TIMEOUT is OR-ed into *dev_status.  Nothing is
 * loaded, computed or written and the context stays usable, so a test can
 * check that a bounded wait that gives up is reported to the caller.
 * Errors: GIFT_ERR_INVALID_ARG (null layer or dev_status, stall_polls == 0,
 * empty layer, rank 0), the argument checks of gift_encode / gift_decode,
 * GIFT_ERR_UNSUPPORTED (the layer does not take the tensor-core path).
 * ------------------------------------------------------------------------ */
gift_status gift_codec_stall_test(const gift_layer* layer /* host */, int encode, uint32_t stall_polls,
                                  uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Planning query (launches nothing, reads no pointer of `layers`): how the
 * tensor-core whitened codec lays out its first launch over these layers.
 * A 128-row panel is one CTA's work in the pages' per-layer round trip; when
 * a launch holds too few panels to fill the GPU (a single layer, say), the
 * codec gives each panel to a thread-block cluster of 2 or 4 CTAs that split
 * its 128-column chunks and add their partial projections G U (decode: W_hat
 * U) in cluster-rank order.  The pages have no counterpart: this is a layout
 * decision of this implementation.
 *   encode: nonzero for the encoder's plan, 0 for the decoder's.
 *   *split (host): 1, 2 or 4, or 0 if no layer takes the tensor-core path
 *   (bf16, rank 32, d_in <= 8192).
 * Errors: GIFT_ERR_INVALID_ARG (null split, n < 0, null layers with n > 0),
 * GIFT_ERR_SHAPE (d_in not a positive multiple of 128, d_out < 0),
 * GIFT_ERR_CUDA (no usable device).
 * ------------------------------------------------------------------------ */
gift_status gift_codec_split(const gift_layer* layers /* host */, int n, int encode, int* split /* host */);

/* ------------------------------------------------------------------------
 * One-step round-trip error (Tables I-II: relative reconstruction error of
 * the FP8 round trip against the full-precision gradient).
 *
 *   out[0] = ||G_hat - G||_F / ||G||_F,  out[1] = ||G_hat - G||_F^2,
 *   out[2] = ||G||_F^2, all accumulated in fp64 in a fixed order
 *   (deterministic).  out: 3 doubles on the device.
 * ------------------------------------------------------------------------ */
gift_status gift_error_workspace_size(int64_t d_out, int64_t d_in, size_t* bytes /* host */);

gift_status gift_roundtrip_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out,
                                 int64_t d_in, double* out, void* ws, size_t ws_bytes,
                                 gift_stream_t stream);

/* ------------------------------------------------------------------------
 * The same error in whitened coordinates (the geometry-aware norm in which
 * the review page's "direction-dependent distortion" is measured):
 *
 *   out[0] = ||(G_hat - G) M||_F / ||G M||_F,  out[1] = ||(G_hat - G) M||_F^2,
 *   out[2] = ||G M||_F^2,
 *
 * M = rho^{-1/2} I + U diag((lambda + rho)^{-1/2} - rho^{-1/2}) U^T from the
 * factor (U, lambda, rho) given here (rank 0: M = I, the plain relative
 * error).  fp32 products, fp64 sums in a fixed order (deterministic).
 * G, G_hat: d_out x d_in, dtype dt, 16-byte aligned; U: d_in x rank fp32,
 * 16-byte aligned; out: 3 doubles on the device; ws: device scratch of at
 * least gift_whitened_error_workspace_size bytes, 16-byte aligned.
 * Errors: GIFT_ERR_INVALID_ARG (null pointer, bad dtype), GIFT_ERR_SHAPE
 * (d_in not a multiple of 128, rank outside 0..32 or above d_in),
 * GIFT_ERR_WORKSPACE, GIFT_ERR_ALIGN, GIFT_ERR_CUDA.
 * ------------------------------------------------------------------------ */
gift_status gift_whitened_error_workspace_size(int64_t d_out, int64_t d_in, size_t* bytes /* host */);

gift_status gift_whitened_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out, int64_t d_in,
                                const float* U, const float* lambda, const float* rho, int rank, double* out,
                                void* ws, size_t ws_bytes, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 codec (abstract: NVFP4 is the second low-precision format the
 * whitening is applied to).  The pages give no recipe; this library uses the
 * two-level one of the NVFP4 format, decisions in fp32:
 *
 *   W = G (rank 0) or G M (rank 32);  S_t = amax(W) / (6 * 448);
 *   per row and block b of 16 columns:  amax_b = max |W|,
 *   block_scales[b] = E4M3_RNE_satfinite(amax_b / (6 S_t));
 *   codes = E2M1_RNE_satfinite(W * (1 / (value(block_scales[b]) * S_t)))
 *   (a block whose scale decodes to 0, or whose reciprocal overflows fp32,
 *   gets scale code 0 and all-zero codes).
 *
 * codes: d_out x d_in/2 bytes, two E2M1 codes per byte, column 2i in the low
 * nibble, 16-byte aligned.  block_scales: d_out x d_in/16 E4M3 bytes, 8-byte
 * aligned.  tensor_scale: one fp32 in device memory, 4-byte aligned.
 * Encode needs the tensor-wide maximum before any block is coded, so it
 * makes two passes over W (the first folds amax(W) into *tensor_scale, the
 * second writes the codes, then *tensor_scale becomes S_t); *tensor_scale
 * holds intermediate values while the call's work runs.
 * rank must be 0 (any dtype, d_in % 16 == 0) or 32 with bf16 G / G_hat and
 * d_in % 128 == 0, d_in <= 8192 (tensor-core path); other ranks return
 * GIFT_ERR_UNSUPPORTED.  G / G_hat and U 16-byte aligned.
 * Decode: G_hat = W_hat (rank 0) or W_hat M^{-1} with
 * W_hat = value(code) * value(block scale) * S_t.
 * dev_status (nullable): GIFT_DEV_NONFINITE (amax(W) or S_t not finite),
 * GIFT_DEV_TIMEOUT (tensor-core path).
 * ------------------------------------------------------------------------ */
gift_status gift_encode_nvfp4(const void* G, gift_dtype gdt, int64_t d_out, int64_t d_in, const float* U,
                              const float* lambda, const float* rho, int rank, uint8_t* codes,
                              uint8_t* block_scales, float* tensor_scale, uint32_t* dev_status,
                              gift_stream_t stream);

gift_status gift_decode_nvfp4(const uint8_t* codes, const uint8_t* block_scales, const float* tensor_scale,
                              int64_t d_out, int64_t d_in, const float* U, const float* lambda,
                              const float* rho, int rank, void* G_hat, gift_dtype out_dt,
                              uint32_t* dev_status, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * Dense input-side transforms: the variants GIFT is simplified from (review
 * page, "What carries the argument": full two-sided K-FAC whitening, then
 * the input side alone at full rank (Fig. 2 caption), then rank 32; section
 * IV.A, Eq. (14) writes the input side with the Cholesky factor L_A^{-T}).
 *
 * gift_dense_factor: from A (d x d fp32, symmetric positive definite, e.g.
 * A_out of gift_factor_refresh), in fp64:
 *   GIFT_DENSE_CHOLESKY: A = L L^T, M = L^{-T}, M_inv = L^T (both upper
 *                        triangular; W = G M has input-side covariance I);
 *   GIFT_DENSE_INVSQRT:  M = A^{-1/2}, M_inv = A^{1/2} (coupled Newton-Schulz
 *                        iteration, at most 60 steps; the rank-r construction
 *                        of gift_encode at r = d_in).
 * Outputs (device, d x d, row-major): M, M_inv in fp32; M_split as three bf16
 * parts [hi ; mid ; lo] (3 x d x d, x ~ hi + mid + lo, each part the bf16
 * rounding of what the earlier ones leave) and M_inv_split as a bf16 pair
 * [hi ; lo] (2 x d x d): the operands of gift_dense_encode / gift_dense_decode.
 * (The entries of a whitening transform are large next to W = G M, whose sum
 * cancels, so the encoder takes M to fp32 accuracy; G_hat needs less.)  d % 128 == 0, 128 <= d <= 8192.
 * ws: device scratch of gift_dense_factor_workspace_size bytes, 16-byte
 * aligned.  dev_status (nullable): GIFT_DEV_RANK_DEFICIENT (a non-positive
 * Cholesky pivot, replaced by a tiny one), GIFT_DEV_NONFINITE.
 * Errors: GIFT_ERR_INVALID_ARG (null pointer, bad kind), GIFT_ERR_SHAPE,
 * GIFT_ERR_WORKSPACE, GIFT_ERR_ALIGN, GIFT_ERR_CUDA.
 * ------------------------------------------------------------------------ */
#define GIFT_DENSE_CHOLESKY 1
#define GIFT_DENSE_INVSQRT 2

gift_status gift_dense_factor_workspace_size(int64_t d, int kind, size_t* bytes /* host */);

gift_status gift_dense_factor(const float* A, int64_t d, int kind, float* M, float* M_inv, uint16_t* M_split,
                              uint16_t* M_inv_split, void* ws, size_t ws_bytes, uint32_t* dev_status,
                              gift_stream_t stream);

/* fp32 d x d matrix -> its `parts` bf16 parts (2: [hi ; lo], 3: [hi ; mid ;
 * lo]) as gift_dense_factor writes them, for a transform made elsewhere. */
gift_status gift_dense_split(const float* M, int64_t d, int parts, uint16_t* M_split, gift_stream_t stream);

/* ------------------------------------------------------------------------
 * E4M3 codec under a dense transform (tensor cores, bf16 gradients):
 *   encode  W = G M; per row and block of 128 columns, scales = amax/448 and
 *           codes = E4M3_RNE_satfinite(W * (448/amax)) as in gift_encode;
 *   decode  G_hat = W_hat M_inv, W_hat = value(codes) * scale per block,
 *           written as out_dt (bf16 by round-to-nearest-even, or fp32).
 * G: d_out x d_in bf16.  M_split: the three bf16 parts [hi ; mid ; lo] of M,
 * M_inv_split: the bf16 pair [hi ; lo] of M^{-1}, each part d_in x d_in.  upper_triangular != 0 declares M (M_inv) upper triangular
 * (the Cholesky form), so products skip its zero blocks.  d_in % 128 == 0,
 * 128 <= d_in <= 8192, d_out >= 0.  All pointers 16-byte aligned except
 * dev_status (4).  dev_status (nullable): GIFT_DEV_NONFINITE,
 * GIFT_DEV_TIMEOUT.  Errors: GIFT_ERR_INVALID_ARG, GIFT_ERR_SHAPE,
 * GIFT_ERR_ALIGN, GIFT_ERR_CUDA.
 * ------------------------------------------------------------------------ */
gift_status gift_dense_encode(const void* G, int64_t d_out, int64_t d_in, const uint16_t* M_split,
                              int upper_triangular, uint8_t* codes, float* scales, uint32_t* dev_status,
                              gift_stream_t stream);

gift_status gift_dense_decode(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                              const uint16_t* M_inv_split, int upper_triangular, void* G_hat, gift_dtype out_dt,
                              uint32_t* dev_status, gift_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GIFT_H_ */
