// C-ABI entry points of libgift (declared in include/gift.h).
//
// Each entry point validates every argument on the host first and returns a
// status before touching CUDA, so argument errors are reported identically
// with or without a GPU.  Only then does it check the device (sm_100) and
// enqueue kernels on the caller's stream.  Nothing here allocates device
// memory; scratch space comes from the caller's workspace.
#include <cstdio>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

using namespace gift;

namespace {

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
inline bool dtype_ok(int d) { return d == GIFT_F32 || d == GIFT_BF16; }

constexpr int kMaxDevices = 64;

// sm_100 check, cached per device (the only state the library keeps).
gift_status device_ok() {
  static int major_cache[kMaxDevices];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < kMaxDevices; ++i) major_cache[i] = -1;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GIFT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GIFT_ERR_UNSUPPORTED;
  int major = major_cache[dev];
  if (major < 0) {
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GIFT_ERR_CUDA;
    major_cache[dev] = major;
  }
  return major == 10 ? GIFT_OK : GIFT_ERR_UNSUPPORTED;
}

inline gift_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GIFT_OK : GIFT_ERR_CUDA; }

gift_status check_codec_args(const void* G, int gdt, int64_t d_out, int64_t d_in, const float* U,
                             const float* lambda, const float* rho, int rank, const void* codes, const float* scales) {
  if (!dtype_ok(gdt)) return GIFT_ERR_INVALID_ARG;
  if (d_out < 0 || d_in <= 0) return GIFT_ERR_INVALID_ARG;
  if (d_in % GIFT_E4M3_BLOCK != 0) return GIFT_ERR_SHAPE;
  if (d_in > (1 << 20) || d_out > ((int64_t)1 << 31)) return GIFT_ERR_SHAPE;
  if (rank < 0 || rank > GIFT_MAX_RANK) return GIFT_ERR_SHAPE;
  if (d_out == 0) return GIFT_OK;  // empty gradient: nothing is read or written
  if (!G || !codes || !scales) return GIFT_ERR_INVALID_ARG;
  if (rank > 0 && (!U || !lambda || !rho)) return GIFT_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(codes) || !aligned16(scales)) return GIFT_ERR_ALIGN;
  if (rank > 0 && (!aligned16(U) || !aligned(lambda, 4) || !aligned(rho, 4))) return GIFT_ERR_ALIGN;
  return GIFT_OK;
}

// Whitened bf16 layers with rank 32 go to the tensor-core kernels when they
// are built in; everything else runs on the CUDA-core kernels.
inline bool use_tc(int dt, int rank, int64_t d_in) {
  return dt == GIFT_BF16 && rank == GIFT_MAX_RANK && tc_codec_available() && d_in <= 8192;
}

}  // namespace

extern "C" {

const char* gift_status_string(gift_status s) {
  switch (s) {
    case GIFT_OK: return "GIFT_OK";
    case GIFT_ERR_INVALID_ARG: return "GIFT_ERR_INVALID_ARG: null pointer, bad enum or bad size";
    case GIFT_ERR_SHAPE: return "GIFT_ERR_SHAPE: unsupported shape or rank";
    case GIFT_ERR_ALIGN: return "GIFT_ERR_ALIGN: pointer not 16-byte aligned";
    case GIFT_ERR_WORKSPACE: return "GIFT_ERR_WORKSPACE: workspace missing or too small";
    case GIFT_ERR_CUDA: return "GIFT_ERR_CUDA: CUDA runtime or launch failure";
    case GIFT_ERR_UNSUPPORTED: return "GIFT_ERR_UNSUPPORTED: device is not sm_100";
  }
  return "GIFT_ERR_UNKNOWN";
}

int gift_version(void) { return GIFT_VERSION; }

// ---------------------------------------------------------------------------
gift_status gift_refresh_workspace_size(int64_t N, int64_t d_in, int rank, int oversample, int a_out_given,
                                        size_t* bytes) {
  if (!bytes) return GIFT_ERR_INVALID_ARG;
  if (N < 1 || d_in <= 0 || rank < 1 || oversample < 0) return GIFT_ERR_INVALID_ARG;
  if (d_in % GIFT_E4M3_BLOCK != 0 || d_in > 32768) return GIFT_ERR_SHAPE;
  if (rank + oversample > GIFT_MAX_SUBSPACE || rank + oversample > d_in) return GIFT_ERR_SHAPE;
  RefreshPlan p;
  refresh_plan(N, d_in, rank, oversample, a_out_given != 0, &p);
  *bytes = p.total;
  return GIFT_OK;
}

gift_status gift_factor_refresh(const void* X, gift_dtype xdt, int64_t N, int64_t d_in, int rank, int oversample,
                                int iters, uint64_t seed, float* U, float* lambda, float* rho, float* A_out,
                                void* ws, size_t ws_bytes, uint32_t* dev_status, gift_stream_t stream) {
  if (!X || !U || !lambda || !rho) return GIFT_ERR_INVALID_ARG;
  if (!dtype_ok(xdt)) return GIFT_ERR_INVALID_ARG;
  if (iters < 0 || iters > 1000) return GIFT_ERR_INVALID_ARG;
  size_t need = 0;
  gift_status st = gift_refresh_workspace_size(N, d_in, rank, oversample, A_out != nullptr, &need);
  if (st != GIFT_OK) return st;
  if (need > 0 && (!ws || ws_bytes < need)) return GIFT_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(U) || !aligned(lambda, 4) || !aligned(rho, 4)) return GIFT_ERR_ALIGN;
  if ((A_out && !aligned16(A_out)) || (ws && !aligned16(ws)) || (dev_status && !aligned(dev_status, 4)))
    return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  RefreshPlan p;
  refresh_plan(N, d_in, rank, oversample, A_out != nullptr, &p);
  p.iters = iters;
  p.seed = seed;
  return cuda_status(launch_refresh(p, X, xdt, U, lambda, rho, A_out, ws, dev_status, (cudaStream_t)stream));
}

gift_status gift_factor_refresh_many(const gift_refresh_job* jobs, int n, int rank, int oversample, int iters,
                                     gift_stream_t stream) {
  if (n < 0 || (n > 0 && !jobs)) return GIFT_ERR_INVALID_ARG;
  if (iters < 0 || iters > 1000) return GIFT_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const gift_refresh_job& J = jobs[i];
    if (!J.X || !J.U || !J.lambda || !J.rho) return GIFT_ERR_INVALID_ARG;
    if (!dtype_ok(J.xdt)) return GIFT_ERR_INVALID_ARG;
    size_t need = 0;
    gift_status st = gift_refresh_workspace_size(J.N, J.d_in, rank, oversample, J.A_out != nullptr, &need);
    if (st != GIFT_OK) return st;
    if (need > 0 && (!J.ws || J.ws_bytes < need)) return GIFT_ERR_WORKSPACE;
    if (!aligned16(J.X) || !aligned16(J.U) || !aligned(J.lambda, 4) || !aligned(J.rho, 4)) return GIFT_ERR_ALIGN;
    if ((J.A_out && !aligned16(J.A_out)) || (J.ws && !aligned16(J.ws)) ||
        (J.dev_status && !aligned(J.dev_status, 4)))
      return GIFT_ERR_ALIGN;
  }
  if (n == 0) return GIFT_OK;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  std::vector<RefreshPlan> plans(n);
  std::vector<RefreshIO> io(n);
  for (int i = 0; i < n; ++i) {
    const gift_refresh_job& J = jobs[i];
    refresh_plan(J.N, J.d_in, rank, oversample, J.A_out != nullptr, &plans[i]);
    plans[i].iters = iters;
    plans[i].seed = J.seed;
    io[i] = RefreshIO{J.X, (gift_dtype)J.xdt, J.U, J.lambda, J.rho, J.A_out, J.ws, J.dev_status};
  }
  return cuda_status(launch_refresh_batch(plans.data(), io.data(), n, (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------
gift_status gift_encode(const void* G, gift_dtype gdt, int64_t d_out, int64_t d_in, const float* U,
                        const float* lambda, const float* rho, int rank, uint8_t* codes, float* scales,
                        uint32_t* dev_status, gift_stream_t stream) {
  gift_status st = check_codec_args(G, gdt, d_out, d_in, U, lambda, rho, rank, codes, scales);
  if (st != GIFT_OK) return st;
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (d_out == 0) return GIFT_OK;
  if ((st = device_ok()) != GIFT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (rank == 0)
    return cuda_status(
        launch_euclid_encode(G, gdt, d_out * (d_in / GIFT_E4M3_BLOCK), codes, scales, dev_status, s));
  if (use_tc(gdt, rank, d_in)) {
    TcLayer L{G, nullptr, codes, scales, U, lambda, rho, (int)d_out, (int)d_in, rank};
    return cuda_status(launch_whiten_encode_tc(&L, 1, dev_status, s));
  }
  return cuda_status(
      launch_whiten_encode_simt(G, gdt, d_out, d_in, U, lambda, rho, rank, codes, scales, dev_status, s));
}

gift_status gift_decode(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in, const float* U,
                        const float* lambda, const float* rho, int rank, void* G_hat, gift_dtype out_dt,
                        uint32_t* dev_status, gift_stream_t stream) {
  gift_status st = check_codec_args(G_hat, out_dt, d_out, d_in, U, lambda, rho, rank, codes, scales);
  if (st != GIFT_OK) return st;
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (d_out == 0) return GIFT_OK;
  if ((st = device_ok()) != GIFT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (rank == 0)
    return cuda_status(
        launch_euclid_decode(codes, scales, d_out * (d_in / GIFT_E4M3_BLOCK), G_hat, out_dt, dev_status, s));
  if (use_tc(out_dt, rank, d_in)) {
    TcLayer L{nullptr, G_hat, (uint8_t*)codes, (float*)scales, U, lambda, rho, (int)d_out, (int)d_in, rank};
    return cuda_status(launch_whiten_decode_tc(&L, 1, dev_status, s));
  }
  return cuda_status(
      launch_whiten_decode_simt(codes, scales, d_out, d_in, U, lambda, rho, rank, G_hat, out_dt, dev_status, s));
}

// ---------------------------------------------------------------------------
static gift_status run_many(const gift_layer* layers, int n, uint32_t* dev_status, gift_stream_t stream,
                            bool encode) {
  if (n < 0 || (n > 0 && !layers)) return GIFT_ERR_INVALID_ARG;
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  for (int i = 0; i < n; ++i) {
    const gift_layer& L = layers[i];
    const void* g = encode ? L.G : (const void*)L.G_hat;
    gift_status st = check_codec_args(g, L.dtype, L.d_out, L.d_in, L.U, L.lambda, L.rho, L.rank, L.codes, L.scales);
    if (st != GIFT_OK) return st;
    if (L.U_split && !aligned16(L.U_split)) return GIFT_ERR_ALIGN;
  }
  if (n == 0) return GIFT_OK;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  std::vector<TcLayer> tc;
  std::vector<EuclidLayer> eu[2];  // by dtype
  for (int i = 0; i < n; ++i) {
    const gift_layer& L = layers[i];
    if (L.d_out == 0) continue;
    cudaError_t e = cudaSuccess;
    const int64_t nb = L.d_out * (L.d_in / GIFT_E4M3_BLOCK);
    if (L.rank == 0) {
      eu[L.dtype].push_back(encode ? EuclidLayer{L.G, L.codes, L.scales, nb}
                                   : EuclidLayer{L.codes, L.G_hat, L.scales, nb});
    } else if (use_tc(L.dtype, L.rank, L.d_in)) {
      tc.push_back(TcLayer{L.G, L.G_hat, L.codes, L.scales, L.U, L.lambda, L.rho, (int)L.d_out, (int)L.d_in, L.rank});
      tc.back().U_split = L.U_split;
    } else {
      e = encode ? launch_whiten_encode_simt(L.G, (gift_dtype)L.dtype, L.d_out, L.d_in, L.U, L.lambda, L.rho, L.rank,
                                             L.codes, L.scales, dev_status, s)
                 : launch_whiten_decode_simt(L.codes, L.scales, L.d_out, L.d_in, L.U, L.lambda, L.rho, L.rank,
                                             L.G_hat, (gift_dtype)L.dtype, dev_status, s);
    }
    if (e != cudaSuccess) return GIFT_ERR_CUDA;
  }
  for (int dt = 0; dt < 2; ++dt)
    if (!eu[dt].empty() &&
        launch_euclid_group(eu[dt].data(), (int)eu[dt].size(), (gift_dtype)dt, encode, dev_status, s) != cudaSuccess)
      return GIFT_ERR_CUDA;
  if (!tc.empty()) {
    cudaError_t e = encode ? launch_whiten_encode_tc(tc.data(), (int)tc.size(), dev_status, s)
                           : launch_whiten_decode_tc(tc.data(), (int)tc.size(), dev_status, s);
    if (e != cudaSuccess) return GIFT_ERR_CUDA;
  }
  return GIFT_OK;
}

gift_status gift_codec_split(const gift_layer* layers, int n, int encode, int* split) {
  if (!split || n < 0 || (n > 0 && !layers)) return GIFT_ERR_INVALID_ARG;
  std::vector<TcLayer> tc;
  for (int i = 0; i < n; ++i) {
    const gift_layer& L = layers[i];
    if (L.d_in < GIFT_E4M3_BLOCK || L.d_in % GIFT_E4M3_BLOCK != 0 || L.d_out < 0) return GIFT_ERR_SHAPE;
    if (L.d_out > 0 && L.rank > 0 && use_tc(L.dtype, L.rank, L.d_in)) {
      tc.push_back(TcLayer{L.G, L.G_hat, L.codes, L.scales, L.U, L.lambda, L.rho, (int)L.d_out, (int)L.d_in, L.rank});
      tc.back().U_split = L.U_split;
    }
  }
  *split = 0;
  if (tc.empty()) return GIFT_OK;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  const int S = tc_codec_split(tc.data(), (int)tc.size(), encode != 0);
  if (S < 1) return GIFT_ERR_SHAPE;
  *split = S;
  return GIFT_OK;
}

gift_status gift_split_u(const float* U, int64_t d_in, int rank, uint16_t* U_split, gift_stream_t stream) {
  if (!U || !U_split || rank != 32 || d_in < 1) return GIFT_ERR_INVALID_ARG;
  if (!aligned16(U) || !aligned16(U_split)) return GIFT_ERR_ALIGN;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  return cuda_status(launch_split_u(U, d_in, U_split, (cudaStream_t)stream));
}

gift_status gift_split_u_many(const gift_layer* layers, int n, gift_stream_t stream) {
  if (n < 0 || (n > 0 && !layers)) return GIFT_ERR_INVALID_ARG;
  std::vector<const float*> U;
  std::vector<uint16_t*> out;
  std::vector<int64_t> d;
  for (int i = 0; i < n; ++i) {
    const gift_layer& L = layers[i];
    if (!L.U_split || L.rank != 32) continue;
    if (!L.U || L.d_in < 1) return GIFT_ERR_INVALID_ARG;
    if (!aligned16(L.U) || !aligned16(L.U_split)) return GIFT_ERR_ALIGN;
    U.push_back(L.U);
    out.push_back(const_cast<uint16_t*>(L.U_split));
    d.push_back(L.d_in);
  }
  if (U.empty()) return GIFT_OK;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  return cuda_status(launch_split_u_many(U.data(), out.data(), d.data(), (int)U.size(), (cudaStream_t)stream));
}

gift_status gift_encode_many(const gift_layer* layers, int n, uint32_t* dev_status, gift_stream_t stream) {
  return run_many(layers, n, dev_status, stream, true);
}
gift_status gift_decode_many(const gift_layer* layers, int n, uint32_t* dev_status, gift_stream_t stream) {
  return run_many(layers, n, dev_status, stream, false);
}

gift_status gift_codec_stall_test(const gift_layer* layer, int encode, uint32_t stall_polls, uint32_t* dev_status,
                                  gift_stream_t stream) {
  if (!layer || !dev_status || stall_polls == 0) return GIFT_ERR_INVALID_ARG;
  const gift_layer& L = *layer;
  const void* g = encode ? L.G : (const void*)L.G_hat;
  gift_status st = check_codec_args(g, L.dtype, L.d_out, L.d_in, L.U, L.lambda, L.rho, L.rank, L.codes, L.scales);
  if (st != GIFT_OK) return st;
  if (!aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (L.d_out == 0 || L.rank == 0) return GIFT_ERR_INVALID_ARG;
  if ((st = device_ok()) != GIFT_OK) return st;
  if (!use_tc(L.dtype, L.rank, L.d_in)) return GIFT_ERR_UNSUPPORTED;
  if (L.U_split && !aligned16(L.U_split)) return GIFT_ERR_ALIGN;
  TcLayer T{L.G, L.G_hat, L.codes, L.scales, L.U, L.lambda, L.rho, (int)L.d_out, (int)L.d_in, L.rank};
  T.U_split = L.U_split;
  cudaStream_t s = (cudaStream_t)stream;
  return cuda_status(encode ? launch_whiten_encode_tc(&T, 1, dev_status, s, stall_polls)
                            : launch_whiten_decode_tc(&T, 1, dev_status, s, stall_polls));
}

// ---------------------------------------------------------------------------
gift_status gift_error_workspace_size(int64_t d_out, int64_t d_in, size_t* bytes) {
  if (!bytes || d_out < 1 || d_in < 1) return GIFT_ERR_INVALID_ARG;
  if (d_in % GIFT_E4M3_BLOCK != 0) return GIFT_ERR_SHAPE;
  *bytes = error_ws_bytes(d_out * d_in);
  return GIFT_OK;
}

gift_status gift_roundtrip_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out, int64_t d_in,
                                 double* out, void* ws, size_t ws_bytes, gift_stream_t stream) {
  if (!G || !G_hat || !out) return GIFT_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return GIFT_ERR_INVALID_ARG;
  size_t need = 0;
  gift_status st = gift_error_workspace_size(d_out, d_in, &need);
  if (st != GIFT_OK) return st;
  if (!ws || ws_bytes < need) return GIFT_ERR_WORKSPACE;
  if (!aligned16(G) || !aligned16(G_hat) || !aligned(out, 8) || !aligned16(ws)) return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  return cuda_status(launch_roundtrip_error(G, G_hat, dt, d_out * d_in, out, ws, (cudaStream_t)stream));
}

gift_status gift_whitened_error_workspace_size(int64_t d_out, int64_t d_in, size_t* bytes) {
  if (!bytes || d_out < 1 || d_in < 1) return GIFT_ERR_INVALID_ARG;
  if (d_in % GIFT_E4M3_BLOCK != 0) return GIFT_ERR_SHAPE;
  *bytes = whitened_error_ws_bytes(d_out);
  return GIFT_OK;
}

gift_status gift_whitened_error(const void* G, const void* G_hat, gift_dtype dt, int64_t d_out, int64_t d_in,
                                const float* U, const float* lambda, const float* rho, int rank, double* out,
                                void* ws, size_t ws_bytes, gift_stream_t stream) {
  if (!G || !G_hat || !out) return GIFT_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return GIFT_ERR_INVALID_ARG;
  if (rank < 0 || rank > GIFT_MAX_RANK) return GIFT_ERR_SHAPE;
  if (rank > 0 && (!U || !lambda || !rho)) return GIFT_ERR_INVALID_ARG;
  size_t need = 0;
  gift_status st = gift_whitened_error_workspace_size(d_out, d_in, &need);
  if (st != GIFT_OK) return st;
  if (rank > d_in) return GIFT_ERR_SHAPE;
  if (!ws || ws_bytes < need) return GIFT_ERR_WORKSPACE;
  if (!aligned16(G) || !aligned16(G_hat) || !aligned(out, 8) || !aligned16(ws)) return GIFT_ERR_ALIGN;
  if (rank > 0 && (!aligned16(U) || !aligned(lambda, 4) || !aligned(rho, 4))) return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  return cuda_status(launch_whitened_error(G, G_hat, dt, d_out, d_in, U, lambda, rho, rank, out, ws,
                                           (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------
static gift_status check_nvfp4_args(const void* G, int gdt, int64_t d_out, int64_t d_in, const float* U,
                                    const float* lambda, const float* rho, int rank, const void* codes,
                                    const void* sb, const float* ts) {
  if (!dtype_ok(gdt)) return GIFT_ERR_INVALID_ARG;
  if (d_out < 0 || d_in <= 0) return GIFT_ERR_INVALID_ARG;
  if (rank < 0 || rank > GIFT_MAX_RANK) return GIFT_ERR_SHAPE;
  if (d_in % GIFT_NVFP4_BLOCK != 0 || (rank > 0 && d_in % GIFT_E4M3_BLOCK != 0)) return GIFT_ERR_SHAPE;
  if (d_in > (1 << 20) || d_out > ((int64_t)1 << 31)) return GIFT_ERR_SHAPE;
  if (rank > 0 && (rank != GIFT_MAX_RANK || gdt != GIFT_BF16 || d_in > 8192)) return GIFT_ERR_UNSUPPORTED;
  if (d_out == 0) return GIFT_OK;  // empty gradient: nothing is read or written
  if (!G || !codes || !sb || !ts) return GIFT_ERR_INVALID_ARG;
  if (rank > 0 && (!U || !lambda || !rho)) return GIFT_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(codes) || !aligned(sb, 8) || !aligned(ts, 4)) return GIFT_ERR_ALIGN;
  if (rank > 0 && (!aligned16(U) || !aligned(lambda, 4) || !aligned(rho, 4))) return GIFT_ERR_ALIGN;
  return GIFT_OK;
}

gift_status gift_encode_nvfp4(const void* G, gift_dtype gdt, int64_t d_out, int64_t d_in, const float* U,
                              const float* lambda, const float* rho, int rank, uint8_t* codes,
                              uint8_t* block_scales, float* tensor_scale, uint32_t* dev_status, gift_stream_t stream) {
  gift_status st = check_nvfp4_args(G, gdt, d_out, d_in, U, lambda, rho, rank, codes, block_scales, tensor_scale);
  if (st != GIFT_OK) return st;
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (d_out == 0) return GIFT_OK;
  if ((st = device_ok()) != GIFT_OK) return st;
  if (rank > 0 && !tc_codec_available()) return GIFT_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  // *tensor_scale first accumulates amax(W) as the bits of a non-negative float
  if (cudaMemsetAsync(tensor_scale, 0, sizeof(float), s) != cudaSuccess) return GIFT_ERR_CUDA;
  if (rank == 0) {
    const int64_t nb = d_out * (d_in / GIFT_NVFP4_BLOCK);
    if ((st = cuda_status(launch_nvfp4_amax(G, gdt, nb, tensor_scale, s))) != GIFT_OK) return st;
    if ((st = cuda_status(launch_nvfp4_quant(G, gdt, nb, tensor_scale, codes, block_scales, s))) != GIFT_OK) return st;
  } else {
    TcLayer L{G, nullptr, codes, nullptr, U, lambda, rho, (int)d_out, (int)d_in, rank};
    L.block_scales = block_scales;
    L.tensor_scale = tensor_scale;
    L.fmt = kFmtNvfp4Amax;
    if ((st = cuda_status(launch_whiten_encode_tc(&L, 1, dev_status, s))) != GIFT_OK) return st;
    L.fmt = kFmtNvfp4;
    if ((st = cuda_status(launch_whiten_encode_tc(&L, 1, dev_status, s))) != GIFT_OK) return st;
  }
  return cuda_status(launch_nvfp4_finalize(tensor_scale, dev_status, s));
}

gift_status gift_decode_nvfp4(const uint8_t* codes, const uint8_t* block_scales, const float* tensor_scale,
                              int64_t d_out, int64_t d_in, const float* U, const float* lambda, const float* rho,
                              int rank, void* G_hat, gift_dtype out_dt, uint32_t* dev_status,
                              gift_stream_t stream) {
  gift_status st =
      check_nvfp4_args(G_hat, out_dt, d_out, d_in, U, lambda, rho, rank, codes, block_scales, tensor_scale);
  if (st != GIFT_OK) return st;
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (d_out == 0) return GIFT_OK;
  if ((st = device_ok()) != GIFT_OK) return st;
  if (rank > 0 && !tc_codec_available()) return GIFT_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if (rank == 0)
    return cuda_status(launch_nvfp4_decode(codes, block_scales, tensor_scale, d_out * (d_in / GIFT_NVFP4_BLOCK),
                                           G_hat, out_dt, dev_status, s));
  TcLayer L{nullptr, G_hat, (uint8_t*)codes, nullptr, U, lambda, rho, (int)d_out, (int)d_in, rank};
  L.block_scales = (uint8_t*)block_scales;
  L.tensor_scale = (float*)tensor_scale;
  L.fmt = kFmtNvfp4;
  return cuda_status(launch_whiten_decode_tc(&L, 1, dev_status, s));
}

// ---------------------------------------------------------------------------
gift_status gift_decode_sum(const uint8_t* const* codes, const float* const* scales, int n_parts, int64_t d_out,
                            int64_t d_in, const float* U, const float* lambda, const float* rho, int rank,
                            float alpha, void* G_hat, gift_dtype out_dt, uint32_t* dev_status, gift_stream_t stream) {
  if (!codes || !scales || n_parts < 1 || n_parts > kDecodeSumMaxParts) return GIFT_ERR_INVALID_ARG;
  for (int r = 0; r < n_parts; ++r) {
    gift_status st = check_codec_args(G_hat, out_dt, d_out, d_in, U, lambda, rho, rank, codes[r], scales[r]);
    if (st != GIFT_OK) return st;
  }
  if (dev_status && !aligned(dev_status, 4)) return GIFT_ERR_ALIGN;
  if (d_out == 0) return GIFT_OK;
  gift_status st = device_ok();
  if (st != GIFT_OK) return st;
  return cuda_status(launch_decode_sum(codes, scales, n_parts, d_out, d_in, U, lambda, rho, rank, alpha, G_hat, out_dt,
                                       dev_status, (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------
static gift_status check_dense_d(int64_t d) {
  if (d < GIFT_E4M3_BLOCK || d % GIFT_E4M3_BLOCK != 0 || d > 8192) return GIFT_ERR_SHAPE;
  return GIFT_OK;
}

gift_status gift_dense_factor_workspace_size(int64_t d, int kind, size_t* bytes) {
  if (!bytes || (kind != GIFT_DENSE_CHOLESKY && kind != GIFT_DENSE_INVSQRT)) return GIFT_ERR_INVALID_ARG;
  gift_status st = check_dense_d(d);
  if (st != GIFT_OK) return st;
  *bytes = dense_factor_ws_bytes(d, kind);
  return GIFT_OK;
}

gift_status gift_dense_factor(const float* A, int64_t d, int kind, float* M, float* M_inv, uint16_t* M_split,
                              uint16_t* M_inv_split, void* ws, size_t ws_bytes, uint32_t* dev_status,
                              gift_stream_t stream) {
  if (!A || !M || !M_inv || !M_split || !M_inv_split) return GIFT_ERR_INVALID_ARG;
  size_t need = 0;
  gift_status st = gift_dense_factor_workspace_size(d, kind, &need);
  if (st != GIFT_OK) return st;
  if (!ws || ws_bytes < need) return GIFT_ERR_WORKSPACE;
  if (!aligned16(A) || !aligned16(M) || !aligned16(M_inv) || !aligned16(M_split) || !aligned16(M_inv_split) ||
      !aligned16(ws) || (dev_status && !aligned(dev_status, 4)))
    return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  return cuda_status(launch_dense_factor(A, (int)d, kind, M, M_inv, M_split, M_inv_split, ws, dev_status,
                                         (cudaStream_t)stream));
}

gift_status gift_dense_split(const float* M, int64_t d, int parts, uint16_t* M_split, gift_stream_t stream) {
  if (!M || !M_split || (parts != 2 && parts != 3)) return GIFT_ERR_INVALID_ARG;
  gift_status st = check_dense_d(d);
  if (st != GIFT_OK) return st;
  if (!aligned16(M) || !aligned16(M_split)) return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  return cuda_status(launch_dense_split(M, (int)d, parts, M_split, (cudaStream_t)stream));
}

gift_status gift_dense_encode(const void* G, int64_t d_out, int64_t d_in, const uint16_t* M_split,
                              int upper_triangular, uint8_t* codes, float* scales, uint32_t* dev_status,
                              gift_stream_t stream) {
  if (d_out < 0) return GIFT_ERR_INVALID_ARG;
  gift_status st = check_dense_d(d_in);
  if (st != GIFT_OK) return st;
  if (d_out > ((int64_t)1 << 24)) return GIFT_ERR_SHAPE;
  if (d_out == 0) return GIFT_OK;
  if (!G || !M_split || !codes || !scales) return GIFT_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(M_split) || !aligned16(codes) || !aligned16(scales) ||
      (dev_status && !aligned(dev_status, 4)))
    return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  if (!tc_codec_available()) return GIFT_ERR_UNSUPPORTED;
  return cuda_status(launch_dense_encode(G, (int)d_out, (int)d_in, M_split, upper_triangular != 0, codes, scales,
                                         dev_status, (cudaStream_t)stream));
}

gift_status gift_dense_decode(const uint8_t* codes, const float* scales, int64_t d_out, int64_t d_in,
                              const uint16_t* M_inv_split, int upper_triangular, void* G_hat, gift_dtype out_dt,
                              uint32_t* dev_status, gift_stream_t stream) {
  if (d_out < 0 || !dtype_ok(out_dt)) return GIFT_ERR_INVALID_ARG;
  gift_status st = check_dense_d(d_in);
  if (st != GIFT_OK) return st;
  if (d_out > ((int64_t)1 << 24)) return GIFT_ERR_SHAPE;
  if (d_out == 0) return GIFT_OK;
  if (!codes || !scales || !M_inv_split || !G_hat) return GIFT_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(M_inv_split) || !aligned16(G_hat) ||
      (dev_status && !aligned(dev_status, 4)))
    return GIFT_ERR_ALIGN;
  if ((st = device_ok()) != GIFT_OK) return st;
  if (!tc_codec_available()) return GIFT_ERR_UNSUPPORTED;
  return cuda_status(launch_dense_decode(codes, scales, (int)d_out, (int)d_in, M_inv_split, upper_triangular != 0,
                                         G_hat, out_dt, dev_status, (cudaStream_t)stream));
}

}  // extern "C"
