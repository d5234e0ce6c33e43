// Factor refresh for callers that cannot allocate device memory.
//
// gift_factor_refresh needs a workspace from the caller.  Some callers have
// no way to provide one: code whose device memory is owned entirely by
// someone else's pool, or a step that must not call cudaMalloc because the
// allocation can synchronise the device.  gift_factor_refresh_noalloc runs
// the same refresh with its scratch in one array that lives in this file and
// is part of the library's device image: it exists on every GPU that loads
// the library, from load until the process exits, and no call allocates
// anything.
//
// Limits: d_in <= 4096 and rank + oversample <= 64, which bounds the scratch
// (sampled subspace, its image, a Cholesky-QR temporary, fp64 Gram partials
// and the small factors) at 5,308,416 bytes.  A must be given by the caller as an output buffer,
// and the token range is not split, so the whole scratch need is known.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace gift {
namespace {

constexpr int64_t kNoAllocMaxDin = 4096;
constexpr int kNoAllocMaxSubspace = 64;
constexpr size_t kNoAllocScratchBytes = 5308416;

// Scratch shared by every call on a device.  Host code cannot use this name
// as a device address: it only names the host-side shadow of the symbol, so
// the device address is looked up with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_refresh_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

// Unique id of the calling thread's current context (0 if it cannot be read).
// A device reset destroys the primary context and the module image with it;
// the next context gets a new id, so a cached address is never reused across
// a reset.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = (PFN_cuCtxGetCurrent_v4000)p;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (PFN_cuCtxGetId_v12000)p;
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device.  It is looked
// up with the device current on the first call, and again whenever the
// device's context has changed since (after a cudaDeviceReset, say).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();  // 0 before the runtime has made a context
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_refresh_scratch);  // makes the context if there is none yet
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace gift

using namespace gift;

extern "C" gift_status gift_factor_refresh_noalloc(const void* X, gift_dtype xdt, int64_t N, int64_t d_in, int rank,
                                                   int oversample, int iters, uint64_t seed, float* U,
                                                   float* lambda, float* rho, float* A_out, uint32_t* dev_status,
                                                   gift_stream_t stream) {
  if (!X || !U || !lambda || !rho || !A_out) return GIFT_ERR_INVALID_ARG;
  if (xdt != GIFT_F32 && xdt != GIFT_BF16) return GIFT_ERR_INVALID_ARG;
  if (iters < 0 || iters > 1000) return GIFT_ERR_INVALID_ARG;
  if (N < 1 || d_in <= 0 || rank < 1 || oversample < 0) return GIFT_ERR_INVALID_ARG;
  if (d_in % GIFT_E4M3_BLOCK != 0 || d_in > kNoAllocMaxDin) return GIFT_ERR_SHAPE;
  if (rank + oversample > kNoAllocMaxSubspace || rank + oversample > d_in) return GIFT_ERR_SHAPE;
  const auto al = [](const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; };
  if (!al(X, 16) || !al(U, 16) || !al(A_out, 16) || !al(lambda, 4) || !al(rho, 4) ||
      (dev_status && !al(dev_status, 4)))
    return GIFT_ERR_ALIGN;
  RefreshPlan p;
  // one token range and one k-slice: A_out is written directly, nothing is split
  refresh_plan(N, d_in, rank, oversample, /*a_out_given=*/true, &p, /*no_split=*/true);
  if (p.total > kNoAllocScratchBytes) return GIFT_ERR_SHAPE;
  p.iters = iters;
  p.seed = seed;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GIFT_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GIFT_ERR_CUDA;
  if (major != 10) return GIFT_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return GIFT_ERR_CUDA;
  return launch_refresh(p, X, xdt, U, lambda, rho, A_out, ws, dev_status, (cudaStream_t)stream) == cudaSuccess
             ? GIFT_OK
             : GIFT_ERR_CUDA;
}
