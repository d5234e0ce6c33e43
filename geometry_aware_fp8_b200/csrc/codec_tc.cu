// Whitened E4M3 codec on the tcgen05 tensor cores (bf16 gradients).
// Not yet enabled: the C-ABI routes every layer to the CUDA-core kernels
// while tc_codec_available() returns false.
#include "common.cuh"
#include "internal.h"

namespace gift {

bool tc_codec_available() { return false; }

cudaError_t launch_whiten_encode_tc(const TcLayer*, int, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_whiten_decode_tc(const TcLayer*, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gift
