// Chunked prefill on tcgen05 tensor cores (dk = dv = 128, bf16 operands, fp32 state).
#include "kda_internal.cuh"

namespace kda {

bool chunk64_available() { return false; }

cudaError_t launch_chunk64(const FwdParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kda
