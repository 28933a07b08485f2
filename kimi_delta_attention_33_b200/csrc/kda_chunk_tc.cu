// kda_chunk_tc.cu -- chunked prefill on the 5th-generation tensor cores (tcgen05 / TMEM).
// Placeholder until the tensor-core pipeline lands: every shape goes to the CUDA-core kernel.
#include "kda_internal.h"

namespace kda {

bool chunk_tc_supported(const ChunkArgs&) { return false; }

cudaError_t launch_chunk_tc(const ChunkArgs&) { return cudaErrorNotSupported; }

}  // namespace kda
