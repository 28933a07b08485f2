// kda_noalloc.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers only ever hold pointers to buffers that someone else owns: a host application
// or plugin that receives its tensors from an outer runtime with a fixed device-memory budget
// and no allocator to hand out, or a latency-critical serving loop where allocating on the call
// path is forbidden.  Such a caller cannot provide the workspace kda_chunk_fwd asks for.  This
// entry point supplies that workspace itself, from a fixed array in device memory that is part
// of this library (every GPU that loads the library holds it until the process exits), and then
// runs kda_chunk_fwd with it.  The array is far smaller than the per-chunk records of the two-pass
// schedule, so these calls always take the single-pass schedule: same results, one kernel.
#include <cuda_runtime.h>

#include <cstdio>

#include "kda_internal.h"

namespace {

// Upper bound on the workspace kda_chunk_fwd may need; larger requests are rejected.
constexpr size_t kScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
// Every size kda_chunk_fwd accepts needs only its status block in the schedule chosen here.
static_assert(kda::kChunkStatusBytes <= kScratchBytes, "the status block must fit in the built-in array");

// The workspace of every kda_chunk_fwd_noalloc call.  In host code this name is only a
// stand-in for the symbol, not a device address: its address on the current device comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// The array's address in the current device's context, resolved on every call (it allocates
// nothing), so that a context torn down and recreated in between -- cudaDeviceReset, or another
// driver context made current -- never leaves a stale pointer behind.
kda_status scratch_address(void** p, const char* who) {
    *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(p, g_noalloc_scratch);
    if (e != cudaSuccess || *p == nullptr) {
        char msg[192];
        snprintf(msg, sizeof(msg), "%s: cudaGetSymbolAddress of the built-in workspace failed (%s)", who,
                 cudaGetErrorString(e));
        kda::set_last_error(msg);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                                            const void* beta, const float* A_log, const float* dt_bias,
                                            const float* S0, int B, int T, int H, int HV, int K, int V, int chunk,
                                            kda_gate_mode gate_mode, float lower_bound, float scale,
                                            kda_dtype dtype, void* o, float* S_T, kda_stream_t stream) {
    // The smallest workspace kda_chunk_fwd accepts: with it, kda_chunk_fwd runs its single-pass
    // schedule, which needs no scratch beyond the status word.  Sizes kda_chunk_fwd rejects outright
    // (need == 0) are reported by its own validation below.
    const size_t need = kda::chunk_min_workspace(B, T, H, HV, K, V, chunk);
    if (need > kScratchBytes) {
        char msg[192];
        snprintf(msg, sizeof(msg), "kda_chunk_fwd_noalloc: these sizes need %zu bytes of workspace, more than the "
                 "built-in %zu bytes", need, kScratchBytes);
        kda::set_last_error(msg);
        return KDA_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    const kda_status s = scratch_address(&scratch, "kda_chunk_fwd_noalloc");
    if (s != KDA_OK) return s;
    // kda_chunk_fwd clears the status word at the start of the array before launching; nothing else
    // in the array needs to start at zero.
    return kda_chunk_fwd(q, k, v, g, beta, A_log, dt_bias, S0, B, T, H, HV, K, V, chunk, gate_mode, lower_bound,
                         scale, dtype, o, S_T, scratch, kScratchBytes, stream);
}

extern "C" kda_status kda_chunk_fwd_noalloc_read_status(kda_stream_t stream) {
    void* scratch = nullptr;
    const kda_status s = scratch_address(&scratch, "kda_chunk_fwd_noalloc_read_status");
    if (s != KDA_OK) return s;
    return kda_read_status(scratch, stream);
}
