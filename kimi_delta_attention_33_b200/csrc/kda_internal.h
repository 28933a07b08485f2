// kda_internal.h -- argument bundles and launcher declarations between the C ABI and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/kda.h"

namespace kda {

struct DecodeArgs {
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    int B, H, HV, K, V;
    int gate_mode;
    float lower_bound, scale;
    int dtype;
    unsigned int flags;  // kda_input_flags
    float* S;
    void* o;
    cudaStream_t stream;
};

struct ChunkArgs {
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias, *S0;
    int B, T, H, HV, K, V, chunk;
    int gate_mode;
    float lower_bound, scale;
    int dtype;
    unsigned int flags;  // kda_input_flags
    void* o;
    float* S_T;
    unsigned int* status;  // device status word (first bytes of the workspace)
    void* scratch;         // workspace beyond the status block
    size_t scratch_bytes;
    cudaStream_t stream;
};

struct GateArgs {
    const void* g_raw;
    int dtype;
    const float *A_log, *dt_bias;
    long long n;  // B*T*HV*K
    int HV, K;
    int gate_mode;
    float lower_bound;
    float* g_out;
    cudaStream_t stream;
};

struct BackwardArgs {
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias, *S0;
    const void* dO;
    const float* dS_T;
    int B, T, H, HV, K, V;
    int gate_mode;
    float lower_bound, scale;
    int dtype;
    float *dq, *dk, *dv, *dg, *dbeta, *dS0, *dA_log, *ddt_bias;
    void* workspace;
    cudaStream_t stream;
};

struct MlaArgs {
    const void *q, *W_UK, *W_UV, *c;
    const int* lengths;
    int B, T, H, d_q, d_v, R;
    float scale;
    void* o;
    void* workspace;
    cudaStream_t stream;
};

// Status word values written by kernels with bounded waits.
enum : unsigned int { STATUS_OK = 0u, STATUS_TIMEOUT = 1u };

// Sets the thread-local message kda_last_error() returns.
void set_last_error(const char* msg);

cudaError_t launch_decode_step(const DecodeArgs& a);
cudaError_t launch_gate(const GateArgs& a);
cudaError_t launch_chunk_simt(const ChunkArgs& a);
cudaError_t launch_chunk_tc(const ChunkArgs& a);
// Two-pass tensor-core prefill (same shapes as the single-pass one): per-chunk records (and, for
// long sequences, the segment carries of the split state pass) need chunk_split_workspace(B, T, HV)
// bytes of scratch beyond the status block.
struct ScanPlan {
    int L;   // chunks per segment of the state pass
    int NS;  // segments (1: the state pass runs each sequence as one chain)
};
ScanPlan chunk_scan_plan(long long pairs, int NC);
size_t chunk_split_workspace(int B, int T, int HV);
cudaError_t launch_chunk_split(const ChunkArgs& a);

// Reverse mode: saved states every few tokens, backward_workspace(B, T, HV, K, V) bytes.
size_t backward_workspace(int B, int T, int HV, int K, int V);
cudaError_t launch_backward(const BackwardArgs& a);

// Absorbed MLA decode: q_abs, the per-split partial results; mla_workspace(B, T, H, R) bytes.
int mla_nsplit(int B, int T, int H);
size_t mla_workspace(int B, int T, int H, int R);
cudaError_t launch_mla_decode(const MlaArgs& a);

// Bytes of status block at the start of every chunk-prefill workspace.
constexpr size_t kChunkStatusBytes = 256;
// Smallest workspace kda_chunk_fwd accepts for these sizes (0 if it rejects the sizes).
size_t chunk_min_workspace(int B, int T, int H, int HV, int K, int V, int chunk);

}  // namespace kda
