// kda_api.cu -- the C ABI declared in include/kda.h: host-side validation, kernel choice,
// status codes and the thread-local error string.  No exception crosses this file's
// extern "C" functions and nothing here allocates device memory.
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "kda_internal.h"

#define KDA_VERSION_STRING "kda-b200 0.1.0 (sm_100a)"

namespace {

thread_local char g_err[512] = "";

kda_status fail(kda_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

kda_status ok() {
    g_err[0] = '\0';
    return KDA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool kv_dim_ok(int x) { return x == 16 || x == 32 || x == 64 || x == 128; }

kda_status cuda_fail(cudaError_t e, const char* what) {
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Validation shared by the prefill and decode entry points.
kda_status check_common(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        const float* A_log, int B, int H, int HV, int K, int V, int gate_mode, float lower_bound,
                        int dtype, const void* o) {
    if (!q || !k || !v || !g || !beta || !o) return fail(KDA_ERR_INVALID_ARG, "null tensor pointer (q, k, v, g, beta and o are required)");
    if (B < 1 || H < 1 || HV < 1 || K < 1 || V < 1) return fail(KDA_ERR_INVALID_ARG, "sizes must be >= 1 (B=%d H=%d HV=%d K=%d V=%d)", B, H, HV, K, V);
    if (HV % H != 0) return fail(KDA_ERR_INVALID_ARG, "HV (%d) must be a multiple of H (%d)", HV, H);
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (gate_mode != KDA_GATE_NONE && gate_mode != KDA_GATE_SAFE && gate_mode != KDA_GATE_STANDARD)
        return fail(KDA_ERR_INVALID_ARG, "unknown gate mode %d", gate_mode);
    if (gate_mode != KDA_GATE_NONE && !A_log) return fail(KDA_ERR_INVALID_ARG, "A_log is required when the gate is applied in the op");
    if (gate_mode == KDA_GATE_SAFE && !(std::isfinite(lower_bound) && lower_bound < 0.0f))
        return fail(KDA_ERR_INVALID_ARG, "safe gate needs a finite lower_bound < 0 (got %g)", (double)lower_bound);
    if (!kv_dim_ok(K) || !kv_dim_ok(V)) return fail(KDA_ERR_UNSUPPORTED, "K and V must each be 16, 32, 64 or 128 (K=%d V=%d)", K, V);
    return KDA_OK;
}

constexpr size_t kStatusBytes = kda::kChunkStatusBytes;
constexpr unsigned int kInputFlagsAll = KDA_INPUT_L2NORM_QK | KDA_INPUT_BETA_LOGITS;

bool sizes_ok(int B, int T, int H, int HV, int K, int V, int chunk) {
    return B >= 1 && T >= 1 && H >= 1 && HV >= 1 && HV % H == 0 && kv_dim_ok(K) && kv_dim_ok(V) &&
           (chunk == 16 || chunk == 64);
}

// Up to this many (sequence, value head) pairs the two-pass schedule is the faster one on a
// 148-SM B200: with more, one CTA per pair already keeps most SMs busy in the single pass, while
// the two-pass schedule adds the round trip of the per-chunk records through memory.
constexpr long long kTwoPassMaxPairs = 96;

// The tensor-core schedules cover K = V = 128, chunk 64 with bf16 inputs.  With float32 inputs the
// stated tolerance (1e-4) is tighter than tf32 products allow, so those (and the other shapes) run
// on the CUDA-core kernel in fp32.
bool split_shape(int K, int V, int chunk) { return K == 128 && V == 128 && chunk == 64; }

// Sizes the two-pass schedule takes: at most kTwoPassMaxPairs pairs; fewer than 2^30 chunks in all (the
// prep kernel counts its tasks in an int); the tensor maps of its input copies need a token stride
// (heads x 256 bytes) times T below 2^40 bytes.
bool two_pass_sizes(int B, int T, int HV) {
    const long long pairs = (long long)B * HV;
    return pairs <= kTwoPassMaxPairs && pairs * (((long long)T + 63) / 64) < (1ll << 30) &&
           (long long)T * HV * 256 < (1ll << 40);
}

}  // namespace

namespace kda {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

size_t chunk_min_workspace(int B, int T, int H, int HV, int K, int V, int chunk) {
    return sizes_ok(B, T, H, HV, K, V, chunk) ? kStatusBytes : 0;
}
}  // namespace kda

extern "C" {

const char* kda_last_error(void) { return g_err; }

const char* kda_version(void) { return KDA_VERSION_STRING; }

kda_status kda_gate(const void* g_raw, kda_dtype dtype, const float* A_log, const float* dt_bias, int B, int T,
                    int HV, int K, kda_gate_mode mode, float lower_bound, float* g_out, kda_stream_t stream) {
    if (!g_raw || !A_log || !g_out) return fail(KDA_ERR_INVALID_ARG, "null pointer (g_raw, A_log and g_out are required)");
    if (B < 1 || T < 1 || HV < 1 || K < 1) return fail(KDA_ERR_INVALID_ARG, "sizes must be >= 1");
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (mode != KDA_GATE_SAFE && mode != KDA_GATE_STANDARD) return fail(KDA_ERR_INVALID_ARG, "kda_gate needs SAFE or STANDARD mode");
    if (mode == KDA_GATE_SAFE && !(std::isfinite(lower_bound) && lower_bound < 0.0f))
        return fail(KDA_ERR_INVALID_ARG, "safe gate needs a finite lower_bound < 0 (got %g)", (double)lower_bound);
    const long long n = (long long)B * T * HV * K;
    if (n >= (1ll << 31)) return fail(KDA_ERR_UNSUPPORTED, "B*T*HV*K must be < 2^31");
    kda::GateArgs a{g_raw, (int)dtype, A_log, dt_bias, n, HV, K, (int)mode, lower_bound, g_out, (cudaStream_t)stream};
    cudaError_t e = kda::launch_gate(a);
    if (e != cudaSuccess) return cuda_fail(e, "gate kernel launch");
    return ok();
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int HV, int K, int V, int chunk) {
    if (!sizes_ok(B, T, H, HV, K, V, chunk)) return 0;
    if (split_shape(K, V, chunk) && two_pass_sizes(B, T, HV)) return kStatusBytes + kda::chunk_split_workspace(B, T, HV);
    return kStatusBytes;
}

int kda_chunk_fwd_schedule(int B, int T, int H, int HV, int K, int V, int chunk, kda_dtype dtype,
                           size_t workspace_bytes) {
    if (!sizes_ok(B, T, H, HV, K, V, chunk) || (dtype != KDA_F32 && dtype != KDA_BF16) || workspace_bytes < kStatusBytes)
        return -1;
    if (dtype != KDA_BF16 || !split_shape(K, V, chunk)) return KDA_SCHEDULE_CUDA_CORE;
    if (two_pass_sizes(B, T, HV) && workspace_bytes - kStatusBytes >= kda::chunk_split_workspace(B, T, HV))
        return kda::chunk_scan_plan((long long)B * HV, (T + 63) / 64).NS > 1 ? KDA_SCHEDULE_TC_TWO_PASS_SCAN
                                                                              : KDA_SCHEDULE_TC_TWO_PASS;
    return KDA_SCHEDULE_TC_SINGLE_PASS;
}

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            const float* A_log, const float* dt_bias, const float* S0, int B, int T, int H, int HV,
                            int K, int V, int chunk, kda_gate_mode gate_mode, float lower_bound, float scale,
                            kda_dtype dtype, unsigned int input_flags, void* o, float* S_T, void* workspace,
                            size_t workspace_bytes, kda_stream_t stream) {
    kda_status s = check_common(q, k, v, g, beta, A_log, B, H, HV, K, V, (int)gate_mode, lower_bound, (int)dtype, o);
    if (s != KDA_OK) return s;
    if (input_flags & ~kInputFlagsAll) return fail(KDA_ERR_INVALID_ARG, "unknown input flag bits 0x%x", input_flags);
    if (T < 1) return fail(KDA_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    if (chunk != 16 && chunk != 64) return fail(KDA_ERR_UNSUPPORTED, "chunk must be 16 or 64 (got %d)", chunk);
    if ((long long)B * T * HV * (K > V ? K : V) >= (1ll << 40)) return fail(KDA_ERR_UNSUPPORTED, "tensor too large");
    const void* ptrs[] = {q, k, v, g, beta, A_log, dt_bias, S0, o, S_T, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    if (!workspace || workspace_bytes < kStatusBytes)
        return fail(KDA_ERR_INVALID_ARG, "workspace of at least %zu bytes is required (got %zu)", kStatusBytes,
                    workspace_bytes);
    if (o == q || o == k || o == v || o == g || o == beta) return fail(KDA_ERR_INVALID_ARG, "o must not alias an input");
    if (!(scale > 0.0f)) scale = 1.0f / std::sqrt((float)K);
    kda::ChunkArgs a{q, k, v, g, beta, A_log, dt_bias, S0, B, T, H, HV, K, V, chunk, (int)gate_mode, lower_bound,
                     scale, (int)dtype, input_flags, o, S_T, static_cast<unsigned int*>(workspace),
                     static_cast<char*>(workspace) + kStatusBytes, workspace_bytes - kStatusBytes,
                     (cudaStream_t)stream};
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "status word reset");
    const int schedule = kda_chunk_fwd_schedule(B, T, H, HV, K, V, chunk, dtype, workspace_bytes);
    if (schedule == KDA_SCHEDULE_TC_TWO_PASS || schedule == KDA_SCHEDULE_TC_TWO_PASS_SCAN) {
        e = kda::launch_chunk_split(a);
        if (e != cudaSuccess) return cuda_fail(e, "two-pass tensor-core chunk kernel launch");
    } else if (schedule == KDA_SCHEDULE_TC_SINGLE_PASS) {
        e = kda::launch_chunk_tc(a);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core chunk kernel launch");
    } else {
        e = kda::launch_chunk_simt(a);
        if (e != cudaSuccess) return cuda_fail(e, "chunk kernel launch");
    }
    return ok();
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         const float* A_log, const float* dt_bias, const float* S0, int B, int T, int H, int HV,
                         int K, int V, int chunk, kda_gate_mode gate_mode, float lower_bound, float scale,
                         kda_dtype dtype, void* o, float* S_T, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream) {
    return kda_chunk_fwd_ex(q, k, v, g, beta, A_log, dt_bias, S0, B, T, H, HV, K, V, chunk, gate_mode, lower_bound,
                            scale, dtype, 0u, o, S_T, workspace, workspace_bytes, stream);
}

kda_status kda_read_status(const void* workspace, kda_stream_t stream) {
    if (!workspace) return fail(KDA_ERR_INVALID_ARG, "null workspace");
    unsigned int word = 0;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read-back");
    if (word != kda::STATUS_OK) {
        const unsigned int zero = 0;
        cudaMemcpy(const_cast<void*>(workspace), &zero, sizeof(zero), cudaMemcpyHostToDevice);
        return fail(KDA_ERR_TIMEOUT, "an on-device wait gave up (status word 0x%x); outputs are undefined", word);
    }
    return ok();
}

kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                 const float* A_log, const float* dt_bias, int B, int H, int HV, int K, int V,
                                 kda_gate_mode gate_mode, float lower_bound, float scale, kda_dtype dtype,
                                 unsigned int input_flags, float* S, void* o, kda_stream_t stream) {
    kda_status s = check_common(q, k, v, g, beta, A_log, B, H, HV, K, V, (int)gate_mode, lower_bound, (int)dtype, o);
    if (s != KDA_OK) return s;
    if (input_flags & ~kInputFlagsAll) return fail(KDA_ERR_INVALID_ARG, "unknown input flag bits 0x%x", input_flags);
    if (!S) return fail(KDA_ERR_INVALID_ARG, "null state pointer S");
    if ((long long)B * HV >= (1ll << 31)) return fail(KDA_ERR_UNSUPPORTED, "B*HV must be < 2^31");
    const void* ptrs[] = {q, k, v, g, beta, A_log, dt_bias, S, o};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    if (o == q || o == k || o == v || o == g || o == beta || o == S) return fail(KDA_ERR_INVALID_ARG, "o must not alias an input");
    if (!(scale > 0.0f)) scale = 1.0f / std::sqrt((float)K);
    kda::DecodeArgs a{q, k, v, g, beta, A_log, dt_bias, B, H, HV, K, V, (int)gate_mode, lower_bound, scale,
                      (int)dtype, input_flags, S, o, (cudaStream_t)stream};
    cudaError_t e = kda::launch_decode_step(a);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
    return ok();
}

kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const void* g, const void* beta,
                              const float* A_log, const float* dt_bias, int B, int H, int HV, int K, int V,
                              kda_gate_mode gate_mode, float lower_bound, float scale, kda_dtype dtype, float* S,
                              void* o, kda_stream_t stream) {
    return kda_recurrent_step_ex(q, k, v, g, beta, A_log, dt_bias, B, H, HV, K, V, gate_mode, lower_bound, scale,
                                 dtype, 0u, S, o, stream);
}

size_t kda_backward_workspace_size(int B, int T, int H, int HV, int K, int V) {
    if (!sizes_ok(B, T, H, HV, K, V, 64)) return 0;
    return kda::backward_workspace(B, T, HV, K, V);
}

kda_status kda_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        const float* A_log, const float* dt_bias, const float* S0, const void* dO, const float* dS_T,
                        int B, int T, int H, int HV, int K, int V, kda_gate_mode gate_mode, float lower_bound,
                        float scale, kda_dtype dtype, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                        float* dS0, float* dA_log, float* ddt_bias, void* workspace, size_t workspace_bytes,
                        kda_stream_t stream) {
    kda_status s = check_common(q, k, v, g, beta, A_log, B, H, HV, K, V, (int)gate_mode, lower_bound, (int)dtype, dO);
    if (s != KDA_OK) return s;
    if (T < 1) return fail(KDA_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    if (!dq || !dk || !dv || !dg || !dbeta) return fail(KDA_ERR_INVALID_ARG, "dq, dk, dv, dg and dbeta are required");
    if ((long long)B * T * HV * (K > V ? K : V) >= (1ll << 40)) return fail(KDA_ERR_UNSUPPORTED, "tensor too large");
    const void* ptrs[] = {q, k, v, g, beta, A_log, dt_bias, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    const size_t need = kda::backward_workspace(B, T, HV, K, V);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "workspace of at least %zu bytes is required (got %zu)", need, workspace_bytes);
    const void* outs[] = {dq, dk, dv, dg, dbeta, dS0, dA_log, ddt_bias};
    const void* ins[] = {q, k, v, g, beta, A_log, dt_bias, S0, dO, dS_T};
    for (const void* po : outs)
        for (const void* pi : ins)
            if (po && po == pi) return fail(KDA_ERR_INVALID_ARG, "outputs must not alias inputs");
    if (!(scale > 0.0f)) scale = 1.0f / std::sqrt((float)K);
    kda::BackwardArgs a{q, k, v, g, beta, A_log, dt_bias, S0, dO, dS_T, B, T, H, HV, K, V, (int)gate_mode,
                        lower_bound, scale, (int)dtype, dq, dk, dv, dg, dbeta, dS0, dA_log, ddt_bias, workspace,
                        (cudaStream_t)stream};
    cudaError_t e = kda::launch_backward(a);
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return ok();
}

static bool mla_sizes_ok(int B, int T, int H, int d_q, int d_v, int r) {
    return B >= 1 && T >= 1 && H >= 1 && (d_q == 64 || d_q == 128) && (d_v == 64 || d_v == 128) &&
           (r == 128 || r == 256 || r == 512) && (long long)B * T * r < (1ll << 40) && (long long)B * H < (1ll << 24);
}

size_t kda_mla_decode_workspace_size(int B, int T, int H, int d_q, int d_v, int r) {
    return mla_sizes_ok(B, T, H, d_q, d_v, r) ? kda::mla_workspace(B, T, H, r) : 0;
}

kda_status kda_mla_decode(const void* q, const void* W_UK, const void* W_UV, const void* c, const int* lengths, int B,
                          int T, int H, int d_q, int d_v, int r, float scale, kda_dtype dtype, void* o,
                          void* workspace, size_t workspace_bytes, kda_stream_t stream) {
    if (!q || !W_UK || !W_UV || !c || !o) return fail(KDA_ERR_INVALID_ARG, "null tensor pointer (q, W_UK, W_UV, c, o)");
    if (B < 1 || T < 1 || H < 1) return fail(KDA_ERR_INVALID_ARG, "sizes must be >= 1 (B=%d T=%d H=%d)", B, T, H);
    if (dtype != KDA_BF16) return fail(KDA_ERR_UNSUPPORTED, "kda_mla_decode is built for bf16 only");
    if (!mla_sizes_ok(B, T, H, d_q, d_v, r))
        return fail(KDA_ERR_UNSUPPORTED, "unsupported sizes (d_q, d_v in {64, 128}; r in {128, 256, 512})");
    const void* ptrs[] = {q, W_UK, W_UV, c, lengths, o, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
    const size_t need = kda::mla_workspace(B, T, H, r);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "workspace of at least %zu bytes is required (got %zu)", need, workspace_bytes);
    if (o == q || o == c || o == W_UK || o == W_UV) return fail(KDA_ERR_INVALID_ARG, "o must not alias an input");
    if (!(scale > 0.0f)) scale = 1.0f / std::sqrt((float)d_q);
    kda::MlaArgs a{q, W_UK, W_UV, c, lengths, B, T, H, d_q, d_v, r, scale, o, workspace, (cudaStream_t)stream};
    const cudaError_t e = kda::launch_mla_decode(a);
    if (e != cudaSuccess) return cuda_fail(e, "MLA decode kernel launch");
    return ok();
}

}  // extern "C"
