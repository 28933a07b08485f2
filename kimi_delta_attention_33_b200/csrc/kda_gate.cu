// kda_gate.cu -- the gate activation as a stand-alone elementwise kernel.
// KDA notes, "Gate 激活", code box kda_gate_reference: input = g_raw + dt_bias[hv, :],
// rate = exp(A_log[hv]); SAFE -> L * sigmoid(rate * input), STANDARD -> -rate * softplus(input).
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

template <typename T>
__global__ void gate_kernel(const T* __restrict__ g_raw, const float* __restrict__ A_log,
                            const float* __restrict__ dt_bias, long long n, int HV, int K, int mode,
                            float lower_bound, float* __restrict__ g_out) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int d = (int)(i % K);
        const int hv = (int)((i / K) % HV);
        const float bias = dt_bias ? dt_bias[hv * K + d] : 0.0f;
        g_out[i] = gate_value(to_f32(g_raw[i]), bias, expf(A_log[hv]), mode, lower_bound);
    }
}

cudaError_t launch_gate(const GateArgs& a) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (a.n + 255) / 256;
    const long long cap = (long long)sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (a.dtype == KDA_BF16)
        gate_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, a.stream>>>(
            static_cast<const __nv_bfloat16*>(a.g_raw), a.A_log, a.dt_bias, a.n, a.HV, a.K, a.gate_mode,
            a.lower_bound, a.g_out);
    else
        gate_kernel<float><<<(unsigned)blocks, 256, 0, a.stream>>>(static_cast<const float*>(a.g_raw), a.A_log,
                                                                    a.dt_bias, a.n, a.HV, a.K, a.gate_mode,
                                                                    a.lower_bound, a.g_out);
    return cudaGetLastError();
}

}  // namespace kda
