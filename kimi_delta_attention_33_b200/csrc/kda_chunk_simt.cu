// kda_chunk_simt.cu -- chunked prefill on the FP32 CUDA cores.
//
// This is the path for the small shapes (K or V below 128, chunk 16) and the
// correctness baseline of the tensor-core kernel.  It follows the DeltaNet-family
// digest, section "Chunkwise KDA", in the key-major layout, one CTA per
// (b, hv, V-tile) (value columns are independent: the causal solve runs per value
// channel), chunks in order:
//   Gam_i   = sum_{m<=i} g_m                                in-chunk cumulative log decay
//   A_ij    = scale sum_d q_id k_jd e^{Gam_id - Gam_jd}      j <= i   (read matrix)
//   R_ij    = beta_i sum_d k_id k_jd e^{Gam_id - Gam_jd}    j <  i   (coupling)
//   Ebar_i  = beta_i (v_i - (k_i . e^{Gam_i}) S)            provisional errors
//   E_i     = Ebar_i - sum_{j<i} R_ij E_j                   causal solve, row by row
//   O_i     = scale (q_i . e^{Gam_i}) S + sum_{j<=i} A_ij E_j
//   S      <- diag(e^{Gam_last}) S + sum_j (k_j . e^{Gam_last - Gam_j})^T E_j
// Every decay factor is the exponential of a difference of prefix sums, each
// evaluated directly, so no factor can overflow whatever the gate values.
// A partial last chunk is zero-padded: zero q, k, g, beta and v rows leave the
// prefix sums flat and contribute nothing.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

constexpr int SIMT_THREADS = 256;

template <int K, int C, int VT>
struct SimtSmem {
    static constexpr int KP = K + 1;   // padded row stride of the [C][K] arrays
    static constexpr int CP = C + 1;   // padded row stride of A and R
    static constexpr int VP = VT + 1;  // padded row stride of E
    static constexpr size_t floats = 4 * (size_t)C * KP + 2 * (size_t)C * CP + (size_t)C * VT + (size_t)C * VP +
                                     (size_t)K * VT + C;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename Elt, int K, int C, int VT>
__global__ void __launch_bounds__(SIMT_THREADS)
chunk_simt_kernel(const Elt* __restrict__ q, const Elt* __restrict__ k, const Elt* __restrict__ v,
                  const Elt* __restrict__ g, const Elt* __restrict__ beta, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, const float* __restrict__ S0, int T, int H, int HV, int V,
                  int gate_mode, float lower_bound, float scale, unsigned int flags, Elt* __restrict__ o,
                  float* __restrict__ S_T) {
    using Sm = SimtSmem<K, C, VT>;
    constexpr int KP = Sm::KP, CP = Sm::CP, VP = Sm::VP;
    constexpr int NT = SIMT_THREADS;
    extern __shared__ float smem[];
    float* sQ = smem;                 // [C][KP] q
    float* sK = sQ + C * KP;          // [C][KP] k
    float* sG = sK + C * KP;          // [C][KP] g, then Gam
    float* sX = sG + C * KP;          // [C][KP] decay factors
    float* sA = sX + C * KP;          // [C][CP]
    float* sR = sA + C * CP;          // [C][CP]
    float* sV = sR + C * CP;          // [C][VT]
    float* sE = sV + C * VT;          // [C][VP]
    float* sS = sE + C * VP;          // [K][VT] state tile
    float* sB = sS + K * VT;          // [C] beta

    const int pair = blockIdx.x;
    const int b = pair / HV, hv = pair - b * HV;
    const int h = hv / (HV / H);
    const int v0 = blockIdx.y * VT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float rate = (gate_mode != KDA_GATE_NONE) ? expf(A_log[hv]) : 0.0f;

    for (int idx = tid; idx < K * VT; idx += NT) {
        const int d = idx / VT, c = idx - d * VT;
        sS[idx] = S0 ? S0[((size_t)pair * K + d) * V + v0 + c] : 0.0f;
    }

    for (int t0 = 0; t0 < T; t0 += C) {
        const int n = min(C, T - t0);
        __syncthreads();  // previous chunk finished with every array
        for (int idx = tid; idx < C * K; idx += NT) {
            const int i = idx / K, d = idx - i * K;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (i < n) {
                const size_t tok = (size_t)b * T + t0 + i;
                qv = to_f32(q[(tok * H + h) * K + d]);
                kv = to_f32(k[(tok * H + h) * K + d]);
                const float bias = (dt_bias != nullptr && gate_mode != KDA_GATE_NONE) ? dt_bias[hv * K + d] : 0.0f;
                gv = gate_value(to_f32(g[(tok * HV + hv) * K + d]), bias, rate, gate_mode, lower_bound);
            }
            sQ[i * KP + d] = qv;
            sK[i * KP + d] = kv;
            sG[i * KP + d] = gv;
        }
        for (int idx = tid; idx < C * VT; idx += NT) {
            const int i = idx / VT, c = idx - i * VT;
            sV[idx] = (i < n) ? to_f32(v[(((size_t)b * T + t0 + i) * HV + hv) * V + v0 + c]) : 0.0f;
        }
        for (int i = tid; i < C; i += NT) {
            const float bl = (i < n) ? to_f32(beta[((size_t)b * T + t0 + i) * HV + hv]) : 0.0f;
            sB[i] = (i < n && (flags & KDA_INPUT_BETA_LOGITS)) ? beta_from_logit(bl) : bl;
        }
        __syncthreads();
        if (flags & KDA_INPUT_L2NORM_QK) {  // q, k rows divided by their norms, one warp per row
            for (int i = warp; i < n; i += NT / 32) {
                float qq = 0.f, kk = 0.f;
                for (int d = lane; d < K; d += 32) {
                    qq += sQ[i * KP + d] * sQ[i * KP + d];
                    kk += sK[i * KP + d] * sK[i * KP + d];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    qq += __shfl_xor_sync(0xffffffffu, qq, off);
                    kk += __shfl_xor_sync(0xffffffffu, kk, off);
                }
                const float iq = inv_l2norm(qq), ik = inv_l2norm(kk);
                for (int d = lane; d < K; d += 32) {
                    sQ[i * KP + d] *= iq;
                    sK[i * KP + d] *= ik;
                }
            }
            __syncthreads();
        }

        // in-chunk inclusive prefix sums of the log decay, one key channel per thread
        for (int d = tid; d < K; d += NT) {
            float acc = 0.f;
            for (int i = 0; i < C; ++i) {
                acc += sG[i * KP + d];
                sG[i * KP + d] = acc;
            }
        }
        __syncthreads();

        // read matrix A and coupling R, decay factors taken exactly per (i, j, d)
        for (int p = tid; p < C * C; p += NT) {
            const int i = p / C, j = p - i * C;
            float a = 0.f, r = 0.f;
            if (j <= i) {
                for (int d = 0; d < K; ++d) {
                    const float e = __expf(sG[i * KP + d] - sG[j * KP + d]);
                    const float kj = sK[j * KP + d] * e;
                    a += sQ[i * KP + d] * kj;
                    r += sK[i * KP + d] * kj;
                }
            }
            sA[i * CP + j] = (j <= i) ? scale * a : 0.f;
            sR[i * CP + j] = (j < i) ? sB[i] * r : 0.f;
        }
        for (int idx = tid; idx < C * K; idx += NT) {
            const int i = idx / K, d = idx - i * K;
            sX[i * KP + d] = __expf(sG[i * KP + d]);  // decay from the chunk boundary to token i
        }
        __syncthreads();

        // provisional errors against the chunk-entry state
        for (int idx = tid; idx < C * VT; idx += NT) {
            const int i = idx / VT, c = idx - i * VT;
            float acc = 0.f;
            for (int d = 0; d < K; ++d) acc += sK[i * KP + d] * sX[i * KP + d] * sS[d * VT + c];
            sE[i * VP + c] = sB[i] * (sV[idx] - acc);
        }
        __syncthreads();

        // causal solve per value channel: each warp owns VT/8 columns, rows in order
        constexpr int CPW = VT / (NT / 32);
        for (int i = 1; i < n; ++i) {
#pragma unroll
            for (int cc = 0; cc < CPW; ++cc) {
                const int c = warp * CPW + cc;
                float part = 0.f;
                for (int j = lane; j < i; j += 32) part += sR[i * CP + j] * sE[j * VP + c];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (lane == 0) sE[i * VP + c] -= part;
            }
            __syncwarp();
        }
        __syncthreads();

        // chunk outputs: read the decayed entry state, then the in-chunk writes
        for (int idx = tid; idx < C * VT; idx += NT) {
            const int i = idx / VT, c = idx - i * VT;
            if (i >= n) continue;
            float acc = 0.f;
            for (int d = 0; d < K; ++d) acc += sQ[i * KP + d] * sX[i * KP + d] * sS[d * VT + c];
            acc *= scale;
            for (int j = 0; j <= i; ++j) acc += sA[i * CP + j] * sE[j * VP + c];
            o[(((size_t)b * T + t0 + i) * HV + hv) * V + v0 + c] = from_f32<Elt>(acc);
        }
        __syncthreads();

        // keys decayed to the chunk end
        for (int idx = tid; idx < C * K; idx += NT) {
            const int j = idx / K, d = idx - j * K;
            sX[j * KP + d] = sK[j * KP + d] * __expf(sG[(C - 1) * KP + d] - sG[j * KP + d]);
        }
        __syncthreads();

        // chunk-end state
        for (int idx = tid; idx < K * VT; idx += NT) {
            const int d = idx / VT, c = idx - d * VT;
            float acc = __expf(sG[(C - 1) * KP + d]) * sS[idx];
            for (int j = 0; j < C; ++j) acc += sX[j * KP + d] * sE[j * VP + c];
            sS[idx] = acc;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < K * VT; idx += NT) {
            const int d = idx / VT, c = idx - d * VT;
            S_T[((size_t)pair * K + d) * V + v0 + c] = sS[idx];
        }
    }
}

template <typename Elt, int K, int C, int VT>
static cudaError_t launch_simt(const ChunkArgs& a) {
    using Sm = SimtSmem<K, C, VT>;
    auto kern = chunk_simt_kernel<Elt, K, C, VT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sm::bytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.HV, a.V / VT);
    kern<<<grid, SIMT_THREADS, Sm::bytes, a.stream>>>(
        static_cast<const Elt*>(a.q), static_cast<const Elt*>(a.k), static_cast<const Elt*>(a.v),
        static_cast<const Elt*>(a.g), static_cast<const Elt*>(a.beta), a.A_log, a.dt_bias, a.S0, a.T, a.H, a.HV, a.V,
        a.gate_mode, a.lower_bound, a.scale, a.flags, static_cast<Elt*>(a.o), a.S_T);
    return cudaGetLastError();
}

template <typename Elt, int K, int C>
static cudaError_t simt_vt(const ChunkArgs& a) {
    if (a.V == 16) return launch_simt<Elt, K, C, 16>(a);
    return launch_simt<Elt, K, C, 32>(a);
}

template <typename Elt, int K>
static cudaError_t simt_c(const ChunkArgs& a) {
    return a.chunk == 16 ? simt_vt<Elt, K, 16>(a) : simt_vt<Elt, K, 64>(a);
}

template <typename Elt>
static cudaError_t simt_k(const ChunkArgs& a) {
    switch (a.K) {
        case 16: return simt_c<Elt, 16>(a);
        case 32: return simt_c<Elt, 32>(a);
        case 64: return simt_c<Elt, 64>(a);
        case 128: return simt_c<Elt, 128>(a);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_simt(const ChunkArgs& a) {
    return a.dtype == KDA_BF16 ? simt_k<__nv_bfloat16>(a) : simt_k<float>(a);
}

}  // namespace kda
