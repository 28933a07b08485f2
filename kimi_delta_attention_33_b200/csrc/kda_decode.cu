// kda_decode.cu -- fused recurrent decode step (one token per sequence), HBM-streaming.
//
// DeltaNet-family digest, "decode के लिए fused recurrent Triton kernel": the recurrent
// schedule runs decay, the key-side prediction reduction, the residual, the outer-product
// write and the query read-out for one token.  Here one CTA owns one (b, hv) state
// S in R^{K x V} (fp32, key-major, 64 KiB at K = V = 128) and moves it through registers
// exactly once: every thread loads its rows of S with 128-bit streaming loads, and both
// reductions over K (p = k . S_dec and u = q . S_dec) come out of that single read.
// Value columns are independent in every step, so a state may be split into NSPLIT column
// blocks owned by separate CTAs (smaller CTAs, more of them resident per SM); each recomputes
// the per-token vectors and q . k it needs.
// The read-out uses q . S_t = q . S_dec + beta (q . k) r, which follows from steps 3-4 of
// the recurrence (KDA notes, "KDA 递归核心", §逐步公式), so S_t never has to be re-read.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

template <int K, int V, int NSPLIT = 1>
struct DecodeShape {
    static constexpr int VC = V / NSPLIT;                              // value columns per CTA
    static constexpr int NT = (K * VC / 4 < 256) ? K * VC / 4 : 256;  // threads per CTA
    static constexpr int TPR = VC / 4;                                 // threads per state row
    static constexpr int RPP = NT / TPR;                               // rows per pass
    static constexpr int R = K / RPP;                                  // rows per thread
    static_assert(R >= 1 && RPP * R == K && VC * NSPLIT == V, "decode shape");
};

template <typename T, int K, int V, int NSPLIT = 1>
__global__ void __launch_bounds__(DecodeShape<K, V, NSPLIT>::NT)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const T* __restrict__ g, const T* __restrict__ beta, const float* __restrict__ A_log,
                   const float* __restrict__ dt_bias, int H, int HV, int gate_mode, float lower_bound,
                   float scale, unsigned int flags, float* __restrict__ S, T* __restrict__ o) {
    using Sh = DecodeShape<K, V, NSPLIT>;
    constexpr int NT = Sh::NT, TPR = Sh::TPR, RPP = Sh::RPP, R = Sh::R, VC = Sh::VC;
    __shared__ float s_q[K], s_k[K], s_a[K];
    __shared__ float s_p[RPP][VC], s_u[RPP][VC];
    __shared__ float s_r[VC];
    __shared__ float s_qk, s_iq, s_ik;  // q . k; 1 / ||q||, 1 / ||k|| (1 unless q, k are normalised here)

    const int pair = blockIdx.x / NSPLIT;  // b * HV + hv
    const int v0 = (blockIdx.x - pair * NSPLIT) * VC;
    const int b = pair / HV, hv = pair - b * HV;
    const int h = hv / (HV / H);
    const int tid = threadIdx.x;
    const int cg = tid % TPR, rg = tid / TPR;
    float* Sp = S + (size_t)pair * K * V + v0;

    // 1. stream this thread's rows of S in first, so the loads are all in flight together
    float4 st[R];
#pragma unroll
    for (int i = 0; i < R; ++i) st[i] = __ldcs(reinterpret_cast<const float4*>(Sp + (size_t)(rg + RPP * i) * V + 4 * cg));

    // 2. per-token vectors: q, k of head h; decay factor exp(g) per key channel
    const float rate = (gate_mode != KDA_GATE_NONE) ? expf(A_log[hv]) : 0.0f;
    for (int d = tid; d < K; d += NT) {
        s_q[d] = to_f32(q[((size_t)b * H + h) * K + d]);
        s_k[d] = to_f32(k[((size_t)b * H + h) * K + d]);
        const float bias = (dt_bias != nullptr && gate_mode != KDA_GATE_NONE) ? dt_bias[hv * K + d] : 0.0f;
        s_a[d] = expf(gate_value(to_f32(g[(size_t)pair * K + d]), bias, rate, gate_mode, lower_bound));
    }
    __syncthreads();
    // q . k, and the norms when q and k are normalised here: the reductions below run on the raw
    // vectors and are rescaled where their results are used (p by 1/||k||, u by 1/||q||, the write
    // by 1/||k||), so the normalisation needs no extra pass over the state
    if (tid < 32) {
        float acc = 0.0f, qq = 0.0f, kk = 0.0f;
        for (int d = tid; d < K; d += 32) {
            acc += s_q[d] * s_k[d];
            qq += s_q[d] * s_q[d];
            kk += s_k[d] * s_k[d];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            acc += __shfl_xor_sync(0xffffffffu, acc, off);
            qq += __shfl_xor_sync(0xffffffffu, qq, off);
            kk += __shfl_xor_sync(0xffffffffu, kk, off);
        }
        if (tid == 0) {
            const bool norm = (flags & KDA_INPUT_L2NORM_QK) != 0;
            const float iq = norm ? inv_l2norm(qq) : 1.0f, ik = norm ? inv_l2norm(kk) : 1.0f;
            s_iq = iq;
            s_ik = ik;
            s_qk = acc * iq * ik;
        }
    }

    // 3. decay rows (step 1) and the two partial reductions over this thread's rows
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f), u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int d = rg + RPP * i;
        const float a = s_a[d], kd = s_k[d], qd = s_q[d];
        st[i].x *= a; st[i].y *= a; st[i].z *= a; st[i].w *= a;
        p.x += kd * st[i].x; p.y += kd * st[i].y; p.z += kd * st[i].z; p.w += kd * st[i].w;
        u.x += qd * st[i].x; u.y += qd * st[i].y; u.z += qd * st[i].z; u.w += qd * st[i].w;
    }
    *reinterpret_cast<float4*>(&s_p[rg][4 * cg]) = p;
    *reinterpret_cast<float4*>(&s_u[rg][4 * cg]) = u;
    __syncthreads();

    // 4. finish the reductions per value column: residual r (step 2) and the read-out (step 4)
    const float braw = to_f32(beta[pair]);
    const float bt = (flags & KDA_INPUT_BETA_LOGITS) ? beta_from_logit(braw) : braw;
    const float iq = s_iq, ik = s_ik;
    if (tid < VC) {
        float pp = 0.0f, uu = 0.0f;
#pragma unroll
        for (int j = 0; j < RPP; ++j) { pp += s_p[j][tid]; uu += s_u[j][tid]; }
        pp *= ik;
        uu *= iq;
        const float r = to_f32(v[(size_t)pair * V + v0 + tid]) - pp;
        s_r[tid] = r;
        o[(size_t)pair * V + v0 + tid] = from_f32<T>(scale * (uu + bt * s_qk * r));
    }
    __syncthreads();

    // 5. rank-1 write (step 3) and the single store of S_t
    const float4 r4 = *reinterpret_cast<const float4*>(&s_r[4 * cg]);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int d = rg + RPP * i;
        const float w = bt * ik * s_k[d];
        st[i].x += w * r4.x; st[i].y += w * r4.y; st[i].z += w * r4.z; st[i].w += w * r4.w;
        __stcs(reinterpret_cast<float4*>(Sp + (size_t)d * V + 4 * cg), st[i]);
    }
}

template <typename T, int K, int V, int NSPLIT = 1>
static cudaError_t launch_decode(const DecodeArgs& a) {
    using Sh = DecodeShape<K, V, NSPLIT>;
    decode_step_kernel<T, K, V, NSPLIT><<<a.B * a.HV * NSPLIT, Sh::NT, 0, a.stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        static_cast<const T*>(a.g), static_cast<const T*>(a.beta), a.A_log, a.dt_bias, a.H, a.HV, a.gate_mode,
        a.lower_bound, a.scale, a.flags, a.S, static_cast<T*>(a.o));
    return cudaGetLastError();
}

template <typename T, int K>
static cudaError_t dispatch_v(const DecodeArgs& a) {
    switch (a.V) {
        case 16: return launch_decode<T, K, 16>(a);
        case 32: return launch_decode<T, K, 32>(a);
        case 64: return launch_decode<T, K, 64>(a);
        // 128 value columns: two CTAs per state (32 KiB each) -- about 7 % more bandwidth than one
        // 64 KiB CTA per state on B256 H32 K=V=128, since more of the smaller CTAs stay resident
        case 128: return launch_decode<T, K, 128, 2>(a);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t dispatch_k(const DecodeArgs& a) {
    switch (a.K) {
        case 16: return dispatch_v<T, 16>(a);
        case 32: return dispatch_v<T, 32>(a);
        case 64: return dispatch_v<T, 64>(a);
        case 128: return dispatch_v<T, 128>(a);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_step(const DecodeArgs& a) {
    return a.dtype == KDA_BF16 ? dispatch_k<__nv_bfloat16>(a) : dispatch_k<float>(a);
}

}  // namespace kda
