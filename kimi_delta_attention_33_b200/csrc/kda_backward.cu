// kda_backward.cu -- reverse mode of the KDA forward pass (the gradient of a scalar loss through
// kda_chunk_fwd), on the FP32 CUDA cores.
//
// The pages define the forward method only; the adjoint here is derived from its four steps (KDA notes,
// "KDA 递归核心", §逐步公式) and the gate (KDA notes, "Gate 激活", table "两种 Gate"), one step at a time
// and in reverse order.  Per (b, hv) and token t, with a = exp(g_t) per key channel:
//   forward   S_dec = diag(a) S_{t-1};  r = v_t - k_t^T S_dec;  S_t = S_dec + beta_t k_t r^T;  o_t = s q_t^T S_t
//   reverse   dS += s q_t dO_t^T                      dq_t  = s S_t dO_t
//             u = dS^T k_t   (over key rows)          dbeta_t = u . r,  dr = beta_t u,  dv_t = dr
//             dk_t = beta_t dS r - S_dec dr           dS_dec = dS - k_t dr^T
//             dg_t = a (.) rowsum(dS_dec (.) S_{t-1})  dS = diag(a) dS_dec   (-> dS_{t-1})
// dq and dk of a q/k head add up over the value heads that read it (GVA), and every row quantity adds
// up over the value columns.
//
// Layout: one CTA per (b, hv, block of VB = min(V, 8) value columns); value columns are independent in
// the forward pass, so each CTA runs the recurrence on its columns alone.  Thread (row group rg, column
// group cg) holds rows rg + RPP i (i < R) and columns 4 cg .. 4 cg + 3 of the state and of dS in
// registers.  Reductions over key rows (the residual's prediction and u) go through warp shuffles and a
// double-buffered shared array; row quantities summed over this CTA's columns are added into the fp32
// outputs with atomics (the other column blocks and value heads add theirs).
//   1. forward sweep over all tokens, the state saved every CK tokens to the workspace;
//   2. the blocks of CK tokens in reverse: the block's states recomputed from its checkpoint into
//      shared memory, then its tokens in reverse order.
// The per-token inputs of a block (decay, k, q, v, dO, beta) are staged in shared memory once per block
// by loads that are all in flight together, so a token step does not wait for its own global loads.
// A second, elementwise kernel chains dg through the gate when the op applied it.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int BWD_CK = 8;  // tokens between saved states

template <int K, int V>
struct BwdShape {
    static constexpr int VB = V < 8 ? V : 8;                           // value columns per CTA
    static constexpr int NT = (K * VB / 4 < 128) ? K * VB / 4 : 128;   // threads
    static constexpr int TPR = VB / 4;                                 // threads per state row
    static constexpr int RPP = NT / TPR;                               // row groups
    static constexpr int R = K / RPP;                                  // rows per thread
    static constexpr int NW = NT / 32;                                 // warps
    static_assert(NT % 32 == 0 && RPP * R == K && TPR * 4 == VB, "backward shape");
    // sPrev [CK][K][VB], sR [CK][VB], sRed 2 x [NW][VB], then the staged block: decay, k, q [CK][K], v, dO [CK][VB],
    // beta [CK], and dt_bias [K]
    static constexpr size_t smem_floats = (size_t)BWD_CK * K * VB + (size_t)BWD_CK * VB + 2 * (size_t)NW * VB +
                                          3 * (size_t)BWD_CK * K + 2 * (size_t)BWD_CK * VB + BWD_CK + K;
    static constexpr size_t smem_bytes = smem_floats * sizeof(float);
};

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 f4_shfl_xor(float4 a, int off) {
    return make_float4(__shfl_xor_sync(0xffffffffu, a.x, off), __shfl_xor_sync(0xffffffffu, a.y, off),
                       __shfl_xor_sync(0xffffffffu, a.z, off), __shfl_xor_sync(0xffffffffu, a.w, off));
}

// Sum over all key rows of this CTA of a per-thread partial over its rows, for its four columns; every
// thread gets the result for its own columns.  `buf` alternates between two [NW][VB] arrays.
template <int TPR, int NW, int VB>
__device__ __forceinline__ float4 reduce_over_rows(float4 part, float* buf, int lane, int warp, int cg) {
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1) part = f4_add(part, f4_shfl_xor(part, off));
    if (lane < TPR) *reinterpret_cast<float4*>(buf + warp * VB + 4 * cg) = part;
    __syncthreads();
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) s = f4_add(s, *reinterpret_cast<const float4*>(buf + w * VB + 4 * cg));
    return s;
}

// Sum of x over this thread's four columns and the TPR lanes that share its rows (lanes cg = 0 .. TPR-1
// are adjacent); lane cg = 0 holds the total for the CTA's VB columns.
template <int TPR>
__device__ __forceinline__ float sum_over_cols(float4 x) {
    float s = (x.x + x.y) + (x.z + x.w);
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

}  // namespace

template <typename Elt, int K, int V>
__global__ void __launch_bounds__(BwdShape<K, V>::NT)
recurrent_bwd_kernel(const Elt* __restrict__ q, const Elt* __restrict__ k, const Elt* __restrict__ v,
                     const Elt* __restrict__ g, const Elt* __restrict__ beta, const float* __restrict__ A_log,
                     const float* __restrict__ dt_bias, const float* __restrict__ S0, const Elt* __restrict__ dO,
                     const float* __restrict__ dS_T, int T, int H, int HV, int gate_mode, float lower_bound,
                     float scale, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                     float* __restrict__ dg, float* __restrict__ dbeta, float* __restrict__ dS0,
                     float* __restrict__ ckpt) {
    using Sh = BwdShape<K, V>;
    constexpr int VB = Sh::VB, TPR = Sh::TPR, RPP = Sh::RPP, R = Sh::R, NW = Sh::NW, NVB = V / VB;
    extern __shared__ float bsm[];
    float* sPrev = bsm;                        // [CK][K][VB] state entering each token of the block
    float* sR = sPrev + BWD_CK * K * VB;       // [CK][VB] residuals
    float* sRed = sR + BWD_CK * VB;            // 2 x [NW][VB] reduction buffers
    float* sA = sRed + 2 * NW * VB;            // staged block: [CK][K] decay exp(g)
    float* sK = sA + BWD_CK * K;               //               [CK][K] k
    float* sQ = sK + BWD_CK * K;               //               [CK][K] q
    float* sV = sQ + BWD_CK * K;               //               [CK][VB] v (this CTA's columns)
    float* sDO = sV + BWD_CK * VB;             //               [CK][VB] dO
    float* sB = sDO + BWD_CK * VB;             //               [CK] beta
    float* sBias = sB + BWD_CK;                // [K] dt_bias (zeros when absent)

    const int vbi = blockIdx.x % NVB, pair = blockIdx.x / NVB;
    const int b = pair / HV, hv = pair - b * HV, h = hv / (HV / H);
    const int c0 = vbi * VB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid % TPR, rg = tid / TPR;
    const float rate = (gate_mode != KDA_GATE_NONE) ? expf(A_log[hv]) : 0.0f;
    for (int d = tid; d < K; d += Sh::NT)
        sBias[d] = (dt_bias != nullptr && gate_mode != KDA_GATE_NONE) ? dt_bias[hv * K + d] : 0.0f;
    const int NCK = (T + BWD_CK - 1) / BWD_CK;
    float* my_ckpt = ckpt + (size_t)blockIdx.x * NCK * K * VB;
    int red = 0;  // which reduction buffer the next reduction uses

    auto tok_qk = [&](int t) { return ((size_t)b * T + t) * H + h; };      // row of q / k (times K)
    auto tok_v = [&](int t) { return ((size_t)b * T + t) * HV + hv; };     // row of v, g, dO (times V or K)
    // the inputs of block blk's tokens into shared memory (rows past T left as they are: never read); callers
    // put a barrier before (the previous block's values are read no more) and after
    auto stage = [&](int blk, bool backward) {
        const int t0 = blk * BWD_CK, n = min(BWD_CK, T - t0);
        for (int idx = tid; idx < n * K; idx += Sh::NT) {
            const int j = idx / K, row = idx - j * K, t = t0 + j;
            sA[idx] = expf(gate_value(to_f32(g[tok_v(t) * K + row]), sBias[row], rate, gate_mode, lower_bound));
            sK[idx] = to_f32(k[tok_qk(t) * K + row]);
            if (backward) sQ[idx] = to_f32(q[tok_qk(t) * K + row]);
        }
        for (int idx = tid; idx < n * VB; idx += Sh::NT) {
            const int j = idx / VB, c = idx - j * VB, t = t0 + j;
            sV[idx] = to_f32(v[tok_v(t) * V + c0 + c]);
            if (backward) sDO[idx] = to_f32(dO[tok_v(t) * V + c0 + c]);
        }
        if (tid < n) sB[tid] = to_f32(beta[tok_v(t0 + tid)]);
    };
    auto reduce = [&](float4 part) {
        const float4 s = reduce_over_rows<TPR, NW, VB>(part, sRed + red * NW * VB, lane, warp, cg);
        red ^= 1;
        return s;
    };

    // one forward step on this thread's state rows, token j of the staged block: decay, residual (returned),
    // rank-1 write
    float4 S[R];
    auto forward_step = [&](int j) {
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
        float kd[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float a = sA[j * K + rg + RPP * i];
            kd[i] = sK[j * K + rg + RPP * i];
            S[i] = make_float4(a * S[i].x, a * S[i].y, a * S[i].z, a * S[i].w);
            p = make_float4(p.x + kd[i] * S[i].x, p.y + kd[i] * S[i].y, p.z + kd[i] * S[i].z, p.w + kd[i] * S[i].w);
        }
        p = reduce(p);
        const float4 vv = *reinterpret_cast<const float4*>(sV + j * VB + 4 * cg);
        const float4 r = make_float4(vv.x - p.x, vv.y - p.y, vv.z - p.z, vv.w - p.w);
        const float bt = sB[j];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float w = bt * kd[i];
            S[i] = make_float4(S[i].x + w * r.x, S[i].y + w * r.y, S[i].z + w * r.z, S[i].w + w * r.w);
        }
        return r;
    };

    // ---- 1. forward sweep, the entering state of every block of CK tokens saved ---------------------
#pragma unroll
    for (int i = 0; i < R; ++i)
        S[i] = S0 ? *reinterpret_cast<const float4*>(S0 + ((size_t)pair * K + rg + RPP * i) * V + c0 + 4 * cg)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int blk = 0; blk < NCK; ++blk) {
        __syncthreads();  // the previous block's staged inputs are read no more (and sBias is written, at the start)
        stage(blk, false);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4*>(my_ckpt + ((size_t)blk * K + rg + RPP * i) * VB + 4 * cg) = S[i];
        const int n = min(BWD_CK, T - blk * BWD_CK);
        for (int j = 0; j < n; ++j) forward_step(j);
    }

    // ---- 2. blocks in reverse ----------------------------------------------------------------------
    float4 dS[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
        dS[i] = dS_T ? *reinterpret_cast<const float4*>(dS_T + ((size_t)pair * K + rg + RPP * i) * V + c0 + 4 * cg)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int blk = NCK - 1; blk >= 0; --blk) {
        const int t0 = blk * BWD_CK, n = min(BWD_CK, T - t0);
        __syncthreads();  // the previous block's staged inputs are read no more
        stage(blk, true);
        __syncthreads();
        // recompute: the state entering each token into shared memory (each thread its own entries),
        // the residuals too; S ends as the state after the block's last token
#pragma unroll
        for (int i = 0; i < R; ++i)
            S[i] = *reinterpret_cast<const float4*>(my_ckpt + ((size_t)blk * K + rg + RPP * i) * VB + 4 * cg);
        for (int j = 0; j < n; ++j) {
#pragma unroll
            for (int i = 0; i < R; ++i)
                *reinterpret_cast<float4*>(sPrev + ((size_t)j * K + rg + RPP * i) * VB + 4 * cg) = S[i];
            const float4 r = forward_step(j);
            *reinterpret_cast<float4*>(sR + j * VB + 4 * cg) = r;  // same values from every row group
        }
        // reverse through the block; S holds the state after token t
        for (int j = n - 1; j >= 0; --j) {
            const int t = t0 + j;
            const size_t rq = tok_qk(t) * K, rv = tok_v(t);
            const float4 dOc = *reinterpret_cast<const float4*>(sDO + j * VB + 4 * cg);
            float qd[R], kd[R], a[R];
#pragma unroll
            for (int i = 0; i < R; ++i) {
                a[i] = sA[j * K + rg + RPP * i];
                qd[i] = sQ[j * K + rg + RPP * i];
                kd[i] = sK[j * K + rg + RPP * i];
            }
            // dq_t = s S_t dO_t ; dS += s q_t dO_t^T
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float part =
                    sum_over_cols<TPR>(make_float4(S[i].x * dOc.x, S[i].y * dOc.y, S[i].z * dOc.z, S[i].w * dOc.w));
                if (cg == 0) atomicAdd(dq + rq + rg + RPP * i, scale * part);
                const float w = scale * qd[i];
                dS[i] = make_float4(dS[i].x + w * dOc.x, dS[i].y + w * dOc.y, dS[i].z + w * dOc.z, dS[i].w + w * dOc.w);
            }
            // u = dS^T k_t over the key rows
            float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < R; ++i)
                u = make_float4(u.x + kd[i] * dS[i].x, u.y + kd[i] * dS[i].y, u.z + kd[i] * dS[i].z, u.w + kd[i] * dS[i].w);
            u = reduce(u);
            const float4 r = *reinterpret_cast<const float4*>(sR + j * VB + 4 * cg);
            const float bt = sB[j];
            const float4 dr = make_float4(bt * u.x, bt * u.y, bt * u.z, bt * u.w);
            if (rg == 0) {  // dbeta_t = u . r over this CTA's columns; dv_t = dr
                float db = dot4(u, r);
#pragma unroll
                for (int off = 1; off < TPR; off <<= 1) db += __shfl_xor_sync((1u << TPR) - 1u, db, off);
                if (cg == 0) atomicAdd(dbeta + rv, db);
                *reinterpret_cast<float4*>(dv + rv * V + c0 + 4 * cg) = dr;
            }
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float4 Sp = *reinterpret_cast<const float4*>(sPrev + ((size_t)j * K + rg + RPP * i) * VB + 4 * cg);
                const float4 Sd = make_float4(a[i] * Sp.x, a[i] * Sp.y, a[i] * Sp.z, a[i] * Sp.w);
                // dk_t = beta dS r - S_dec dr
                const float pk = sum_over_cols<TPR>(make_float4(bt * dS[i].x * r.x - Sd.x * dr.x, bt * dS[i].y * r.y - Sd.y * dr.y,
                                                                bt * dS[i].z * r.z - Sd.z * dr.z, bt * dS[i].w * r.w - Sd.w * dr.w));
                if (cg == 0) atomicAdd(dk + rq + rg + RPP * i, pk);
                // dS_dec = dS - k dr^T ; dg_t = a rowsum(dS_dec S_{t-1}) ; dS_{t-1} = a dS_dec
                const float4 dSd = make_float4(dS[i].x - kd[i] * dr.x, dS[i].y - kd[i] * dr.y, dS[i].z - kd[i] * dr.z,
                                               dS[i].w - kd[i] * dr.w);
                const float pg = sum_over_cols<TPR>(make_float4(dSd.x * Sp.x, dSd.y * Sp.y, dSd.z * Sp.z, dSd.w * Sp.w));
                if (cg == 0) atomicAdd(dg + rv * K + rg + RPP * i, a[i] * pg);
                dS[i] = make_float4(a[i] * dSd.x, a[i] * dSd.y, a[i] * dSd.z, a[i] * dSd.w);
                S[i] = Sp;
            }
        }
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4*>(dS0 + ((size_t)pair * K + rg + RPP * i) * V + c0 + 4 * cg) = dS[i];
    }
}

// dg (with respect to the gate output, the log decay) chained back through the gate, in place, with the
// parameter gradients (KDA notes, "Gate 激活": input x = g_raw + dt_bias, rate = exp(A_log)):
//   SAFE      g = L sigmoid(rate x):  dg/dx = L s (1 - s) rate,  dg/dA_log = L s (1 - s) rate x
//   STANDARD  g = -rate softplus(x):  dg/dx = -rate sigmoid(x),  dg/dA_log = -rate softplus(x)
// One CTA per (block of 64 tokens, value head), thread = key channel: the token loop sums ddt_bias and
// dA_log per channel, then one atomic per channel and one per CTA.
template <typename Elt>
__global__ void __launch_bounds__(128)
gate_bwd_kernel(const Elt* __restrict__ g_raw, const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                long long rows, int HV, int K, int mode, float lower_bound, float* __restrict__ dg,
                float* __restrict__ ddt_bias, float* __restrict__ dA_log) {
    __shared__ float s_part[4];
    const int hv = blockIdx.y;
    const long long r0 = (long long)blockIdx.x * 64;
    const float rate = expf(A_log[hv]);
    float acc_a = 0.f;
    for (int d = threadIdx.x; d < K; d += blockDim.x) {
        const float bias = dt_bias ? dt_bias[hv * K + d] : 0.0f;
        float sb = 0.f;
        for (long long rr = r0; rr < r0 + 64 && rr < rows; ++rr) {
            const size_t idx = ((size_t)rr * HV + hv) * K + d;
            const float x = to_f32(g_raw[idx]) + bias;
            float dgdx, dgda;
            if (mode == KDA_GATE_SAFE) {
                const float z = rate * x;
                const float s = 1.0f / (1.0f + expf(-z));
                dgdx = lower_bound * s * (1.0f - s) * rate;
                dgda = lower_bound * s * (1.0f - s) * z;
            } else {
                const float s = 1.0f / (1.0f + expf(-x));
                const float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
                dgdx = -rate * s;
                dgda = -rate * sp;
            }
            const float gd = dg[idx];
            dg[idx] = gd * dgdx;
            sb += gd * dgdx;
            acc_a += gd * dgda;
        }
        if (ddt_bias) atomicAdd(ddt_bias + hv * K + d, sb);
    }
    float s = acc_a;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0 && dA_log) atomicAdd(dA_log + hv, s_part[0] + s_part[1] + s_part[2] + s_part[3]);
}

namespace {

template <typename Elt, int K, int V>
cudaError_t launch_bwd(const BackwardArgs& a) {
    using Sh = BwdShape<K, V>;
    auto kern = recurrent_bwd_kernel<Elt, K, V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((long long)a.B * a.HV * (V / Sh::VB)), Sh::NT, Sh::smem_bytes, a.stream>>>(
        static_cast<const Elt*>(a.q), static_cast<const Elt*>(a.k), static_cast<const Elt*>(a.v),
        static_cast<const Elt*>(a.g), static_cast<const Elt*>(a.beta), a.A_log, a.dt_bias, a.S0,
        static_cast<const Elt*>(a.dO), a.dS_T, a.T, a.H, a.HV, a.gate_mode, a.lower_bound, a.scale, a.dq, a.dk, a.dv,
        a.dg, a.dbeta, a.dS0, static_cast<float*>(a.workspace));
    return cudaGetLastError();
}

template <typename Elt, int K>
cudaError_t bwd_v(const BackwardArgs& a) {
    switch (a.V) {
        case 16: return launch_bwd<Elt, K, 16>(a);
        case 32: return launch_bwd<Elt, K, 32>(a);
        case 64: return launch_bwd<Elt, K, 64>(a);
        case 128: return launch_bwd<Elt, K, 128>(a);
    }
    return cudaErrorInvalidValue;
}

template <typename Elt>
cudaError_t bwd_k(const BackwardArgs& a) {
    switch (a.K) {
        case 16: return bwd_v<Elt, 16>(a);
        case 32: return bwd_v<Elt, 32>(a);
        case 64: return bwd_v<Elt, 64>(a);
        case 128: return bwd_v<Elt, 128>(a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t backward_workspace(int B, int T, int HV, int K, int V) {
    const size_t nck = ((size_t)T + BWD_CK - 1) / BWD_CK;
    return (size_t)B * HV * nck * K * V * sizeof(float);
}

cudaError_t launch_backward(const BackwardArgs& a) {
    // the outputs that several CTAs add into start at zero
    const size_t nqk = (size_t)a.B * a.T * a.H * a.K, ng = (size_t)a.B * a.T * a.HV * a.K;
    cudaError_t e;
    if ((e = cudaMemsetAsync(a.dq, 0, nqk * sizeof(float), a.stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dk, 0, nqk * sizeof(float), a.stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dg, 0, ng * sizeof(float), a.stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dbeta, 0, (size_t)a.B * a.T * a.HV * sizeof(float), a.stream)) != cudaSuccess) return e;
    e = a.dtype == KDA_BF16 ? bwd_k<__nv_bfloat16>(a) : bwd_k<float>(a);
    if (e != cudaSuccess || a.gate_mode == KDA_GATE_NONE) return e;
    if (a.ddt_bias && (e = cudaMemsetAsync(a.ddt_bias, 0, (size_t)a.HV * a.K * sizeof(float), a.stream)) != cudaSuccess)
        return e;
    if (a.dA_log && (e = cudaMemsetAsync(a.dA_log, 0, (size_t)a.HV * sizeof(float), a.stream)) != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.T;
    const dim3 grid((unsigned)((rows + 63) / 64), (unsigned)a.HV);
    if (a.dtype == KDA_BF16)
        gate_bwd_kernel<__nv_bfloat16><<<grid, 128, 0, a.stream>>>(static_cast<const __nv_bfloat16*>(a.g), a.A_log,
                                                                   a.dt_bias, rows, a.HV, a.K, a.gate_mode,
                                                                   a.lower_bound, a.dg, a.ddt_bias, a.dA_log);
    else
        gate_bwd_kernel<float><<<grid, 128, 0, a.stream>>>(static_cast<const float*>(a.g), a.A_log, a.dt_bias, rows,
                                                           a.HV, a.K, a.gate_mode, a.lower_bound, a.dg, a.ddt_bias,
                                                           a.dA_log);
    return cudaGetLastError();
}

}  // namespace kda
