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
// Layout: one warp per (b, hv, block of VB value columns); value columns are independent in the forward
// pass, so each warp runs the recurrence on its columns alone, and a CTA holds NWB such warps of one
// (b, hv), which share the staged per-token inputs.  Lane (row group rg, column group cg) holds rows
// R rg .. R rg + R - 1 and columns 2 cg, 2 cg + 1 of the warp's block of the state and of dS in registers, as
// pairs for the packed fp32x2 arithmetic, so reductions over key rows (the residual's prediction and u)
// are warp shuffles, with no barrier on the per-token chain; two columns a lane keep the chain short and
// give each SM sub-partition two warps to interleave.  Row quantities (dq, dk, dg) and dbeta, summed over
// each warp's columns, are kept per warp in shared memory for the block of tokens, then summed over the
// CTA's warps and added into the fp32 outputs (one float4 atomic per four key channels; the other CTAs
// of the value head, and the other value heads of a q/k head, add theirs).
//   1. forward sweep over all tokens, the state saved every CK tokens and the residual r of every token
//      to the workspace;
//   2. the blocks of CK tokens in reverse: the block's states recomputed from its checkpoint into
//      shared memory (with the saved residuals this is a rank-1 update a token, no reduction), then its
//      tokens in reverse order.
// The per-token inputs of a block (decay, k, q, v, dO, beta) are staged in shared memory once per block,
// from 16-byte loads; the next block's are loaded into registers while this one is computed.  The decay
// a = exp(gate) is computed once per (token, value head, key channel) by a small elementwise kernel into
// the workspace, not again by every CTA that reads it.
// A second, elementwise kernel chains dg through the gate when the op applied it.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int BWD_CK = 8;          // tokens between saved states
constexpr int GATE_BWD_ROWS = 16;  // (b, t) rows per CTA of the gate's backward

template <int K, int V>
struct BwdShape {
    static constexpr int RG = K < 32 ? K : 32;                       // row groups (lanes along the key rows)
    static constexpr int TPR = 32 / RG;                              // lanes along the value columns
    static constexpr int VB = 2 * TPR;                               // value columns per warp
    static constexpr int R = K / RG;                                 // rows per lane
    static constexpr int NCB = V / VB;                               // column blocks per (b, hv)
    static constexpr int NWB = NCB < 4 ? NCB : 4;                    // warps (column blocks) per CTA
    static constexpr int NT = 32 * NWB;                              // threads
    static constexpr int CW = NWB * VB;                              // value columns per CTA
    // 16-byte vectors a thread loads per block: decay (fp32) rows, k / q rows, v / dO columns (VN elements a vector)
    template <typename Elt> static constexpr int VN = 16 / (int)sizeof(Elt);
    static constexpr int EA = (BWD_CK * K / 4 + NT - 1) / NT;
    template <typename Elt> static constexpr int EK = (BWD_CK * K / VN<Elt> + NT - 1) / NT;
    template <typename Elt> static constexpr int EV = (BWD_CK * CW / VN<Elt> + NT - 1) / NT;
    static constexpr int ER = (BWD_CK * CW / 4 + NT - 1) / NT;  // saved residuals (fp32)
    static_assert(RG * TPR == 32 && R * RG == K && NCB % NWB == 0, "backward shape");
    static_assert(K % 16 == 0 && CW % 8 == 0, "16-byte staging vectors");
    // sPrev [NWB][CK][K][VB]; the staged block: decay, k, q [CK][K], v, dO, r [CK][CW], beta [CK]; the block's
    // per-warp row sums dq, dk, dg [NWB][CK][K] and dbeta [NWB][CK]
    static constexpr size_t smem_floats = (size_t)NWB * BWD_CK * K * VB + 3 * (size_t)BWD_CK * K +
                                          3 * (size_t)BWD_CK * CW + BWD_CK + 3 * (size_t)NWB * BWD_CK * K +
                                          (size_t)NWB * BWD_CK;
    static constexpr size_t smem_bytes = smem_floats * sizeof(float);
};

// packed fp32x2 arithmetic (each half rounded as the scalar operation)
__device__ __forceinline__ float2 f2_splat(float s) { return make_float2(s, s); }
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }

// a 16-byte vector of inputs, as fp32, into shared memory (dst 16-byte aligned)
__device__ __forceinline__ void put_f32(float* dst, uint4 raw, const float*) { *reinterpret_cast<uint4*>(dst) = raw; }
__device__ __forceinline__ void put_f32(float* dst, uint4 raw, const __nv_bfloat16*) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);  // bf16 is the top half of an fp32
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }

// Sum over the warp's key rows of a per-lane partial over its rows, for its two columns; every lane gets
// the result for its own columns (the lanes of a column group differ in the bits from TPR up).
template <int TPR>
__device__ __forceinline__ float2 sum_over_rows(float2 part) {
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1)
        part = f2_add(part, make_float2(__shfl_xor_sync(0xffffffffu, part.x, off), __shfl_xor_sync(0xffffffffu, part.y, off)));
    return part;
}

// Sum of x over this lane's two columns and the TPR lanes that share its rows (lanes cg = 0 .. TPR-1
// are adjacent); every one of them gets the total for the warp's VB columns.
template <int TPR>
__device__ __forceinline__ float sum_over_cols(float2 x) {
    float s = x.x + x.y;
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// R consecutive floats (a lane's key rows) from / to shared memory, as one vector access (R in {1, 2, 4};
// the address is R-float aligned)
template <int R>
__device__ __forceinline__ void rows_of(const float* p, float (&x)[R]) {
    if constexpr (R == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x, x[1] = v.y, x[2] = v.z, x[3] = v.w;
    } else if constexpr (R == 2) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x, x[1] = v.y;
    } else {
        x[0] = *p;
    }
}
template <int R>
__device__ __forceinline__ void put_rows(float* p, const float (&x)[R]) {
    if constexpr (R == 4) *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else if constexpr (R == 2) *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    else *p = x[0];
}

}  // namespace

template <typename Elt, int K, int V>
__global__ void __launch_bounds__(BwdShape<K, V>::NT)
recurrent_bwd_kernel(const Elt* __restrict__ q, const Elt* __restrict__ k, const Elt* __restrict__ v,
                     const float* __restrict__ decay, const Elt* __restrict__ beta, const float* __restrict__ S0,
                     const Elt* __restrict__ dO, const float* __restrict__ dS_T, int T, int H, int HV, float scale,
                     float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dg,
                     float* __restrict__ dbeta, float* __restrict__ dS0, float* __restrict__ ckpt,
                     float* __restrict__ rres) {
    using Sh = BwdShape<K, V>;
    constexpr int VB = Sh::VB, TPR = Sh::TPR, R = Sh::R, NT = Sh::NT, NWB = Sh::NWB, CW = Sh::CW;
    constexpr int CK = BWD_CK, VN = Sh::template VN<Elt>, EA = Sh::EA, EK = Sh::template EK<Elt>,
                  EV = Sh::template EV<Elt>, ER = Sh::ER;
    extern __shared__ float bsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* sPrev = bsm + (size_t)warp * CK * K * VB;  // [CK][R][32 lanes][2] state entering each token (this warp's)
    float* sA = bsm + (size_t)NWB * CK * K * VB;  // staged block: [CK][K] decay exp(g)
    float* sK = sA + CK * K;                   //               [CK][K] k
    float* sQ = sK + CK * K;                   //               [CK][K] q
    float* sV = sQ + CK * K;                   //               [CK][CW] v (this CTA's columns)
    float* sDO = sV + CK * CW;                 //               [CK][CW] dO
    float* sRr = sDO + CK * CW;                //               [CK][CW] r (saved by the forward sweep)
    float* sB = sRr + CK * CW;                 //               [CK] beta
    float* sDq = sB + CK;                      // [NWB][CK][K] dq of the block, each warp's over its columns
    float* sDk = sDq + NWB * CK * K;           // [NWB][CK][K] dk
    float* sDg = sDk + NWB * CK * K;           // [NWB][CK][K] dg
    float* sDb = sDg + NWB * CK * K;           // [NWB][CK] dbeta
    float* wDq = sDq + warp * CK * K;          // this warp's
    float* wDk = sDk + warp * CK * K;
    float* wDg = sDg + warp * CK * K;

    constexpr int CPP = Sh::NCB / NWB;         // CTAs per (b, hv)
    const int pair = blockIdx.x / CPP;
    const int b = pair / HV, hv = pair - b * HV, h = hv / (HV / H);
    const int cc0 = (blockIdx.x - pair * CPP) * CW;  // first value column of the CTA
    const int c0 = cc0 + warp * VB;                  // first value column of the warp
    const int cg = lane % TPR, rg = lane / TPR;
    const int NCK = (T + CK - 1) / CK;
    float* my_ckpt = ckpt + ((size_t)pair * Sh::NCB + c0 / VB) * NCK * K * VB;

    auto tok_qk = [&](int t) { return ((size_t)b * T + t) * H + h; };      // row of q / k (times K)
    auto tok_v = [&](int t) { return ((size_t)b * T + t) * HV + hv; };     // row of v, g, dO (times V or K)

    // the next block's inputs as loaded: 16-byte vectors of decay rows, k / q rows, and the CTA's v / dO columns
    uint4 la[EA], lk[EK], lq[EK], lv[EV], lo[EV];
    float4 lr[ER];
    Elt lb;
    constexpr int KV = K / VN, CV = CW / VN;  // vectors in a k / q row, in the CTA's v / dO columns
    auto load_block = [&](int blk, bool backward) {
        const int t0 = blk * CK, n = min(CK, T - t0);
#pragma unroll
        for (int e = 0; e < EA; ++e) {
            const int idx = tid + e * NT, j = idx / (K / 4), x = idx - j * (K / 4);
            if (idx < n * (K / 4)) la[e] = reinterpret_cast<const uint4*>(decay + tok_v(t0 + j) * K)[x];
        }
#pragma unroll
        for (int e = 0; e < EK; ++e) {
            const int idx = tid + e * NT, j = idx / KV, x = idx - j * KV;
            if (idx < n * KV) {
                lk[e] = reinterpret_cast<const uint4*>(k + tok_qk(t0 + j) * K)[x];
                if (backward) lq[e] = reinterpret_cast<const uint4*>(q + tok_qk(t0 + j) * K)[x];
            }
        }
#pragma unroll
        for (int e = 0; e < EV; ++e) {
            const int idx = tid + e * NT, j = idx / CV, x = idx - j * CV;
            if (idx < n * CV) {
                lv[e] = reinterpret_cast<const uint4*>(v + tok_v(t0 + j) * V + cc0)[x];
                if (backward) lo[e] = reinterpret_cast<const uint4*>(dO + tok_v(t0 + j) * V + cc0)[x];
            }
        }
        if (backward) {
#pragma unroll
            for (int e = 0; e < ER; ++e) {  // written by this CTA in the forward sweep: read through L2
                const int idx = tid + e * NT, j = idx / (CW / 4), x = idx - j * (CW / 4);
                if (idx < n * (CW / 4)) lr[e] = __ldcg(reinterpret_cast<const float4*>(rres + tok_v(t0 + j) * V + cc0) + x);
            }
        }
        if (tid < n) lb = beta[tok_v(t0 + tid)];
    };
    // the loaded block into shared memory as fp32 (rows past T are never read); callers put a barrier
    // before (the previous block's staged values are read no more) and after
    auto stage_block = [&](int n, bool backward) {
#pragma unroll
        for (int e = 0; e < EA; ++e) {
            const int idx = tid + e * NT;
            if (idx < n * (K / 4)) *reinterpret_cast<uint4*>(sA + 4 * idx) = la[e];
        }
#pragma unroll
        for (int e = 0; e < EK; ++e) {
            const int idx = tid + e * NT;
            if (idx < n * KV) {
                put_f32(sK + VN * idx, lk[e], k);
                if (backward) put_f32(sQ + VN * idx, lq[e], q);
            }
        }
#pragma unroll
        for (int e = 0; e < EV; ++e) {
            const int idx = tid + e * NT;
            if (idx < n * CV) {
                put_f32(sV + VN * idx, lv[e], v);
                if (backward) put_f32(sDO + VN * idx, lo[e], dO);
            }
        }
        if (backward) {
#pragma unroll
            for (int e = 0; e < ER; ++e) {
                const int idx = tid + e * NT;
                if (idx < n * (CW / 4)) *reinterpret_cast<float4*>(sRr + 4 * idx) = lr[e];
            }
        }
        if (tid < n) sB[tid] = to_f32(lb);
    };

    // one forward step on this lane's state entries, token j of the staged block: decay, residual
    // (returned), rank-1 write
    float2 S[R];
    auto forward_step = [&](int j) {
        float a[R], kd[R];
        rows_of<R>(sA + j * K + R * rg, a);
        rows_of<R>(sK + j * K + R * rg, kd);
        float2 p = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            S[i] = f2_mul(f2_splat(a[i]), S[i]);
            p = f2_fma(f2_splat(kd[i]), S[i], p);
        }
        p = sum_over_rows<TPR>(p);
        const float2 r = f2_sub(*reinterpret_cast<const float2*>(sV + j * CW + warp * VB + 2 * cg), p);
        const float bt = sB[j];
#pragma unroll
        for (int i = 0; i < R; ++i) S[i] = f2_fma(f2_splat(bt * kd[i]), r, S[i]);
        return r;
    };
    // this lane's state entries in a warp-private copy (saved states, sPrev): entry i of lane l is the pair
    // 32 i + l, so a warp's access to one entry covers 256 contiguous bytes
    auto put_state = [&](float* dst, const float2 (&x)[R]) {
#pragma unroll
        for (int i = 0; i < R; ++i) reinterpret_cast<float2*>(dst)[32 * i + lane] = x[i];
    };
    auto get_state = [&](const float* src, float2 (&x)[R]) {
#pragma unroll
        for (int i = 0; i < R; ++i) x[i] = reinterpret_cast<const float2*>(src)[32 * i + lane];
    };
    constexpr int KVB = K * VB;  // floats of one warp's state block

    // ---- 1. forward sweep, the entering state of every block of CK tokens saved ---------------------
#pragma unroll
    for (int i = 0; i < R; ++i)
        S[i] = S0 ? *reinterpret_cast<const float2*>(S0 + ((size_t)pair * K + R * rg + i) * V + c0 + 2 * cg)
                  : make_float2(0.f, 0.f);
    // the residuals of a block gather in sRr and go to the workspace after the next barrier
    auto store_residuals = [&](int blk) {
        const int t0 = blk * CK, n = min(CK, T - t0);
        for (int idx = tid; idx < n * (CW / 4); idx += NT) {
            const int j = idx / (CW / 4), x = idx - j * (CW / 4);
            reinterpret_cast<float4*>(rres + tok_v(t0 + j) * V + cc0)[x] = *reinterpret_cast<const float4*>(sRr + 4 * idx);
        }
    };
    load_block(0, false);
    for (int blk = 0; blk < NCK; ++blk) {
        const int n = min(CK, T - blk * CK);
        __syncthreads();  // the previous block's staged inputs are read no more, its residuals are complete
        if (blk > 0) store_residuals(blk - 1);  // (the forward stage leaves sRr alone)
        stage_block(n, false);
        __syncthreads();  // and stored: sRr is rewritten from here
        if (blk + 1 < NCK) load_block(blk + 1, false);
        put_state(my_ckpt + (size_t)blk * KVB, S);
        for (int j = 0; j < n; ++j) {
            const float2 r = forward_step(j);
            if (rg == 0) *reinterpret_cast<float2*>(sRr + j * CW + warp * VB + 2 * cg) = r;
        }
    }
    __syncthreads();
    store_residuals(NCK - 1);
    __syncthreads();  // the last block's residuals are read back below, by other threads

    // ---- 2. blocks in reverse ----------------------------------------------------------------------
    float2 dS[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
        dS[i] = dS_T ? *reinterpret_cast<const float2*>(dS_T + ((size_t)pair * K + R * rg + i) * V + c0 + 2 * cg)
                     : make_float2(0.f, 0.f);
    load_block(NCK - 1, true);
    float2 Sck[R];  // the checkpoint of the block processed next, loaded a block ahead
    get_state(my_ckpt + (size_t)(NCK - 1) * KVB, Sck);
    for (int blk = NCK - 1; blk >= 0; --blk) {
        const int t0 = blk * CK, n = min(CK, T - t0);
        __syncthreads();  // the previous block's staged inputs and row sums are read no more
        stage_block(n, true);
        __syncthreads();
        if (blk > 0) load_block(blk - 1, true);
        // recompute: the state entering each token into shared memory (each lane its own entries), from the
        // saved residuals (the same operations as the forward sweep, so the same values); S ends as the state
        // after the block's last token
#pragma unroll
        for (int i = 0; i < R; ++i) S[i] = Sck[i];
        if (blk > 0) get_state(my_ckpt + (size_t)(blk - 1) * KVB, Sck);
        for (int j = 0; j < n; ++j) {
            put_state(sPrev + j * KVB, S);
            float a[R], kd[R];
            rows_of<R>(sA + j * K + R * rg, a);
            rows_of<R>(sK + j * K + R * rg, kd);
            const float2 r = *reinterpret_cast<const float2*>(sRr + j * CW + warp * VB + 2 * cg);
            const float bt = sB[j];
#pragma unroll
            for (int i = 0; i < R; ++i) S[i] = f2_fma(f2_splat(bt * kd[i]), r, f2_mul(f2_splat(a[i]), S[i]));
        }
        // reverse through the block; S holds the state after token t
        for (int j = n - 1; j >= 0; --j) {
            // dOs = s dO_t (this lane's columns)
            const float2 dOs = f2_mul(f2_splat(scale), *reinterpret_cast<const float2*>(sDO + j * CW + warp * VB + 2 * cg));
            float a[R], qd[R], kd[R];
            rows_of<R>(sA + j * K + R * rg, a);
            rows_of<R>(sQ + j * K + R * rg, qd);
            rows_of<R>(sK + j * K + R * rg, kd);
            // dq_t = s S_t dO_t ; dS += s q_t dO_t^T
            float pq[R];
#pragma unroll
            for (int i = 0; i < R; ++i) {
                pq[i] = sum_over_cols<TPR>(f2_mul(S[i], dOs));
                dS[i] = f2_fma(f2_splat(qd[i]), dOs, dS[i]);
            }
            if (cg == 0) put_rows<R>(wDq + j * K + R * rg, pq);
            // u = dS^T k_t over the key rows
            float2 u = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < R; ++i) u = f2_fma(f2_splat(kd[i]), dS[i], u);
            u = sum_over_rows<TPR>(u);
            const float2 r = *reinterpret_cast<const float2*>(sRr + j * CW + warp * VB + 2 * cg);
            const float bt = sB[j];
            const float2 dr = f2_mul(f2_splat(bt), u), ndr = make_float2(-dr.x, -dr.y);
            if (rg == 0) {  // dbeta_t = u . r over this warp's columns; dv_t = dr
                float db = u.x * r.x + u.y * r.y;
#pragma unroll
                for (int off = 1; off < TPR; off <<= 1) db += __shfl_xor_sync((1u << TPR) - 1u, db, off);
                if (cg == 0) sDb[warp * CK + j] = db;
                *reinterpret_cast<float2*>(dv + tok_v(t0 + j) * V + c0 + 2 * cg) = dr;
            }
            const float2 btr = f2_mul(f2_splat(bt), r);
            float pk[R], pg[R];
            float2 Sp[R];
            get_state(sPrev + j * KVB, Sp);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                // dk_t = beta dS r - S_dec dr,  S_dec = a S_{t-1}
                pk[i] = sum_over_cols<TPR>(f2_fma(dS[i], btr, f2_mul(f2_mul(f2_splat(a[i]), Sp[i]), ndr)));
                // dS_dec = dS - k dr^T ; dg_t = a rowsum(dS_dec S_{t-1}) ; dS_{t-1} = a dS_dec
                const float2 dSd = f2_fma(f2_splat(kd[i]), ndr, dS[i]);
                pg[i] = a[i] * sum_over_cols<TPR>(f2_mul(dSd, Sp[i]));
                dS[i] = f2_mul(f2_splat(a[i]), dSd);
                S[i] = Sp[i];
            }
            if (cg == 0) {
                put_rows<R>(wDk + j * K + R * rg, pk);
                put_rows<R>(wDg + j * K + R * rg, pg);
            }
        }
        __syncthreads();  // the block's row sums are complete
        for (int idx = tid; idx < n * (K / 4); idx += NT) {  // four key channels at a time
            const int j = idx / (K / 4), row = 4 * (idx - j * (K / 4));
            float4 sq = make_float4(0.f, 0.f, 0.f, 0.f), sk = sq, sg = sq;
#pragma unroll
            for (int w = 0; w < NWB; ++w) {
                sq = f4_add(sq, *reinterpret_cast<const float4*>(sDq + w * CK * K + 4 * idx));
                sk = f4_add(sk, *reinterpret_cast<const float4*>(sDk + w * CK * K + 4 * idx));
                sg = f4_add(sg, *reinterpret_cast<const float4*>(sDg + w * CK * K + 4 * idx));
            }
            atomicAdd(reinterpret_cast<float4*>(dq + tok_qk(t0 + j) * K + row), sq);
            atomicAdd(reinterpret_cast<float4*>(dk + tok_qk(t0 + j) * K + row), sk);
            atomicAdd(reinterpret_cast<float4*>(dg + tok_v(t0 + j) * K + row), sg);
        }
        if (tid < n) {
            float sb = 0.f;
#pragma unroll
            for (int w = 0; w < NWB; ++w) sb += sDb[w * CK + tid];
            atomicAdd(dbeta + tok_v(t0 + tid), sb);
        }
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < R; ++i)
            *reinterpret_cast<float2*>(dS0 + ((size_t)pair * K + R * rg + i) * V + c0 + 2 * cg) = dS[i];
    }
}

// a = exp(gate(g_raw)) per (b, t, hv, key channel), fp32: the per-token decays of the recurrence (with
// GATE_NONE g is the log decay itself).
template <typename Elt>
__global__ void __launch_bounds__(256)
decay_kernel(const Elt* __restrict__ g, const float* __restrict__ A_log, const float* __restrict__ dt_bias, long long n,
             int HV, int K, int mode, float lower_bound, float* __restrict__ a) {
    for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
        const int d = (int)(i % K), hv = (int)((i / K) % HV);
        const float rate = mode != KDA_GATE_NONE ? expf(A_log[hv]) : 0.0f;
        const float bias = (dt_bias != nullptr && mode != KDA_GATE_NONE) ? dt_bias[hv * K + d] : 0.0f;
        a[i] = expf(gate_value(to_f32(g[i]), bias, rate, mode, lower_bound));
    }
}

// dg (with respect to the gate output, the log decay) chained back through the gate, in place, with the
// parameter gradients (KDA notes, "Gate 激活": input x = g_raw + dt_bias, rate = exp(A_log)):
//   SAFE      g = L sigmoid(rate x):  dg/dx = L s (1 - s) rate,  dg/dA_log = L s (1 - s) rate x
//   STANDARD  g = -rate softplus(x):  dg/dx = -rate sigmoid(x),  dg/dA_log = -rate softplus(x)
// One CTA per (block of GATE_BWD_ROWS (b, t) rows, value head), thread = key channel: the row loop sums
// ddt_bias and dA_log per channel, then one atomic per channel and one per CTA.
template <typename Elt>
__global__ void __launch_bounds__(128)
gate_bwd_kernel(const Elt* __restrict__ g_raw, const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                long long rows, int HV, int K, int mode, float lower_bound, float* __restrict__ dg,
                float* __restrict__ ddt_bias, float* __restrict__ dA_log) {
    __shared__ float s_part[4];
    const int hv = blockIdx.y;
    const long long r0 = (long long)blockIdx.x * GATE_BWD_ROWS;
    const float rate = expf(A_log[hv]);
    float acc_a = 0.f;
    for (int d = threadIdx.x; d < K; d += blockDim.x) {
        const float bias = dt_bias ? dt_bias[hv * K + d] : 0.0f;
        float sb = 0.f;
        for (long long rr = r0; rr < r0 + GATE_BWD_ROWS && rr < rows; ++rr) {
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

// the states saved every CK tokens: [B][HV][V / VB][ceil(T / CK)][K][VB] floats
size_t backward_ckpt_floats(int B, int T, int HV, int K, int V) {
    const size_t nck = ((size_t)T + BWD_CK - 1) / BWD_CK;
    return (size_t)B * HV * nck * K * V;
}

template <typename Elt, int K, int V>
cudaError_t launch_bwd(const BackwardArgs& a) {
    using Sh = BwdShape<K, V>;
    // workspace: the saved states, the decays [B][T][HV][K], the residuals [B][T][HV][V]
    float* ckpt = static_cast<float*>(a.workspace);
    float* decay = ckpt + backward_ckpt_floats(a.B, a.T, a.HV, K, V);
    float* rres = decay + (size_t)a.B * a.T * a.HV * K;
    const long long n = (long long)a.B * a.T * a.HV * K;
    const unsigned dgrid = (unsigned)std::min<long long>((n + 255) / 256, 148ll * 16);
    decay_kernel<Elt><<<dgrid, 256, 0, a.stream>>>(static_cast<const Elt*>(a.g), a.A_log, a.dt_bias, n, a.HV, K,
                                                   a.gate_mode, a.lower_bound, decay);
    auto kern = recurrent_bwd_kernel<Elt, K, V>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((long long)a.B * a.HV * (Sh::NCB / Sh::NWB)), Sh::NT, Sh::smem_bytes, a.stream>>>(
        static_cast<const Elt*>(a.q), static_cast<const Elt*>(a.k), static_cast<const Elt*>(a.v), decay,
        static_cast<const Elt*>(a.beta), a.S0, static_cast<const Elt*>(a.dO), a.dS_T, a.T, a.H, a.HV, a.scale, a.dq,
        a.dk, a.dv, a.dg, a.dbeta, a.dS0, ckpt, rres);
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
    return (backward_ckpt_floats(B, T, HV, K, V) + (size_t)B * T * HV * (K + V)) * sizeof(float);
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
    const dim3 grid((unsigned)((rows + GATE_BWD_ROWS - 1) / GATE_BWD_ROWS), (unsigned)a.HV);
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
