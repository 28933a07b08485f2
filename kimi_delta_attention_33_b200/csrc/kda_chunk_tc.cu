// kda_chunk_tc.cu -- chunked prefill on the 5th-generation tensor cores (tcgen05, TMEM).
//
// DeltaNet-family digest, sections "Chunkwise KDA" and "Chunkwise Triton pipeline", in the
// key-major layout (S in R^{K x V}).  For a chunk of C = 64 tokens entering with state S_c:
//   Gam_i  = sum_{m<=i} g_m                       in-chunk cumulative log decay (fused with the gate)
//   A_ij   = s q_i . (k_j e^{Gam_i - Gam_j})        j <= i  (decayed Q K^T, read matrix)
//   R_ij   = beta_i k_i . (k_j e^{Gam_i - Gam_j})   j <  i  (decayed K K^T, coupling)
//   T      = (I + R)^{-1}                          unit lower triangular (WY / UT transform)
//   E      = T beta (V - Ktil S_c),  Ktil_i = k_i e^{Gam_i}          resolved delta errors
//   O      = Qtil S_c + A E,         Qtil_i = s q_i e^{Gam_i}         chunk outputs
//   S_c+1  = diag(e^{Gam_end}) S_c + Kend^T E,  Kend_j = k_j e^{Gam_end - Gam_j}
// Every product is a tcgen05.mma (kind::tf32, fp32 accumulation in TMEM); bf16 operands are
// not accurate enough for the stated tolerance once the output itself is rounded to bf16.
//
// Decay factors.  Products of the form x_i . (y_j e^{Gam_i - Gam_j}) are factorised around a
// per-channel reference rho = Gam_m (m the middle token of the chunk):
//   Qhat_i = s q_i e^{Gam_i - rho},  Khat_i = k_i e^{Gam_i - rho},  Kchk_j = k_j e^{rho - Gam_j},
// so [Qhat; Khat] Kchk^T gives A and R in one M = 128 MMA.  That is exact as long as no factor
// overflows, which holds when max(Gam_0 - rho, rho - Gam_end) <= 40 on every channel (all factors
// <= e^40, all products, masked ones included, <= 128 e^80 < FLT_MAX).  A chunk whose span is wider
// (strong decay: the safe gate at its floor every token, or a steep standard gate) takes the exact
// path instead: A and R from per-(i, j, d) exponentials on the CUDA cores, rho = 0.
// The same factors serve the state products: with S' = diag(e^rho) S_c,
//   Qtil S_c = Qhat S',   Ktil S_c = Khat S',   and  Kend = Kchk diag(e^{Gam_end - sig}).
//
// Per chunk (one CTA = one (b, hv) pair and one VT-wide slice of the value columns; value
// columns are independent, the pages' causal solve runs per value channel):
//   M1  D1[128 x 64]  = [Qhat; Khat] Kchk^T              -> A (rows 0-63), R (rows 64-127)
//   solve T = (I + R)^{-1} on the CUDA cores (16 x 16 blocks), Tb = T diag(beta)
//   M2  D2[64 x VT]   = Tb V                             -> U
//   M3  D3[128 x VT]  = [Qhat; Khat] S'^T                -> Qtil S_c (rows 0-63), P = Ktil S_c (rows 64-127)
//   M4  D2           += Tb (-P)                          -> E = U - Tb P
//   M5  D3           += [A; *] E                         -> O (rows 0-63)
//   M6  D4           += Kchk^T E,  D4 holding e^sig S_c  -> S_c+1 up to a per-row factor
// D4 keeps the fp32 state in TMEM across chunks; its pending per-row factor e^{Gam_end - sig} is
// applied when the next chunk reads it.  A partial last chunk is zero-padded (zero q, k, g, beta,
// v rows change nothing).
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tc_ptx.cuh"

namespace kda {
using namespace tc;
using bf16 = __nv_bfloat16;

namespace {

constexpr int TC_THREADS = 256;
constexpr int KD = 128;  // key dimension handled by this kernel
constexpr int CH = 64;   // chunk length handled by this kernel
constexpr float SPAN_LIMIT = 40.0f;
constexpr uint32_t WAIT_POLLS = 1u << 26;

template <int VT>
struct TcLayout {
    // shared memory regions (bytes)
    static constexpr uint32_t X1 = 0;                    // [128][128] [Qhat; Khat]            A of M1, M3
    static constexpr uint32_t X2 = X1 + 128 * KD * 4;   // [64][128] Kchk (B of M1); then [128][64] Kchk^T (A of M6)
    static constexpr uint32_t AT = X2 + CH * KD * 4;    // [128][64] rows 0-63 masked A, rows 64-127 T -> Tb
    static constexpr uint32_t VE = AT + 128 * CH * 4;   // [VT][64] V^T (B of M2); then E^T (B of M5, M6)
    static constexpr uint32_t SS = VE + VT * CH * 4;    // [VT][128] S'^T (B of M3)
    static constexpr uint32_t GM = SS + VT * KD * 4;    // [64][128] Gam; then R + solve scratch; then -P^T (B of M4)
    static constexpr uint32_t VEC = GM + CH * KD * 4;   // per-channel vectors
    static constexpr uint32_t RHO = VEC, SIG = VEC + 512, FNEXT = VEC + 1024, FPEND = VEC + 1536;
    static constexpr uint32_t BETA = VEC + 2048;        // [64]
    static constexpr uint32_t MBAR = BETA + 256;        // 8 B
    static constexpr uint32_t TBASE = MBAR + 8;         // 4 B
    static constexpr uint32_t FLAG = TBASE + 4;         // 4 B
    static constexpr uint32_t BYTES = FLAG + 4;
    static constexpr uint32_t Y_SCRATCH = GM + 64 * 64 * 4;  // 3 x 16 x 16 floats after R
    // TMEM columns
    static constexpr int D4 = 0;                       // state, M = 128, N = VT
    static constexpr int D3 = VT;                      // D1 (M = 128, N = 64) then D3 (M = 128, N = VT)
    static constexpr int D2 = VT + 64;                 // M = 64, N = VT
    static constexpr uint32_t TMEM_COLS = (VT + 64 + VT <= 128) ? 128u : 256u;
    static_assert(BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ int gidx(int i, int d) { return i * KD + ((((d >> 2) ^ (i & 7)) << 2) | (d & 3)); }
__device__ __forceinline__ int ridx(int i, int j) { return i * 64 + (j ^ (i & 31)); }

__device__ __forceinline__ void cta_sync_tc() {
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
}

}  // namespace

template <int VT>
__global__ void __launch_bounds__(TC_THREADS, 1)
chunk_tc_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const bf16* __restrict__ g, const bf16* __restrict__ beta, const float* __restrict__ A_log,
                const float* __restrict__ dt_bias, const float* __restrict__ S0, int T, int H, int HV, int V,
                int gate_mode, float lower_bound, float scale, bf16* __restrict__ o, float* __restrict__ S_T,
                unsigned int* __restrict__ status) {
    using L = TcLayout<VT>;
    constexpr int HALF = VT / 2;
    extern __shared__ __align__(1024) unsigned char smem[];
    float* sRho = reinterpret_cast<float*>(smem + L::RHO);
    float* sSig = reinterpret_cast<float*>(smem + L::SIG);
    float* sFnext = reinterpret_cast<float*>(smem + L::FNEXT);
    float* sFpend = reinterpret_cast<float*>(smem + L::FPEND);
    float* sBeta = reinterpret_cast<float*>(smem + L::BETA);
    float* sGam = reinterpret_cast<float*>(smem + L::GM);
    float* sR = reinterpret_cast<float*>(smem + L::GM);
    float* sY = reinterpret_cast<float*>(smem + L::Y_SCRATCH);
    float* sT = reinterpret_cast<float*>(smem + L::AT);  // addressed with cm_off(64 + i, j, 64) / 4
    uint32_t* sFlag = reinterpret_cast<uint32_t*>(smem + L::FLAG);
    const uint32_t s_base = smem_u32(smem);
    const uint32_t mbar = s_base + L::MBAR;

    const int pair = blockIdx.x;
    const int b = pair / HV, hv = pair - b * HV;
    const int h = hv / (HV / H);
    const int v0 = blockIdx.y * VT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wh = warp >> 2;  // TMEM lane quarter, column half
    const float rate = (gate_mode != KDA_GATE_NONE) ? expf(A_log[hv]) : 0.0f;
    const size_t qk_row = (size_t)H * KD;     // elements between consecutive tokens of q / k
    const size_t v_row = (size_t)HV * V, g_row = (size_t)HV * KD;

    // ---- prologue: barrier, TMEM, initial state into D4 -------------------------------------
    if (tid == 0) mbar_init(mbar, 1);
    if (warp == 0) tmem_alloc(s_base + L::TBASE, L::TMEM_COLS);
    if (tid < KD) sFpend[tid] = 1.0f;
    if (tid == 0) *sFlag = 0u;
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::TBASE);
    {
        const int d = 32 * wq + lane;
        TmemRow<HALF> row;
#pragma unroll
        for (int c = 0; c < HALF; c += 4) {
            float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (S0) s4 = *reinterpret_cast<const float4*>(S0 + ((size_t)pair * KD + d) * V + v0 + wh * HALF + c);
            row.r[c] = __float_as_uint(s4.x); row.r[c + 1] = __float_as_uint(s4.y);
            row.r[c + 2] = __float_as_uint(s4.z); row.r[c + 3] = __float_as_uint(s4.w);
        }
        row.store(taddr(tmem, 32 * wq, L::D4 + wh * HALF));
        tmem_wait_st();
    }
    uint32_t phase = 0;
    bool aborted = false;

    for (int t0 = 0; t0 < T && !aborted; t0 += CH) {
        const int n = min(CH, T - t0);
        const int m_ref = (n - 1) >> 1;
        const size_t tok0 = (size_t)b * T + t0;

        // ---- P1: issue every global load of this chunk before any arithmetic -------------------
        uint2 qr[8], kr[8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int u = tid + TC_THREADS * it;
            const int i = ((u >> 8) << 3) + (u & 7), d4 = (u >> 3) & 31;
            qr[it] = make_uint2(0u, 0u);
            kr[it] = make_uint2(0u, 0u);
            if (i < n) {
                qr[it] = __ldg(reinterpret_cast<const uint2*>(q + (tok0 + i) * qk_row + (size_t)h * KD + 4 * d4));
                kr[it] = __ldg(reinterpret_cast<const uint2*>(k + (tok0 + i) * qk_row + (size_t)h * KD + 4 * d4));
            }
        }
        constexpr int VVEC = VT / 32;  // 16-byte vectors of the value tile per thread
        uint4 vr[VVEC];
#pragma unroll
        for (int x = 0; x < VVEC; ++x) {
            const int e = tid + TC_THREADS * x;
            const int j = e / (VT / 8), c8 = e % (VT / 8);
            vr[x] = make_uint4(0u, 0u, 0u, 0u);
            if (j < n) vr[x] = __ldg(reinterpret_cast<const uint4*>(v + (tok0 + j) * v_row + (size_t)hv * V + v0 + 8 * c8));
        }
        const int gd = tid & (KD - 1), gh = tid >> 7;  // gate channel, token half
        float gv[32];
        {
            const bf16* gp = g + (size_t)hv * KD + gd;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const int i = 32 * gh + r;
                gv[r] = (i < n) ? to_f32(gp[(tok0 + i) * g_row]) : 0.f;
            }
        }
        const float bload = (tid < n) ? to_f32(beta[(tok0 + tid) * HV + hv]) : 0.f;  // tid < n <= 64

        // ---- P2: gate + in-chunk inclusive cumulative log decay (two threads per channel) -------
        {
            const float bias = (dt_bias != nullptr && gate_mode != KDA_GATE_NONE) ? dt_bias[hv * KD + gd] : 0.0f;
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const float x = (32 * gh + r < n) ? gate_value(gv[r], bias, rate, gate_mode, lower_bound) : 0.f;
                acc += x;
                gv[r] = acc;
            }
            if (gh == 0) sFnext[gd] = acc;  // scratch: first-half totals
        }
        // value tile as V^T [VT][64] (B operand of M2) and beta
#pragma unroll
        for (int x = 0; x < VVEC; ++x) {
            const int e = tid + TC_THREADS * x;
            const int j = e / (VT / 8), c8 = e % (VT / 8);
            const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&vr[x]);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f2 = __bfloat1622float2(hp[t]);
                *reinterpret_cast<uint32_t*>(smem + L::VE + cm_off(8 * c8 + 2 * t, j, CH)) = to_tf32(f2.x);
                *reinterpret_cast<uint32_t*>(smem + L::VE + cm_off(8 * c8 + 2 * t + 1, j, CH)) = to_tf32(f2.y);
            }
        }
        if (tid < CH) sBeta[tid] = bload;
        __syncthreads();
        {
            const float off = gh ? sFnext[gd] : 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) sGam[gidx(32 * gh + r, gd)] = gv[r] + off;
        }
        __syncthreads();
        if (tid < KD) {
            const int d = tid;
            const float g0 = sGam[gidx(0, d)], gm = sGam[gidx(m_ref, d)], gend = sGam[gidx(n - 1, d)];
            if (!(fmaxf(g0 - gm, gm - gend) <= SPAN_LIMIT)) atomicOr(sFlag, 1u);
            sRho[d] = gm;
            sSig[d] = gend;
        }
        __syncthreads();
        const bool slow = (*reinterpret_cast<volatile uint32_t*>(sFlag)) != 0;
        if (tid < KD) {
            const int d = tid;
            if (slow) sRho[d] = 0.f;  // sig stays Gam_end: Kchk becomes Kend
            else sSig[d] = sRho[d];
            sFnext[d] = __expf(sGam[gidx(CH - 1, d)] - sSig[d]);  // pending row factor of D4 after this chunk
        }
        __syncthreads();

        // ---- P3: [Qhat; Khat] -> X1, Kchk -> AT (B of M1), Kchk^T -> X2 (A of M6);
        //          state: S' = e^rho S_c -> SS (B of M3), D4 <- e^sig S_c ---------------------------
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int u = tid + TC_THREADS * it;
            const int i = ((u >> 8) << 3) + (u & 7), d4 = (u >> 3) & 31;
            const float4 g4 = *reinterpret_cast<const float4*>(sGam + gidx(i, 4 * d4));
            const float4 r4 = *reinterpret_cast<const float4*>(sRho + 4 * d4);
            const float4 s4 = *reinterpret_cast<const float4*>(sSig + 4 * d4);
            const float2 qa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr[it].x));
            const float2 qb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr[it].y));
            const float2 ka = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr[it].x));
            const float2 kb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr[it].y));
            const float e1[4] = {__expf(g4.x - r4.x), __expf(g4.y - r4.y), __expf(g4.z - r4.z), __expf(g4.w - r4.w)};
            const float e2[4] = {__expf(s4.x - g4.x), __expf(s4.y - g4.y), __expf(s4.z - g4.z), __expf(s4.w - g4.w)};
            const float qv[4] = {qa.x, qa.y, qb.x, qb.y}, kv[4] = {ka.x, ka.y, kb.x, kb.y};
            uint4 wq4, wk4, wc4;
            wq4.x = to_tf32(scale * qv[0] * e1[0]); wq4.y = to_tf32(scale * qv[1] * e1[1]);
            wq4.z = to_tf32(scale * qv[2] * e1[2]); wq4.w = to_tf32(scale * qv[3] * e1[3]);
            wk4.x = to_tf32(kv[0] * e1[0]); wk4.y = to_tf32(kv[1] * e1[1]);
            wk4.z = to_tf32(kv[2] * e1[2]); wk4.w = to_tf32(kv[3] * e1[3]);
            wc4.x = to_tf32(kv[0] * e2[0]); wc4.y = to_tf32(kv[1] * e2[1]);
            wc4.z = to_tf32(kv[2] * e2[2]); wc4.w = to_tf32(kv[3] * e2[3]);
            *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(i, 4 * d4, KD)) = wq4;
            *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(64 + i, 4 * d4, KD)) = wk4;
            *reinterpret_cast<uint4*>(smem + L::AT + cm_off(i, 4 * d4, KD)) = wc4;
            *reinterpret_cast<uint32_t*>(smem + L::X2 + cm_off(4 * d4 + 0, i, CH)) = wc4.x;
            *reinterpret_cast<uint32_t*>(smem + L::X2 + cm_off(4 * d4 + 1, i, CH)) = wc4.y;
            *reinterpret_cast<uint32_t*>(smem + L::X2 + cm_off(4 * d4 + 2, i, CH)) = wc4.z;
            *reinterpret_cast<uint32_t*>(smem + L::X2 + cm_off(4 * d4 + 3, i, CH)) = wc4.w;
        }
        {
            const int d = 32 * wq + lane;
            const float f = sFpend[d], eR = __expf(sRho[d]), eS = __expf(sSig[d]);
            TmemRow<HALF> row;
            row.load(taddr(tmem, 32 * wq, L::D4 + wh * HALF));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HALF; ++c) {
                const float sv = f * __uint_as_float(row.r[c]);
                *reinterpret_cast<uint32_t*>(smem + L::SS + cm_off(wh * HALF + c, d, KD)) = to_tf32(eR * sv);
                row.r[c] = __float_as_uint(eS * sv);
            }
            row.store(taddr(tmem, 32 * wq, L::D4 + wh * HALF));
            tmem_wait_st();
        }
        fence_proxy_async();
        cta_sync_tc();

        // ---- P4/P5: A (masked) -> AT rows 0-63, R -> GM --------------------------------------
        if (!slow) {
            if (tid == 0) {
                gemm_tf32(tmem + L::D3, s_base + L::X1, KD / 4 * 128, s_base + L::AT, KD / 4 * 128,
                          idesc_tf32(128, 64), KD / 8, false);
                mma_commit(mbar);
            }
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
            uint32_t raw[32];
            tmem_ld32(taddr(tmem, 32 * wq, L::D3 + 32 * wh), raw);
            tmem_wait_ld();
            const int i = 32 * (wq & 1) + lane;
            if (wq < 2) {
#pragma unroll
                for (int jj = 0; jj < 32; jj += 4) {
                    const int j = 32 * wh + jj;
                    uint4 w4;
                    w4.x = to_tf32(j + 0 <= i ? __uint_as_float(raw[jj + 0]) : 0.f);
                    w4.y = to_tf32(j + 1 <= i ? __uint_as_float(raw[jj + 1]) : 0.f);
                    w4.z = to_tf32(j + 2 <= i ? __uint_as_float(raw[jj + 2]) : 0.f);
                    w4.w = to_tf32(j + 3 <= i ? __uint_as_float(raw[jj + 3]) : 0.f);
                    *reinterpret_cast<uint4*>(smem + L::AT + cm_off(i, j, CH)) = w4;
                }
            } else {
                const float bi = sBeta[i];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = 32 * wh + jj;
                    sR[ridx(i, j)] = (j < i) ? bi * __uint_as_float(raw[jj]) : 0.f;
                }
            }
        } else {
            // exact decay factors: 4096 (i, j) cells, 16 per thread; Gam is still in GM
            float av[16], rr[16];
#pragma unroll 1
            for (int x = 0; x < 16; ++x) {
                const int p = tid + TC_THREADS * x;
                const int i = p >> 6, j = p & 63;
                float a = 0.f, r = 0.f;
                if (j <= i && i < n) {
                    const bf16* qi = q + (tok0 + i) * qk_row + (size_t)h * KD;
                    const bf16* ki = k + (tok0 + i) * qk_row + (size_t)h * KD;
                    const bf16* kj = k + (tok0 + j) * qk_row + (size_t)h * KD;
                    for (int d = 0; d < KD; ++d) {
                        const float e = __expf(sGam[gidx(i, d)] - sGam[gidx(j, d)]);
                        const float kd = to_f32(kj[d]) * e;
                        a += to_f32(qi[d]) * kd;
                        r += to_f32(ki[d]) * kd;
                    }
                }
                av[x] = (j <= i) ? scale * a : 0.f;
                rr[x] = (j < i) ? sBeta[i] * r : 0.f;
            }
            __syncthreads();  // Gam fully read: GM becomes R
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int p = tid + TC_THREADS * x;
                const int i = p >> 6, j = p & 63;
                *reinterpret_cast<uint32_t*>(smem + L::AT + cm_off(i, j, CH)) = to_tf32(av[x]);
                sR[ridx(i, j)] = rr[x];
            }
        }
        __syncthreads();

        // ---- P6: T = (I + R)^{-1} by 16 x 16 blocks, then Tb = T diag(beta) -----------------
        auto Tref = [&](int i, int j) -> float& {
            return *reinterpret_cast<float*>(smem + L::AT + cm_off(64 + i, j, CH));
        };
        if (tid < 64) {
            const int blk = tid >> 4, c = tid & 15, base = 16 * blk;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) acc += (m >= c) ? sR[ridx(base + r, base + m)] * t[m] : 0.f;
                t[r] = (r < c) ? 0.f : ((r == c) ? 1.f : -acc);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tref(base + r, base + c) = t[r];
        }
        __syncthreads();
        for (int lvl = 1; lvl < 4; ++lvl) {
            const int nb = 4 - lvl;
            const int r = tid >> 4, c = tid & 15;
            for (int x = 0; x < nb; ++x) {
                const int I = lvl + x, J = x;
                float acc = 0.f;
                for (int Kb = J; Kb < I; ++Kb)
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc += sR[ridx(16 * I + r, 16 * Kb + m)] * Tref(16 * Kb + m, 16 * J + c);
                sY[x * 256 + r * 16 + c] = acc;
            }
            __syncthreads();
            for (int x = 0; x < nb; ++x) {
                const int I = lvl + x, J = x;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc += Tref(16 * I + r, 16 * I + m) * sY[x * 256 + m * 16 + c];
                Tref(16 * I + r, 16 * J + c) = -acc;
            }
            __syncthreads();
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            const int p = tid + TC_THREADS * x;
            const int i = p >> 6, j = p & 63;
            const float tv = (j <= i) ? Tref(i, j) * sBeta[j] : 0.f;
            *reinterpret_cast<uint32_t*>(&Tref(i, j)) = to_tf32(tv);
        }
        fence_proxy_async();
        cta_sync_tc();

        // ---- M2 (U = Tb V) and M3 ([Qhat; Khat] S'^T) ---------------------------------------
        if (tid == 0) {
            gemm_tf32(tmem + L::D2, s_base + L::AT + 16384, CH / 4 * 128, s_base + L::VE, CH / 4 * 128,
                      idesc_tf32(64, VT), CH / 8, false);
            gemm_tf32(tmem + L::D3, s_base + L::X1, KD / 4 * 128, s_base + L::SS, KD / 4 * 128, idesc_tf32(128, VT),
                      KD / 8, false);
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }

        // ---- P8: -P^T into GM (B of M4) ------------------------------------------------------
        if (wq >= 2) {
            const int j = 32 * (wq & 1) + lane;
            TmemRow<HALF> row;
            row.load(taddr(tmem, 32 * wq, L::D3 + wh * HALF));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HALF; ++c)
                *reinterpret_cast<uint32_t*>(smem + L::GM + cm_off(wh * HALF + c, j, CH)) =
                    to_tf32(-__uint_as_float(row.r[c]));
        }
        fence_proxy_async();
        cta_sync_tc();

        // ---- M4: E = U - Tb P -----------------------------------------------------------------
        if (tid == 0) {
            gemm_tf32(tmem + L::D2, s_base + L::AT + 16384, CH / 4 * 128, s_base + L::GM, CH / 4 * 128,
                      idesc_tf32(64, VT), CH / 8, true);
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }

        // ---- P10: E^T into VE (B of M5, M6); rows live in lanes 32 q + t, t < 16 ------------
        {
            TmemRow<HALF> row;
            row.load(taddr(tmem, 32 * wq, L::D2 + wh * HALF));
            tmem_wait_ld();
            if (lane < 16) {
                const int i = 16 * wq + lane;
#pragma unroll
                for (int c = 0; c < HALF; ++c)
                    *reinterpret_cast<uint32_t*>(smem + L::VE + cm_off(wh * HALF + c, i, CH)) =
                        to_tf32(__uint_as_float(row.r[c]));
            }
        }
        fence_proxy_async();
        cta_sync_tc();

        // ---- M5: O += A E ; M6: D4 += Kchk^T E --------------------------------------------------
        if (tid == 0) {
            gemm_tf32(tmem + L::D3, s_base + L::AT, CH / 4 * 128, s_base + L::VE, CH / 4 * 128, idesc_tf32(128, VT),
                      CH / 8, true);
            gemm_tf32(tmem + L::D4, s_base + L::X2, CH / 4 * 128, s_base + L::VE, CH / 4 * 128, idesc_tf32(128, VT),
                      CH / 8, true);
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }

        // ---- P12: outputs; carry the pending state factor -----------------------------------
        if (wq < 2) {
            const int i = 32 * wq + lane;
            TmemRow<HALF> row;
            row.load(taddr(tmem, 32 * wq, L::D3 + wh * HALF));
            tmem_wait_ld();
            if (i < n) {
                bf16* op = o + (tok0 + i) * v_row + (size_t)hv * V + v0 + wh * HALF;
#pragma unroll
                for (int c = 0; c < HALF; c += 4)
                    store4(op + c, make_float4(__uint_as_float(row.r[c]), __uint_as_float(row.r[c + 1]),
                                               __uint_as_float(row.r[c + 2]), __uint_as_float(row.r[c + 3])));
            }
        }
        if (tid < KD) sFpend[tid] = sFnext[tid];
        if (tid == 0) *sFlag = 0u;
        cta_sync_tc();
    }

    if (aborted) {
        if (tid == 0) atomicOr(status, STATUS_TIMEOUT);
        // give any MMA still in flight one more bounded chance to drain before TMEM is released
        mbar_wait(mbar, phase, WAIT_POLLS);
    } else if (S_T) {
        const int d = 32 * wq + lane;
        const float f = sFpend[d];
        TmemRow<HALF> row;
        row.load(taddr(tmem, 32 * wq, L::D4 + wh * HALF));
        tmem_wait_ld();
        float* sp = S_T + ((size_t)pair * KD + d) * V + v0 + wh * HALF;
#pragma unroll
        for (int c = 0; c < HALF; c += 4)
            *reinterpret_cast<float4*>(sp + c) =
                make_float4(f * __uint_as_float(row.r[c]), f * __uint_as_float(row.r[c + 1]),
                            f * __uint_as_float(row.r[c + 2]), f * __uint_as_float(row.r[c + 3]));
    }
    cta_sync_tc();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

// bf16 inputs only: with float32 inputs the stated tolerance (1e-4) is tighter than tf32 products
// allow, so those run on the CUDA-core kernel in full fp32.
bool chunk_tc_supported(const ChunkArgs& a) {
    return a.dtype == KDA_BF16 && a.K == KD && a.chunk == CH && (a.V == 64 || a.V == 128);
}

template <int VT>
static cudaError_t launch_tc(const ChunkArgs& a) {
    using L = TcLayout<VT>;
    auto kern = chunk_tc_kernel<VT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.HV, a.V / VT);
    kern<<<grid, TC_THREADS, L::BYTES, a.stream>>>(
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k), static_cast<const bf16*>(a.v),
        static_cast<const bf16*>(a.g), static_cast<const bf16*>(a.beta), a.A_log, a.dt_bias, a.S0, a.T, a.H, a.HV, a.V,
        a.gate_mode, a.lower_bound, a.scale, static_cast<bf16*>(a.o), a.S_T, a.status);
    return cudaGetLastError();
}

// Value-tile width: 64 when the (b, hv) pairs alone give about one wave of CTAs, else 32.
int chunk_tc_value_tile(int B, int HV, int V) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (V == 64) return (2 * B * HV >= sms) ? 64 : 32;
    return (2 * B * HV >= sms) ? 64 : 32;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a) {
    const int vt = chunk_tc_value_tile(a.B, a.HV, a.V);
    return vt == 64 ? launch_tc<64>(a) : launch_tc<32>(a);
}

}  // namespace kda
