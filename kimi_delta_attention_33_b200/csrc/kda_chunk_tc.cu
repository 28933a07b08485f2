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
// per-channel reference rho = Gam_31 (the middle row of a full chunk; for a chunk of at most 32
// tokens, its last row):
//   Qhat_i = s q_i e^{Gam_i - rho},  Khat_i = k_i e^{Gam_i - rho},  Kchk_j = k_j e^{sig - Gam_j},
// with sig = rho, so [Qhat; -Khat] Kchk^T gives A and -R/beta in one M = 128 MMA.  That is exact as
// long as no factor overflows, which holds when max(Gam_0 - rho, rho - Gam_end) <= 40 on every
// channel (all factors <= e^40, all products, masked ones included, <= 128 e^80 < FLT_MAX).  A chunk
// whose span is wider (strong decay) takes the exact path instead: A and R from per-(i, j, d)
// exponentials on the CUDA cores, rho = 0 and sig = Gam_end (Kchk is then Kend itself).
//
// State side, transposed so the state stays in TMEM and feeds the tensor core directly.
// One CTA owns one (b, hv) pair: TMEM D4[v][d] holds S_c^T diag(e^rho) (lane = value column v).
//   M1  D1[128 x 64] = [Qhat; -Khat] Kchk^T                  -> A (rows 0-63), -R/beta (rows 64-127)
//   T = (I + R)^{-1} on the CUDA cores (block doubling, 2 x 2 up to 64 x 64), Tb = T diag(beta)
//   M3  D3[v][i]    = D4 (A from TMEM) . [Qhat; -Khat]^T      -> (Qtil S_c)^T (i < 64), -(Ktil S_c)^T (i >= 64)
//   M2  D2[v][j]    = V^T Tb^T                                -> U^T
//   M4  D2         += D3[:, 64:] (A from TMEM) Tb^T           -> E^T = (U - Tb Ktil S_c)^T
//   M5  D3[:, :64] += D2 (A from TMEM) A^T                    -> O^T
//   M6  D4         += D2 (A from TMEM) Kchk                   -> (e^sig S_c + Kchk^T E)^T
// M3..M6 are issued back to back by one thread: the tensor core executes them in order, so each one
// reads the TMEM the previous one wrote without a round trip through the CUDA cores.  After M6,
// D4 = S_c+1^T diag(e^{sig - Gam_end}); that per-key factor is applied with the next chunk's e^rho.
// A partial last chunk is zero-padded (zero q, k, g, beta, v rows change nothing).
#include "kda_chunk64.cuh"
#include "kda_internal.h"

namespace kda {
using namespace tc;
using bf16 = __nv_bfloat16;

namespace {
using namespace c64;

constexpr int SP_THREADS = 512;  // 16 warps: TMEM lane quarter x column quarter
static_assert(SP_THREADS == INV_THREADS, "the triangular inverse assumes 512 threads");

struct TcLayout {
    // shared memory regions (bytes)
    static constexpr uint32_t X1 = 0;          // [128][128] [Qhat; -Khat]   A of M1, B of M3
    static constexpr uint32_t AT = 65536;      // g staging (bf16 [64][128]); Kchk [64][128] (B of M1);
                                               //   then A [64][64] (B of M5) and Tb [64][64] (B of M2, M4)
    static constexpr uint32_t X2 = 98304;      // [128][64] Kchk^T               B of M6
    static constexpr uint32_t VE = 131072;     // [128][64] V^T                  A of M2
    static constexpr uint32_t GM = 163840;     // [64][128] Gam (fp32); then R/T (pitch RP) + doubling scratch
    static constexpr uint32_t XS = GM + 64 * RP * 4;
    static constexpr uint32_t VEC = 196608;    // per-channel vectors
    static constexpr uint32_t RHO = VEC, SIG = VEC + 512, FNEXT = VEC + 1024, FPEND = VEC + 1536;
    static constexpr uint32_t ERHO = VEC + 2048, ESIG = VEC + 2560;
    static constexpr uint32_t BETA = VEC + 3072;  // [64]
    static constexpr uint32_t MBAR = BETA + 256;  // 8 B
    static constexpr uint32_t TBASE = MBAR + 8;   // 4 B
    static constexpr uint32_t SQQ = VEC + 3456;   // [64] sums of squares of the q rows (KDA_INPUT_L2NORM_QK)
    static constexpr uint32_t SQK = VEC + 3712;   // [64] sums of squares of the k rows
    static constexpr uint32_t VS = VEC + 4096;    // bf16 [64][128] staging of the next chunk's v tile
    static constexpr uint32_t BYTES = VS + 64 * VD * 2;
    static_assert(TBASE + 4 <= SQQ && SQK + 256 <= VS, "vector region");
    // TMEM columns (all accumulators M = 128: TMEM lane = row)
    static constexpr int D4 = 0;     // state^T [v][d], 128 columns
    static constexpr int D3 = 128;   // [v][i]: 0-63 outputs, 64-127 -P
    static constexpr int D2 = 256;   // D1 [i][j] for M1, then E^T [v][j]; 64 columns
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(BYTES <= 232448, "shared memory budget");
    static_assert(XS + 1024 * 4 <= VEC, "doubling scratch");
};

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(SP_THREADS, 1)
chunk_tc_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                const bf16* __restrict__ g, const bf16* __restrict__ beta, const float* __restrict__ A_log,
                const float* __restrict__ dt_bias, const float* __restrict__ S0, int T, int H, int HV,
                float lower_bound, float scale, unsigned int flags, bf16* __restrict__ o, float* __restrict__ S_T,
                unsigned int* __restrict__ status) {
    using L = TcLayout;
    constexpr int gate_mode = MODE;
    extern __shared__ __align__(1024) unsigned char smem[];
    float* sRho = reinterpret_cast<float*>(smem + L::RHO);
    float* sSig = reinterpret_cast<float*>(smem + L::SIG);
    float* sFnext = reinterpret_cast<float*>(smem + L::FNEXT);
    float* sFpend = reinterpret_cast<float*>(smem + L::FPEND);
    float* sERho = reinterpret_cast<float*>(smem + L::ERHO);
    float* sESig = reinterpret_cast<float*>(smem + L::ESIG);
    float* sBeta = reinterpret_cast<float*>(smem + L::BETA);
    float* sSqQ = reinterpret_cast<float*>(smem + L::SQQ);
    float* sSqK = reinterpret_cast<float*>(smem + L::SQK);
    const bool norm_qk = (flags & KDA_INPUT_L2NORM_QK) != 0;
    float* sGam = reinterpret_cast<float*>(smem + L::GM);
    float* sRT = reinterpret_cast<float*>(smem + L::GM);  // R, overwritten in place by T
    float* sX = reinterpret_cast<float*>(smem + L::XS);
    const bf16* sG = reinterpret_cast<const bf16*>(smem + L::GM);  // g tile staging (bf16 [64][128])
    const uint32_t s_base = smem_u32(smem);
    const uint32_t mbar = s_base + L::MBAR;

    const int pair = blockIdx.x;
    const int b = pair / HV, hv = pair - b * HV;
    const int h = hv / (HV / H);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int NT = SP_THREADS;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column quarter
    const int vrow = 32 * wq + lane;          // value column held by this thread's TMEM lane
    const float rate = (gate_mode != KDA_GATE_NONE) ? expf(A_log[hv]) : 0.0f;
    const size_t qk_row = (size_t)H * KD;     // elements between consecutive tokens of q / k
    const size_t v_row = (size_t)HV * VD, g_row = (size_t)HV * KD;

    // ---- prologue: barrier, TMEM, initial state (transposed) into D4 ------------------------
    if (tid == 0) mbar_init(mbar, 1);
    if (warp == 0) tmem_alloc(s_base + L::TBASE, L::TMEM_COLS);
    if (tid < KD) sFpend[tid] = 1.0f;
    if (tid < 64) sSqQ[tid] = sSqK[tid] = 0.0f;
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::TBASE);
    {
        TmemRow<32> row;
        const int d0 = 32 * wc;
#pragma unroll
        for (int c = 0; c < 32; ++c)
            row.r[c] = __float_as_uint(S0 ? S0[((size_t)pair * KD + d0 + c) * VD + vrow] : 0.f);
        row.store(taddr(tmem, 32 * wq, L::D4 + d0));
    }
    tmem_wait_st();
    uint32_t phase = 0;
    bool aborted = false;

    // Input staging and the gate, one chunk ahead.  While the tensor core runs chunk c's state chain
    // (which reads X1, AT, X2, VE and TMEM only), the CUDA cores load chunk c+1's q, k, v, beta into
    // registers, bring its g tile into GM by cp.async, and run its gate and in-chunk cumulative decay
    // into GM.  Rows past T are zero-filled.
    const uint32_t gm_addr = s_base + L::GM;
    uint4 qr[2], kr[2];
    float bload;
    const int vc = tid & (VD - 1), q0 = tid >> 7;  // value column, first token quad (quads q0 + 4 x)
    auto load_inputs = [&](int tc0) {
        const int nn = min(CH, T - tc0);
        const size_t tk0 = (size_t)b * T + tc0;
#pragma unroll
        for (int it = 0; it < 2; ++it) {  // g tile -> GM staging, v tile -> VS staging, bf16 [64][128]
            const int u = tid + NT * it;
            const int i = u >> 4, c = u & 15;
            const bool ok = i < nn;
            cp_async16(gm_addr + i * 256 + c * 16, ok ? g + (tk0 + i) * g_row + (size_t)hv * KD + 8 * c : g, ok ? 16u : 0u);
            cp_async16(s_base + L::VS + i * 256 + c * 16, ok ? v + (tk0 + i) * v_row + (size_t)hv * VD + 8 * c : v,
                       ok ? 16u : 0u);
        }
        cp_async_commit();
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int u = tid + NT * it;
            const int i = ((u >> 7) << 3) + (u & 7), d8 = (u >> 3) & 15;
            qr[it] = make_uint4(0u, 0u, 0u, 0u);
            kr[it] = qr[it];
            if (i < nn) {
                qr[it] = __ldg(reinterpret_cast<const uint4*>(q + (tk0 + i) * qk_row + (size_t)h * KD + 8 * d8));
                kr[it] = __ldg(reinterpret_cast<const uint4*>(k + (tk0 + i) * qk_row + (size_t)h * KD + 8 * d8));
            }
        }
        bload = (tid < nn) ? to_f32(beta[(tk0 + tid) * HV + hv]) : 0.f;  // tid < nn <= 64
        if (tid < nn && (flags & KDA_INPUT_BETA_LOGITS)) bload = beta_from_logit(bload);
    };
    // Gate + inclusive in-chunk cumulative log decay of the chunk at tc0 (four threads per key channel),
    // its beta, the fast/exact decision and the per-channel vectors.  Uses sFpend, the pending state
    // factor the chunk starts from.  Returns whether the chunk takes the exact path.
    auto stage_gate = [&](int tc0) -> bool {
        const int nn = min(CH, T - tc0);
        cp_async_wait_all();
        if (norm_qk) add_row_sumsq(qr, kr, sSqQ, sSqK, tid, lane);  // complete after the barriers below
        __syncthreads();
        if (tid < CH) sBeta[tid] = bload;
        const int gd = tid & (KD - 1), gq = tid >> 7;  // channel, quarter of the rows (16 each)
        float gv[16];
        {
            const float bias = (dt_bias != nullptr && gate_mode != KDA_GATE_NONE) ? dt_bias[hv * KD + gd] : 0.0f;
            const float acc =
                gate_rows16_regs<MODE>(sG + 16 * gq * KD + gd, KD, nn - 16 * gq, bias, rate, lower_bound, gv);
            // quarter totals 0-2 and Gam_0 to scratch (vectors that are rewritten below)
            float* part = gq == 0 ? sFnext : gq == 1 ? sRho : sSig;
            if (gq < 3) part[gd] = acc;
            if (gq == 0) sESig[gd] = gv[0];
        }
        __syncthreads();  // the g staging has been read: GM becomes Gam
        // Quarter 3 knows the channel's Gam_31 (the reference point) and Gam_end (rows past the chunk's
        // end add zero) from the totals; one barrier reduction makes the fast / exact decision.
        bool bad = false;
        float gmid = 0.f, gend = 0.f;
        {
            const float p0 = sFnext[gd], p1 = sRho[gd], p2 = sSig[gd], g0 = sESig[gd];
            const float s01 = p0 + p1, s012 = s01 + p2;
            const float off = gq == 0 ? 0.f : gq == 1 ? p0 : gq == 2 ? s01 : s012;
#pragma unroll
            for (int r = 0; r < 16; ++r) sGam[gidx(16 * gq + r, gd)] = gv[r] + off;
            gmid = s01;
            gend = s012 + gv[15];  // the value row 63 receives (quarter 3's own total is gv[15])
            bad = gq == 3 && !(fmaxf(g0 - gmid, gmid - gend) <= SPAN_LIMIT);
        }
        const bool slow_c = __syncthreads_or(bad) != 0;
        if (gq == 3) {
            float rho = gmid, sig = gend;
            if (slow_c) rho = 0.f;  // sig stays Gam_end: Kchk becomes Kend
            else sig = rho;
            sRho[gd] = rho;
            sSig[gd] = sig;
            sERho[gd] = sFpend[gd] * __expf(rho);  // D4 rescale: the pending factor and e^rho
            sESig[gd] = __expf(sig);
            sFnext[gd] = __expf(gend - sig);  // pending per-key factor of D4 after this chunk
        }
        __syncthreads();
        return slow_c;
    };
    load_inputs(0);
    bool slow = stage_gate(0);

    for (int t0 = 0; t0 < T && !aborted; t0 += CH) {
        const int n = min(CH, T - t0);
        const size_t tok0 = (size_t)b * T + t0;
        const bool has_next = t0 + CH < T;

        // ---- P2: V^T -> VE from the VS staging (VE is free: the previous chain is done) ----------
        {
            const unsigned short* sVs = reinterpret_cast<const unsigned short*>(smem + L::VS);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = 4 * (q0 + 4 * x);
                *reinterpret_cast<uint4*>(smem + L::VE + cm_off(vc, j, CH)) =
                    make_uint4(to_tf32(bf16_bits_to_f32(sVs[(j + 0) * VD + vc])),
                               to_tf32(bf16_bits_to_f32(sVs[(j + 1) * VD + vc])),
                               to_tf32(bf16_bits_to_f32(sVs[(j + 2) * VD + vc])),
                               to_tf32(bf16_bits_to_f32(sVs[(j + 3) * VD + vc])));
            }
        }

        // ---- P3: [Qhat; -Khat] -> X1, Kchk -> AT (B of M1), Kchk^T -> X2 (B of M6);
        //          D4 <- S_c^T diag(e^rho) (applies the previous chunk's pending factor too) ----------
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int u = tid + NT * it;
            const int i = ((u >> 7) << 3) + (u & 7), d8 = (u >> 3) & 15;
            float qf[8], kf[8], gf[8], rf[8], sf[8];
            bf16x8_to_f32(qr[it], qf);
            bf16x8_to_f32(kr[it], kf);
            if (norm_qk) scale_row8(qf, kf, sSqQ[i], sSqK[i]);
            *reinterpret_cast<float4*>(gf) = *reinterpret_cast<const float4*>(sGam + gidx(i, 8 * d8));
            *reinterpret_cast<float4*>(gf + 4) = *reinterpret_cast<const float4*>(sGam + gidx(i, 8 * d8 + 4));
            *reinterpret_cast<float4*>(rf) = *reinterpret_cast<const float4*>(sRho + 8 * d8);
            *reinterpret_cast<float4*>(rf + 4) = *reinterpret_cast<const float4*>(sRho + 8 * d8 + 4);
            *reinterpret_cast<float4*>(sf) = *reinterpret_cast<const float4*>(sSig + 8 * d8);
            *reinterpret_cast<float4*>(sf + 4) = *reinterpret_cast<const float4*>(sSig + 8 * d8 + 4);
            uint32_t wq_[8], wk_[8], wc_[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float e1 = __expf(gf[t] - rf[t]), e2 = __expf(sf[t] - gf[t]);
                wq_[t] = to_tf32(scale * qf[t] * e1);
                wk_[t] = to_tf32(-kf[t] * e1);
                wc_[t] = to_tf32(kf[t] * e2);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int d = 8 * d8 + 4 * hh;
                *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(i, d, KD)) =
                    make_uint4(wq_[4 * hh], wq_[4 * hh + 1], wq_[4 * hh + 2], wq_[4 * hh + 3]);
                *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(64 + i, d, KD)) =
                    make_uint4(wk_[4 * hh], wk_[4 * hh + 1], wk_[4 * hh + 2], wk_[4 * hh + 3]);
                *reinterpret_cast<uint4*>(smem + L::AT + cm_off(i, d, KD)) =
                    make_uint4(wc_[4 * hh], wc_[4 * hh + 1], wc_[4 * hh + 2], wc_[4 * hh + 3]);
            }
            // Kchk^T: lanes that share a bank (same i & 3) take different d of their group of 8
            const int rot = lane >> 2;
            rotate_groups8(wc_, rot);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                *reinterpret_cast<uint32_t*>(smem + L::X2 + cm_off(8 * d8 + ((t + rot) & 7), i, CH)) = wc_[t];
        }
        {
            const int d0 = 32 * wc;
            TmemRow<32> row;
            row.load(taddr(tmem, 32 * wq, L::D4 + d0));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
                row.r[c] = __float_as_uint(sERho[d0 + c] * __uint_as_float(row.r[c]));
            row.store(taddr(tmem, 32 * wq, L::D4 + d0));
        }
        tmem_wait_st();
        fence_proxy_async();
        cta_sync_tc();

        // ---- P4/P5: A (masked) -> AT rows 0-63, R -> GM (row pitch RP) ------------------------
        if (!slow) {
            if (tid == 0) {
                gemm_tf32(tmem + L::D2, s_base + L::X1, KD / 4 * 128, s_base + L::AT, KD / 4 * 128,
                          idesc_tf32(128, 64), KD / 8, false);
                mma_commit(mbar);
            }
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
            uint32_t raw[16];
            tmem_ld16(taddr(tmem, 32 * wq, L::D2 + 16 * wc), raw);
            tmem_wait_ld();
            const int i = 32 * (wq & 1) + lane;
            if (wq < 2) {
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int j = 16 * wc + jj;
                    uint4 w4;
                    w4.x = to_tf32(j + 0 <= i ? __uint_as_float(raw[jj + 0]) : 0.f);
                    w4.y = to_tf32(j + 1 <= i ? __uint_as_float(raw[jj + 1]) : 0.f);
                    w4.z = to_tf32(j + 2 <= i ? __uint_as_float(raw[jj + 2]) : 0.f);
                    w4.w = to_tf32(j + 3 <= i ? __uint_as_float(raw[jj + 3]) : 0.f);
                    *reinterpret_cast<uint4*>(smem + L::AT + cm_off(i, j, CH)) = w4;
                }
            } else {
                const float bi = -sBeta[i];  // rows 64-127 of D1 hold -Khat Kchk^T
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int j = 16 * wc + jj;
                    *reinterpret_cast<float4*>(sRT + i * RP + j) =
                        make_float4(j + 0 < i ? bi * __uint_as_float(raw[jj + 0]) : 0.f,
                                    j + 1 < i ? bi * __uint_as_float(raw[jj + 1]) : 0.f,
                                    j + 2 < i ? bi * __uint_as_float(raw[jj + 2]) : 0.f,
                                    j + 3 < i ? bi * __uint_as_float(raw[jj + 3]) : 0.f);
                }
            }
        } else {
            // exact decay factors: 4096 (i, j) cells, 8 per thread; Gam is still in GM
            float av[8], rr[8];
#pragma unroll 1
            for (int x = 0; x < 8; ++x) {
                const int p = tid + NT * x;
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
                if (norm_qk && j <= i && i < n) {
                    const float ikj = inv_l2norm(sSqK[j]);
                    a *= inv_l2norm(sSqQ[i]) * ikj;
                    r *= inv_l2norm(sSqK[i]) * ikj;
                }
                av[x] = (j <= i) ? scale * a : 0.f;
                rr[x] = (j < i) ? sBeta[i] * r : 0.f;
            }
            __syncthreads();  // Gam fully read: GM becomes R
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int p = tid + NT * x;
                const int i = p >> 6, j = p & 63;
                *reinterpret_cast<uint32_t*>(smem + L::AT + cm_off(i, j, CH)) = to_tf32(av[x]);
                sRT[i * RP + j] = rr[x];
            }
        }
        __syncthreads();

        // ---- P6: T = (I + R)^{-1}, in place over R, by six doubling steps (block sizes 2 .. 64) --
        tri_inverse_diag16(sRT, sX, tid);
        tri_inverse_step16(sRT, sX, tid);
        tri_inverse_step32(sRT, sX, tid);
        // Tb = T diag(beta) as tf32 into AT rows 64-127
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int u = tid + NT * x;
            const int i = ((u >> 7) << 3) + (u & 7), j4 = (u >> 3) & 15;
            uint32_t w[4];
            const float4 t4 = *reinterpret_cast<const float4*>(sRT + i * RP + 4 * j4);
            const float tr[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = 4 * j4 + t;
                const float tv = (j < i) ? tr[t] : (j == i ? 1.f : 0.f);
                w[t] = to_tf32(tv * sBeta[j]);
            }
            *reinterpret_cast<uint4*>(smem + L::AT + cm_off(64 + i, 4 * j4, CH)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (tid < 64) sSqQ[tid] = sSqK[tid] = 0.0f;  // read for the last time above; the next chunk's sums follow
        fence_proxy_async();
        cta_sync_tc();
        // ---- state chain: M3, M2, M4, M5, M6 back to back (fast path) --------------------------
        if (tid == 0) {
            gemm_tf32_ts(tmem + L::D3, tmem + L::D4, s_base + L::X1, KD / 4 * 128, idesc_tf32(128, 128), KD / 8, false);
            gemm_tf32(tmem + L::D2, s_base + L::VE, CH / 4 * 128, s_base + L::AT + 16384, CH / 4 * 128,
                      idesc_tf32(128, 64), CH / 8, false);
            gemm_tf32_ts(tmem + L::D2, tmem + L::D3 + 64, s_base + L::AT + 16384, CH / 4 * 128, idesc_tf32(128, 64),
                         CH / 8, true);
            gemm_tf32_ts(tmem + L::D3, tmem + L::D2, s_base + L::AT, CH / 4 * 128, idesc_tf32(128, 64), CH / 8, true);
            if (!slow)
                gemm_tf32_ts(tmem + L::D4, tmem + L::D2, s_base + L::X2, CH / 4 * 128, idesc_tf32(128, 128), CH / 8,
                             true);
            mma_commit(mbar);
        }
        // Next chunk's inputs: GM (R/T) and VS are no longer needed by this chunk.  VS must not be
        // overwritten before this chunk's V^T was built (it was, in P2, before several barriers).
        if (has_next) load_inputs(t0 + CH);
        // fast path: the next chunk's gate runs while the chain executes (touches GM and vectors only)
        bool slow_next = false;
        if (!slow) {
            if (tid < KD) sFpend[tid] = sFnext[tid];
            if (has_next) slow_next = stage_gate(t0 + CH);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }
        if (slow) {
            // exact path: M3 read S_c (rho = 0); M6 needs e^{Gam_end} S_c, i.e. e^sig per key column
            {
                const int d0 = 32 * wc;
                TmemRow<32> row;
                row.load(taddr(tmem, 32 * wq, L::D4 + d0));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) row.r[c] = __float_as_uint(sESig[d0 + c] * __uint_as_float(row.r[c]));
                row.store(taddr(tmem, 32 * wq, L::D4 + d0));
            }
            tmem_wait_st();
            cta_sync_tc();
            if (tid == 0) {
                gemm_tf32_ts(tmem + L::D4, tmem + L::D2, s_base + L::X2, CH / 4 * 128, idesc_tf32(128, 128), CH / 8,
                             true);
                mma_commit(mbar);
            }
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }

        // ---- outputs: O^T in D3 columns 0-63 (lane = value column) ----------------------------
        {
            TmemRow<16> row;
            row.load(taddr(tmem, 32 * wq, L::D3 + 16 * wc));
            tmem_wait_ld();
            bf16* op = o + tok0 * v_row + (size_t)hv * VD + vrow;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int i = 16 * wc + c;
                if (i < n) op[(size_t)i * v_row] = __float2bfloat16_rn(__uint_as_float(row.r[c]));
            }
        }
        if (slow) {
            cta_sync_tc();
            if (tid < KD) sFpend[tid] = sFnext[tid];
            if (has_next) slow_next = stage_gate(t0 + CH);
        }
        slow = slow_next;
        cta_sync_tc();
    }

    if (aborted) {
        if (tid == 0) atomicOr(status, STATUS_TIMEOUT);
        // give any MMA still in flight one more bounded chance to drain before TMEM is released
        mbar_wait(mbar, phase, WAIT_POLLS);
    } else if (S_T) {
        {
            const int d0 = 32 * wc;
            TmemRow<32> row;
            row.load(taddr(tmem, 32 * wq, L::D4 + d0));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
                S_T[((size_t)pair * KD + d0 + c) * VD + vrow] = sFpend[d0 + c] * __uint_as_float(row.r[c]);
        }
    }
    cta_sync_tc();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

namespace {
template <int MODE>
cudaError_t launch_tc(const ChunkArgs& a) {
    using L = TcLayout;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<MODE><<<a.B * a.HV, SP_THREADS, L::BYTES, a.stream>>>(
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k), static_cast<const bf16*>(a.v),
        static_cast<const bf16*>(a.g), static_cast<const bf16*>(a.beta), a.A_log, a.dt_bias, a.S0, a.T, a.H, a.HV,
        a.lower_bound, a.scale, a.flags, static_cast<bf16*>(a.o), a.S_T, a.status);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_chunk_tc(const ChunkArgs& a) {
    // one kernel per gate mode: the gate's 16-row loop is straight-line code in each
    return a.gate_mode == KDA_GATE_SAFE       ? launch_tc<KDA_GATE_SAFE>(a)
           : a.gate_mode == KDA_GATE_STANDARD ? launch_tc<KDA_GATE_STANDARD>(a)
                                              : launch_tc<KDA_GATE_NONE>(a);
}

}  // namespace kda
