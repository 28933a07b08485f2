// kda_chunk_split.cu -- two-pass chunked prefill on the tensor cores (bf16 inputs, K = V = 128,
// chunk 64) for shapes with few (sequence, head) pairs, where one CTA per pair leaves most SMs idle.
//
// DeltaNet-family digest, sections "Chunkwise KDA" and "Chunkwise Triton pipeline": everything of a
// chunk that does not involve the state entering it can be computed for all chunks at once; only
// the state update is sequential.  Notation as in the single-pass kernel (kda_chunk_tc.cu):
//   Gam_i  in-chunk cumulative log decay, rho / sig per-channel reference points,
//   Qhat_i = s q_i e^{Gam_i - rho},  Khat_i = k_i e^{Gam_i - rho},  Kchk_j = k_j e^{sig - Gam_j},
//   A = masked Qhat Kchk^T,  R = masked beta Khat Kchk^T,  T = (I + R)^{-1},  Tb = T diag(beta).
// The factorised operands keep the in-chunk products within range; the state side needs the plain
// ones, Wtil = W diag(e^rho) = Tb Ktil (Ktil_j = k_j e^{Gam_j}), Qtil = Qhat diag(e^rho) = s q e^{Gam}
// and Kend = diag(f) Kchk^T = (k_j e^{Gam_end - Gam_j})^T with f = e^{Gam_end - sig}.  With S_c the
// state entering the chunk the results are
//   E      = U - Wtil S_c        where U = Tb V                   (resolved delta errors)
//   O      = Qtil S_c + A E                                       (chunk outputs)
//   S_c+1  = diag(e^{Gam_end}) S_c + Kend E.
//
// Pass 1 (chunk_prep_kernel, persistent, one chunk per CTA iteration, all chunks in parallel):
// gate, Gam, the operands, M1 = [-Khat; Qhat] Kchk^T -> R and A, the triangular inverse, and
// M7 = [Tb; Tb] [Khat^T; V^T]^T -> W and U, written to a per-chunk record in the workspace:
//   WQ  [Wtil; Qtil]  128 x 128 tf32 in the K-major tiling of kda_tc_ptx.cuh (the A operand of M8)
//   KA  [Kend; A]     192 x 64 tf32, same tiling (A operands of M9 and M10)
//   UT  U^T, fp32 rows of 64 (one per value column)
//   VEC e^{Gam_end} (fp32, 128)
// Pass 2 (chunk_state_kernel, one CTA per (pair, block of VB value columns), chunks in order):
// the state slice S_c[:, block] lives in registers (thread d owns key row d, exact fp32);
// per chunk, with tf32(S_c)^T staged in shared memory as a B operand:
//   M8   D1 = [Wtil; Qtil] S_c           -> Wtil S_c (rows 0-63), Qtil S_c (rows 64-127)
//   E    = U - Wtil S_c  on the CUDA cores, staged as a tf32 B operand
//   M10  D2 = Kend E                      -> S_c+1 = e^{Gam_end} S_c + D2, in registers
//   M9   D1[64:] += A E                   -> O  (issued after M10 with its own commit: off the
//                                             chunk-to-chunk path)
// Chunk records stream in by bulk asynchronous copies (mbarrier completion), double-buffered
// where shared memory allows.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_chunk64.cuh"
#include "kda_internal.h"

namespace kda {
using bf16 = __nv_bfloat16;

namespace {
using namespace c64;

// Per-chunk record in the workspace (bytes).
struct Rec {
    static constexpr uint32_t WQ = 0;        // [128][128] tf32 tiles
    static constexpr uint32_t KA = 65536;    // [192][64] tf32 tiles
    static constexpr uint32_t KA_BYTES = 49152;
    static constexpr uint32_t UT = 114688;   // [128][64] fp32 rows
    static constexpr uint32_t VEC = 147456;  // [128] fp32 e^{Gam_end}, then padding
    static constexpr uint32_t BYTES = 149504;
    static_assert(VEC + 512 <= BYTES && BYTES % 256 == 0, "record layout");
};

struct PrepLayout {
    static constexpr uint32_t X1 = 0;        // [128][128] [-Khat; Qhat] (A of M1); once M1 is done X1 stages
                                             //   the next chunk's input tiles, bf16 [64][128] each: g, v
                                             //   (plain rows), q, k (two 64-column halves each, rows of 128
                                             //   bytes with the 128-byte swizzle)
    static constexpr uint32_t CK = 65536;    // [64][128] Kchk (B of M1); then R / T (pitch RP) + doubling
                                             //   scratch; then U^T [128][64] fp32 (record UT)
    static constexpr uint32_t XS = CK + 64 * RP * 4;
    static constexpr uint32_t KA = 98304;    // [256][64]: Kend^T rows 0-127 (record KA, first part),
                                             //   Tb twice in rows 128-255 (A of M7)
    static constexpr uint32_t GM = 163840;   // Gam (fp32 [64][128]) -> Khat^T [128][64] (B rows 0-127 of M7)
    static constexpr uint32_t VT = 196608;   // V^T [128][64] (B rows 128-255 of M7)
    static constexpr uint32_t VEC = 229376;
    static constexpr uint32_t RHO = VEC, SIG = VEC + 512, BETA = VEC + 1024, ERHO = VEC + 1280, FEND = VEC + 1792;
    static constexpr uint32_t MBAR = VEC + 2304, MBAR_IN = MBAR + 8, TBASE = MBAR_IN + 8;
    static constexpr uint32_t SQQ = VEC + 2336, SQK = VEC + 2592;  // [64] row sums of squares of q, k
    static constexpr uint32_t QT = KA + 32768;    // record Qtil staging, in the Tb rows (free until the inverse)
    static constexpr uint32_t PART = KA + 32768;  // gate: per-channel quarter totals and Gam_0 (5 x [128] fp32),
                                                  //   in the Tb rows, which are free until the inverse
    static constexpr uint32_t STG_G = X1, STG_V = X1 + 16384, STG_Q = X1 + 32768, STG_K = X1 + 49152;
    static constexpr uint32_t BYTES = SQK + 256;
    static constexpr uint32_t TMEM_COLS = 256;  // D1 [128][64] for M1, then [128][256] for M7
    static_assert(XS + 1024 * 4 <= KA, "doubling scratch");
    static_assert(GM + 32768 == VT, "M7's B operand spans GM and VT");
    static_assert(BYTES <= 232448, "shared memory budget");
};

template <int VB>
struct StateLayout {
    static constexpr int NKA = VB <= 32 ? 2 : 1;              // KA / U buffers
    // With 128 value columns the E^T operand takes the place of the U^T rows it is computed from.
    static constexpr bool ALIAS_E = VB > 64;
    static constexpr uint32_t WQ = 0;                          // [128][128]
    static constexpr uint32_t KA0 = 65536;                     // per buffer: KA [192][64], U^T [VB][64], e^{Gam_end}
    static constexpr uint32_t UT_OFF = Rec::KA_BYTES, VEC_OFF = Rec::KA_BYTES + VB * 256;
    static constexpr uint32_t KA_STRIDE = VEC_OFF + 512;
    static constexpr uint32_t SOP = KA0 + NKA * KA_STRIDE;     // tf32 S^T [VB][128]    (B of M8)
    static constexpr uint32_t EOP = ALIAS_E ? KA0 + UT_OFF : SOP + VB * 128 * 4;  // tf32 E^T [VB][64] (B of M9, M10)
    static constexpr uint32_t MBAR = ALIAS_E ? SOP + VB * 128 * 4 : EOP + VB * 64 * 4;  // wq, mma, ka[0], ka[1], out
    static constexpr uint32_t TBASE = MBAR + 40;
    static constexpr uint32_t BYTES = TBASE + 16;
    static constexpr uint32_t TMEM_COLS = 2 * VB < 32 ? 32 : 2 * VB;
    static constexpr int D1 = 0, D2 = VB;
    static __device__ __forceinline__ uint32_t ka(int buf) { return KA0 + buf * KA_STRIDE; }
    static_assert(!ALIAS_E || VB * 64 * 4 <= VB * 256, "E^T fits in the U^T rows");
    static_assert(BYTES <= 232448, "shared memory budget");
};

// What one state-pass CTA computes over its chunks (see chunk_state_kernel).
enum : int { STATE_OUT = 0, STATE_CARRY = 1 };

constexpr int STATE_THREADS = 256;
constexpr int PREP_THREADS = 512;
static_assert(PREP_THREADS == INV_THREADS, "the triangular inverse assumes 512 threads");

struct Task {
    int pair, c, b, hv, h, nn;
    size_t tk0;  // token index (b * T + first token of the chunk)
};

__device__ __forceinline__ Task make_task(int task, int T, int H, int HV, int NC) {
    Task t;
    t.pair = task / NC;
    t.c = task - t.pair * NC;
    t.b = t.pair / HV;
    t.hv = t.pair - t.b * HV;
    t.h = t.hv / (HV / H);
    t.nn = min(CH, T - t.c * CH);
    t.tk0 = (size_t)t.b * T + (size_t)t.c * CH;
    return t;
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// Pass 1: chunk-local work for every chunk.
// ---------------------------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(PREP_THREADS, 1)
chunk_prep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                  const bf16* __restrict__ g, const bf16* __restrict__ beta, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, int T, int H, int HV, int NC, int ntasks,
                  float lower_bound, float scale, unsigned int flags, unsigned char* __restrict__ rec_base,
                  unsigned int* __restrict__ status, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_g) {
    using L = PrepLayout;
    constexpr int NT = PREP_THREADS;
    extern __shared__ __align__(1024) unsigned char smem[];
    float* sRho = reinterpret_cast<float*>(smem + L::RHO);
    float* sSig = reinterpret_cast<float*>(smem + L::SIG);
    float* sPart = reinterpret_cast<float*>(smem + L::PART);
    float* sBeta = reinterpret_cast<float*>(smem + L::BETA);
    float* sERho = reinterpret_cast<float*>(smem + L::ERHO);
    float* sFend = reinterpret_cast<float*>(smem + L::FEND);
    float* sSqQ = reinterpret_cast<float*>(smem + L::SQQ);
    float* sSqK = reinterpret_cast<float*>(smem + L::SQK);
    const bool norm_qk = (flags & KDA_INPUT_L2NORM_QK) != 0;
    float* sGam = reinterpret_cast<float*>(smem + L::GM);
    float* sRT = reinterpret_cast<float*>(smem + L::CK);  // R, overwritten in place by T
    float* sX = reinterpret_cast<float*>(smem + L::XS);
    const bf16* sG = reinterpret_cast<const bf16*>(smem + L::X1);  // staged g tile
    const uint32_t s_base = smem_u32(smem);
    const uint32_t mbar = s_base + L::MBAR, mbar_in = s_base + L::MBAR_IN;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column quarter
    const int rot = lane >> 2;                // store rotation (see rotate_groups8)
    const size_t qk_row = (size_t)H * KD;  // elements between consecutive tokens of q / k (exact path)

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_init(mbar_in, 1);
    }
    if (warp == 0) tmem_alloc(s_base + L::TBASE, L::TMEM_COLS);
    if (tid < 64) sSqQ[tid] = sSqK[tid] = 0.0f;
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::TBASE);
    uint32_t phase = 0, phase_in = 0;
    bool aborted = false, in_pending = false;

    // Inputs of one chunk: the q, k, g and v tiles into X1 by six tensor-map copies issued by thread 32
    // (rows past T read as zero), completing on mbar_in; beta, this head's A_log and this thread's
    // dt_bias entry into registers.  Thread 32 first lets the record stores it issued finish reading
    // X1.  q / k are read back in the operand pass as units u = tid + NT * it: row
    // i = 8 (u / 128) + u % 8, key group d8 = (u / 8) % 16.
    uint32_t beta_bits = 0;  // raw bf16 bits of beta for row tid (tid < 64), converted where used
    float alog_in = 0.f, bias_in = 0.f;
    auto load_inputs = [&](const Task& tk) {
        if (tid == 32) {
            bulk_wait_read();
            mbar_expect_tx(mbar_in, 4u * 16384u);
            const int t0 = tk.c * CH;
            tma_load_4d(s_base + L::STG_G, &tm_g, 0, tk.hv, t0, tk.b, mbar_in);
            tma_load_4d(s_base + L::STG_V, &tm_v, 0, tk.hv, t0, tk.b, mbar_in);
            tma_load_4d(s_base + L::STG_Q, &tm_q, 0, tk.h, t0, tk.b, mbar_in);
            tma_load_4d(s_base + L::STG_Q + 8192, &tm_q, 64, tk.h, t0, tk.b, mbar_in);
            tma_load_4d(s_base + L::STG_K, &tm_k, 0, tk.h, t0, tk.b, mbar_in);
            tma_load_4d(s_base + L::STG_K + 8192, &tm_k, 64, tk.h, t0, tk.b, mbar_in);
        }
        in_pending = true;
        beta_bits = (tid < tk.nn) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(beta) + (tk.tk0 + tid) * HV + tk.hv)
                                  : 0u;
        if (MODE != KDA_GATE_NONE) {
            alog_in = __ldg(A_log + tk.hv);
            bias_in = dt_bias != nullptr ? __ldg(dt_bias + tk.hv * KD + (tid & (KD - 1))) : 0.f;
        }
    };

    int task = blockIdx.x;
    if (task < ntasks) load_inputs(make_task(task, T, H, HV, NC));

    for (; task < ntasks && !aborted; task += gridDim.x) {
        const Task tk = make_task(task, T, H, HV, NC);
        unsigned char* rec = rec_base + (size_t)task * Rec::BYTES;
        const float rate = (MODE != KDA_GATE_NONE) ? expf(alog_in) : 0.0f;

        // ---- gate and inclusive in-chunk cumulative log decay (four threads per key channel) ----
        // Thread (gd, gq) keeps the running sums of rows 16 gq .. 16 gq + 15 of channel gd in registers;
        // the quarter totals give every thread its offset and the channel's Gam_31 (the reference
        // point rho) and Gam_end (rows past the chunk's end add zero), so the fast / exact decision is
        // one barrier reduction.  Gam, rho and sig are made visible by the barrier of the V^T step.
        bool slow;
        {
            const int nn = tk.nn;
            const bool ok_in = mbar_wait(mbar_in, phase_in, WAIT_POLLS);
            if (!__syncthreads_and(ok_in)) { aborted = true; break; }
            phase_in ^= 1u;
            in_pending = false;
            if (tid < CH) {
                const float bl = __uint_as_float(beta_bits << 16);
                sBeta[tid] = (tid < nn && (flags & KDA_INPUT_BETA_LOGITS)) ? beta_from_logit(bl) : bl;
            }
            const int gd = tid & (KD - 1), gq = tid >> 7;  // channel, quarter of the rows (16 each)
            float gv[16];
            const float acc = gate_rows16_regs<MODE>(sG + 16 * gq * KD + gd, KD, nn - 16 * gq, bias_in, rate,
                                                     lower_bound, gv);
            sPart[gq * KD + gd] = acc;
            if (gq == 0) sPart[4 * KD + gd] = gv[0];
            __syncthreads();
            const float p0 = sPart[gd], p1 = sPart[KD + gd], p2 = sPart[2 * KD + gd], p3 = sPart[3 * KD + gd];
            const float g0 = sPart[4 * KD + gd];
            const float s01 = p0 + p1, s012 = s01 + p2;
            const float off = gq == 0 ? 0.f : gq == 1 ? p0 : gq == 2 ? s01 : s012;
            const float gmid = s01, gend = s012 + p3;  // the values rows 31 and 63 receive below
#pragma unroll
            for (int r = 0; r < 16; ++r) sGam[gidx(16 * gq + r, gd)] = gv[r] + off;
            slow = __syncthreads_or(!(fmaxf(g0 - gmid, gmid - gend) <= SPAN_LIMIT)) != 0;
            if (gq == 0) {
                float rho = gmid, sig = gend;
                if (slow) rho = 0.f;  // sig stays Gam_end: Kchk becomes Kend
                else sig = rho;
                sRho[gd] = rho;
                sSig[gd] = sig;
                sERho[gd] = __expf(rho);
                sFend[gd] = __expf(gend - sig);
                reinterpret_cast<float*>(rec + Rec::VEC)[gd] = __expf(gend);
            }
        }

        // ---- V^T into VT from the staged v tile (value column vc, token quads q0 + 4 x) ---------------
        uint4 qr[2], kr[2];  // bf16 q / k of this thread's two operand units
        {
            const unsigned short* sVs = reinterpret_cast<const unsigned short*>(smem + L::X1 + 16384);
            const int vc = tid & (VD - 1), q0 = tid >> 7;
            uint32_t vv[8];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = 4 * (q0 + 4 * x);
                vv[2 * x] = (uint32_t)sVs[(j + 0) * VD + vc] | ((uint32_t)sVs[(j + 1) * VD + vc] << 16);
                vv[2 * x + 1] = (uint32_t)sVs[(j + 2) * VD + vc] | ((uint32_t)sVs[(j + 3) * VD + vc] << 16);
            }
            // this thread's q / k units from the swizzled staging (16-byte chunk c of row i sits at chunk
            // c ^ (i % 8) of its 128-byte row)
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int u = tid + NT * it;
                const int i = ((u >> 7) << 3) + (u & 7), d8 = (u >> 3) & 15;
                const uint32_t off = (uint32_t)(d8 >> 3) * 8192u + (uint32_t)i * 128u + ((uint32_t)((d8 & 7) ^ (i & 7)) << 4);
                qr[it] = *reinterpret_cast<const uint4*>(smem + L::STG_Q + off);
                kr[it] = *reinterpret_cast<const uint4*>(smem + L::STG_K + off);
            }
            if (norm_qk) add_row_sumsq(qr, kr, sSqQ, sSqK, tid, lane);  // totals complete after the barrier
            // the previous chunk's record stores must be done reading CK before P3 rewrites it, and
            // the staged tiles in X1 must all be read
            if (tid == 32) bulk_wait_read();
            __syncthreads();
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = 4 * (q0 + 4 * x);
                *reinterpret_cast<uint4*>(smem + L::VT + cm_off(vc, j, CH)) =
                    make_uint4(to_tf32(__uint_as_float(vv[2 * x] << 16)), to_tf32(__uint_as_float(vv[2 * x] & 0xFFFF0000u)),
                               to_tf32(__uint_as_float(vv[2 * x + 1] << 16)),
                               to_tf32(__uint_as_float(vv[2 * x + 1] & 0xFFFF0000u)));
            }
        }

        // ---- P3: [-Khat; Qhat] -> X1, Kchk -> CK; record parts Kend -> KA rows 0-127, Qtil -> QT -----
        uint32_t kh[2][8];  // tf32 bits of -Khat (rotated), kept for Khat^T once Gam is no longer needed
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            const int u = tid + NT * it;
            const int i = ((u >> 7) << 3) + (u & 7), d8 = (u >> 3) & 15;
            float qf[8], kf[8], gf[8], rf[8], sf[8], ef[8], ff[8];
            bf16x8_to_f32(qr[it], qf);
            bf16x8_to_f32(kr[it], kf);
            if (norm_qk) scale_row8(qf, kf, sSqQ[i], sSqK[i]);
            *reinterpret_cast<float4*>(gf) = *reinterpret_cast<const float4*>(sGam + gidx(i, 8 * d8));
            *reinterpret_cast<float4*>(gf + 4) = *reinterpret_cast<const float4*>(sGam + gidx(i, 8 * d8 + 4));
            *reinterpret_cast<float4*>(rf) = *reinterpret_cast<const float4*>(sRho + 8 * d8);
            *reinterpret_cast<float4*>(rf + 4) = *reinterpret_cast<const float4*>(sRho + 8 * d8 + 4);
            *reinterpret_cast<float4*>(sf) = *reinterpret_cast<const float4*>(sSig + 8 * d8);
            *reinterpret_cast<float4*>(sf + 4) = *reinterpret_cast<const float4*>(sSig + 8 * d8 + 4);
            *reinterpret_cast<float4*>(ef) = *reinterpret_cast<const float4*>(sERho + 8 * d8);
            *reinterpret_cast<float4*>(ef + 4) = *reinterpret_cast<const float4*>(sERho + 8 * d8 + 4);
            *reinterpret_cast<float4*>(ff) = *reinterpret_cast<const float4*>(sFend + 8 * d8);
            *reinterpret_cast<float4*>(ff + 4) = *reinterpret_cast<const float4*>(sFend + 8 * d8 + 4);
            uint32_t wq_[8], wc_[8], qt[8], ke[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float e1 = __expf(gf[t] - rf[t]), e2 = __expf(sf[t] - gf[t]);
                const float qh = scale * qf[t] * e1, kc = kf[t] * e2;
                wq_[t] = to_tf32(qh);
                qt[t] = to_tf32(qh * ef[t]);
                kh[it][t] = to_tf32(-kf[t] * e1);
                wc_[t] = to_tf32(kc);
                ke[t] = to_tf32(kc * ff[t]);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int d = 8 * d8 + 4 * hh;
                *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(i, d, KD)) =
                    make_uint4(kh[it][4 * hh], kh[it][4 * hh + 1], kh[it][4 * hh + 2], kh[it][4 * hh + 3]);
                *reinterpret_cast<uint4*>(smem + L::X1 + cm_off(64 + i, d, KD)) =
                    make_uint4(wq_[4 * hh], wq_[4 * hh + 1], wq_[4 * hh + 2], wq_[4 * hh + 3]);
                *reinterpret_cast<uint4*>(smem + L::CK + cm_off(i, d, KD)) =
                    make_uint4(wc_[4 * hh], wc_[4 * hh + 1], wc_[4 * hh + 2], wc_[4 * hh + 3]);
                *reinterpret_cast<uint4*>(smem + L::QT + cm_off(i, d, KD)) =
                    make_uint4(qt[4 * hh], qt[4 * hh + 1], qt[4 * hh + 2], qt[4 * hh + 3]);
            }
            // Kend (transposed): lanes that share a bank (same i & 3) take different d of their group of 8
            rotate_groups8(ke, rot);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                *reinterpret_cast<uint32_t*>(smem + L::KA + cm_off(8 * d8 + ((t + rot) & 7), i, CH)) = ke[t];
            rotate_groups8(kh[it], rot);  // stored transposed the same way below
        }
        fence_proxy_async();
        cta_sync_tc();
        if (tid == 32) {  // Qtil and Kend are final: their record stores run while M1 does
            bulk_store(rec + Rec::WQ + 32768, s_base + L::QT, 32768);  // Wtil goes straight out later
            bulk_store(rec + Rec::KA, s_base + L::KA, 32768);         // A goes straight to the record later
            bulk_commit();
        }

        // Khat^T into GM (B rows 0-127 of M7) once Gam is no longer read
        auto write_khat_t = [&]() {
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int u = tid + NT * it;
                const int i = ((u >> 7) << 3) + (u & 7), d8 = (u >> 3) & 15;
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    *reinterpret_cast<uint32_t*>(smem + L::GM + cm_off(8 * d8 + ((t + rot) & 7), i, CH)) =
                        kh[it][t] ^ 0x80000000u;
            }
        };

        // ---- A -> record (KA rows 128-191), R -> CK region (pitch RP) ----------------------------
        if (!slow) {
            if (tid == 0) {
                gemm_tf32(tmem, s_base + L::X1, KD / 4 * 128, s_base + L::CK, KD / 4 * 128, idesc_tf32(128, 64), KD / 8,
                          false);
                mma_commit(mbar);
            }
            write_khat_t();
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
            // X1 rows 0-63 are free: stage the next chunk of this CTA during the rest of this one
            if (task + gridDim.x < ntasks) load_inputs(make_task(task + gridDim.x, T, H, HV, NC));
            uint32_t raw[16];
            tmem_ld16(taddr(tmem, 32 * wq, 16 * wc), raw);
            tmem_wait_ld();
            if (wq < 2) {  // rows 0-63 of D1 hold -Khat Kchk^T
                const int i = 32 * wq + lane;
                const float bi = -sBeta[i];
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int j = 16 * wc + jj;
                    *reinterpret_cast<float4*>(sRT + i * RP + j) =
                        make_float4(j + 0 < i ? bi * __uint_as_float(raw[jj + 0]) : 0.f,
                                    j + 1 < i ? bi * __uint_as_float(raw[jj + 1]) : 0.f,
                                    j + 2 < i ? bi * __uint_as_float(raw[jj + 2]) : 0.f,
                                    j + 3 < i ? bi * __uint_as_float(raw[jj + 3]) : 0.f);
                }
            } else {  // rows 64-127 hold A (unmasked): masked, tf32, straight into the record
                const int i = 32 * (wq - 2) + lane;
                unsigned char* ra = rec + Rec::KA + 32768;
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int j = 16 * wc + jj;
                    uint4 w4;
                    w4.x = to_tf32(j + 0 <= i ? __uint_as_float(raw[jj + 0]) : 0.f);
                    w4.y = to_tf32(j + 1 <= i ? __uint_as_float(raw[jj + 1]) : 0.f);
                    w4.z = to_tf32(j + 2 <= i ? __uint_as_float(raw[jj + 2]) : 0.f);
                    w4.w = to_tf32(j + 3 <= i ? __uint_as_float(raw[jj + 3]) : 0.f);
                    *reinterpret_cast<uint4*>(ra + cm_off(i, j, CH)) = w4;
                }
            }
        } else {
            if (task + gridDim.x < ntasks) load_inputs(make_task(task + gridDim.x, T, H, HV, NC));
            // exact decay factors: 4096 (i, j) cells, 8 per thread; Gam is still in GM
            float av[8], rr[8];
#pragma unroll 1
            for (int x = 0; x < 8; ++x) {
                const int p = tid + NT * x;
                const int i = p >> 6, j = p & 63;
                float a = 0.f, r = 0.f;
                if (j <= i && i < tk.nn) {
                    const bf16* qi = q + (tk.tk0 + i) * qk_row + (size_t)tk.h * KD;
                    const bf16* ki = k + (tk.tk0 + i) * qk_row + (size_t)tk.h * KD;
                    const bf16* kj = k + (tk.tk0 + j) * qk_row + (size_t)tk.h * KD;
                    for (int d = 0; d < KD; ++d) {
                        const float e = __expf(sGam[gidx(i, d)] - sGam[gidx(j, d)]);
                        const float kd = to_f32(kj[d]) * e;
                        a += to_f32(qi[d]) * kd;
                        r += to_f32(ki[d]) * kd;
                    }
                }
                if (norm_qk && j <= i && i < tk.nn) {
                    const float ikj = inv_l2norm(sSqK[j]);
                    a *= inv_l2norm(sSqQ[i]) * ikj;
                    r *= inv_l2norm(sSqK[i]) * ikj;
                }
                av[x] = (j <= i) ? scale * a : 0.f;
                rr[x] = (j < i) ? sBeta[i] * r : 0.f;
            }
            __syncthreads();  // Gam fully read: GM becomes Khat^T
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int p = tid + NT * x;
                const int i = p >> 6, j = p & 63;
                *reinterpret_cast<uint32_t*>(rec + Rec::KA + 32768 + cm_off(i, j, CH)) = to_tf32(av[x]);
                sRT[i * RP + j] = rr[x];
            }
            write_khat_t();
        }
        __syncthreads();

        // ---- T = (I + R)^{-1} in place; Tb = T diag(beta) -> KA rows 128-191 and 192-255 ----------
        tri_inverse_diag16(sRT, sX, tid);
        tri_inverse_step16(sRT, sX, tid);
        if (tid == 32) bulk_wait_read();  // the Qtil store has read QT before Tb overwrites it
        tri_inverse_step32(sRT, sX, tid);
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
            const uint4 w4 = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(smem + L::KA + 32768 + cm_off(i, 4 * j4, CH)) = w4;
            *reinterpret_cast<uint4*>(smem + L::KA + 49152 + cm_off(i, 4 * j4, CH)) = w4;
        }
        if (tid < 64) sSqQ[tid] = sSqK[tid] = 0.0f;  // read for the last time above; the next chunk's sums follow
        fence_proxy_async();
        cta_sync_tc();

        // ---- M7: D[128][256] = [Tb; Tb] [Khat^T; V^T]^T; rows 0-63 and 64-127 both hold W | U ------
        if (tid == 0) {
            gemm_tf32(tmem, s_base + L::KA + 32768, CH / 4 * 128, s_base + L::GM, CH / 4 * 128, idesc_tf32(128, 256),
                      CH / 8, false);
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }
        {
            // lane quarters 0-1 read W (rows 0-63), quarters 2-3 read U (rows 64-127); wc picks 32 columns
            const int i = 32 * (wq & 1) + lane;
            uint32_t r0[32];
            tmem_ld32(taddr(tmem, 32 * wq, (wq < 2 ? 0 : 128) + 32 * wc), r0);
            tmem_wait_ld();
            if (wq < 2) {  // Wtil = W diag(e^rho) -> record WQ rows 0-63 (tf32, operand tiling)
                unsigned char* rw = rec + Rec::WQ;
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const float4 er = *reinterpret_cast<const float4*>(sERho + 32 * wc + 4 * c4);
                    *reinterpret_cast<uint4*>(rw + cm_off(i, 32 * wc + 4 * c4, KD)) =
                        make_uint4(to_tf32(er.x * __uint_as_float(r0[4 * c4])),
                                   to_tf32(er.y * __uint_as_float(r0[4 * c4 + 1])),
                                   to_tf32(er.z * __uint_as_float(r0[4 * c4 + 2])),
                                   to_tf32(er.w * __uint_as_float(r0[4 * c4 + 3])));
                }
            } else {  // U^T (fp32, row = value column) -> CK region, free once Tb was built
                float* ut = reinterpret_cast<float*>(smem + L::CK);
#pragma unroll
                for (int cc = 0; cc < 32; ++cc) ut[(32 * wc + cc) * CH + i] = __uint_as_float(r0[cc]);
            }
        }
        fence_proxy_async();
        cta_sync_tc();
        if (tid == 32) {
            bulk_store(rec + Rec::UT, s_base + L::CK, 32768);
            bulk_commit();
        }
    }

    if (aborted) {
        if (tid == 0) atomicOr(status, STATUS_TIMEOUT);
        mbar_wait(mbar, phase, WAIT_POLLS);  // one more bounded chance for an MMA in flight to drain
        if (in_pending) mbar_wait(mbar_in, phase_in, WAIT_POLLS);  // and for staged copies in flight
    }
    if (tid == 32) bulk_wait_all();
    cta_sync_tc();
    // Only now may the state kernel that follows be released: every record store of this CTA is
    // complete.  (Triggering earlier is not safe: in a captured graph the dependent's wait returns
    // once every CTA has triggered, and it sees only the memory written before the trigger.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
// Pass 2: the state recurrence over chunks for one (pair, value block).
// ---------------------------------------------------------------------------------------------
template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t a, uint32_t (&r)[N]) {
    static_assert(N == 8 || N == 16 || N % 32 == 0, "row width");
    if constexpr (N == 8) {
        tmem_ld8(a, r);
    } else if constexpr (N == 16) {
        tmem_ld16(a, r);
    } else {
#pragma unroll
        for (int b = 0; b < N / 32; ++b) tmem_ld32(a + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * b));
    }
}

// Thread layout: warp w serves TMEM lane quarter w % 4 (rows 32 (w % 4) + lane of every
// accumulator) and column half w / 4 of the value block (HALF = VB / 2 columns).
//
// One CTA runs chunks [seg L, min(NC, seg L + L)) of one (sequence, value head) pair for one block of
// VB state columns.  With NS = 1 that is the whole sequence.  For long sequences the chunks are split
// into NS segments: the chunk map S -> e^{Gam_end} S + Kend (U - Wtil S) is affine in S, so a segment
// maps its entering state by S -> M S + b, and the segments can run in parallel (DeltaNet-family digest,
// "Chunkwise Triton pipeline": the state pass is the only traversal between chunks).
//   STATE_CARRY  two CTA halves per (pair, segment but the last) carry X = [M | b] through the segment
//                from [I | 0]:
//                half 0 the M columns (identity start, no U: E = -Wtil X), half 1 the b columns (zero
//                start); X is written to `carry` at the end.  No outputs.
//   STATE_OUT    the chunks from the state entering the segment, with the outputs; the last segment
//                writes S_T.  Unsplit (NS = 1) the entering state is S0; split, every segment reads it
//                from `carry`, where scan_chain_kernel left it (so S_T may alias S0 in both cases).
template <int VB, int MODE>
__global__ void __launch_bounds__(STATE_THREADS, 1)
chunk_state_kernel(const unsigned char* __restrict__ rec_base, const float* __restrict__ S0, int T, int HV, int NC,
                   int L, int NS, bf16* __restrict__ o, float* __restrict__ S_T, float* __restrict__ carry,
                   unsigned int* __restrict__ status) {
    using Lay = StateLayout<VB>;
    constexpr bool OUTS = MODE == STATE_OUT;
    constexpr int NVB = VD / VB;
    constexpr int NH = OUTS ? 1 : 2;
    constexpr int HALF = VB / 2;
    extern __shared__ __align__(1024) unsigned char smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar_wq = s_base + Lay::MBAR, bar_mma = bar_wq + 8, bar_ka0 = bar_wq + 16, bar_out = bar_wq + 32;
    int rest = blockIdx.x;
    const int vbi = rest % NVB;
    rest /= NVB;
    const int half = rest % NH;  // STATE_CARRY: 0 = the M columns, 1 = the b columns
    rest /= NH;
    const int nseg = OUTS ? NS : NS - 1;  // the last segment's map is never applied: no carry CTAs for it
    const int seg = rest % nseg, pair = rest / nseg;
    const int vb0 = vbi * VB;
    const int c_begin = seg * L, c_end = min(NC, c_begin + L);
    const bool use_u = OUTS || half == 1;
    const int b = pair / HV, hv = pair - b * HV;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, c0 = (warp >> 2) * HALF;  // lane quarter, first column of this half
    const int rot = lane >> 2;                          // store rotation (see rotate_groups8)
    const size_t v_row = (size_t)HV * VD;
    const unsigned char* rec0 = rec_base + (size_t)pair * NC * Rec::BYTES;
    auto rec = [&](int c) { return rec0 + (size_t)c * Rec::BYTES; };
    // carry slots of (pair, segment): [2][KD][VD] fp32, M then b
    auto carry_slot = [&](int sg, int hf) { return carry + (((size_t)pair * NS + sg) * 2 + hf) * KD * VD; };

    if (tid == 0) {
        mbar_init(bar_wq, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_ka0, 1);
        mbar_init(bar_ka0 + 8, 1);
        mbar_init(bar_out, 1);
    }
    if (warp == 0) tmem_alloc(s_base + Lay::TBASE, Lay::TMEM_COLS);
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::TBASE);

    // loads in flight, for the bounded drain on abort: bit 0 wq, bit 1 + buf ka
    uint32_t pending = 0;
    auto load_wq = [&](int c) {
        mbar_expect_tx(bar_wq, 65536);
        bulk_load(s_base + Lay::WQ, rec(c) + Rec::WQ, 65536, bar_wq);
        pending |= 1u;
    };
    // the carry pass reads Kend only (no A) and, for the M columns, no U
    constexpr uint32_t KA_LOAD = OUTS ? Rec::KA_BYTES : 32768u;
    auto load_ka = [&](int c, int buf) {
        const uint32_t bar = bar_ka0 + 8 * buf;
        mbar_expect_tx(bar, KA_LOAD + (use_u ? VB * 256u : 0u) + 512u);
        bulk_load(s_base + Lay::ka(buf), rec(c) + Rec::KA, KA_LOAD, bar);
        if (use_u) bulk_load(s_base + Lay::ka(buf) + Lay::UT_OFF, rec(c) + Rec::UT + vb0 * 256, VB * 256, bar);
        bulk_load(s_base + Lay::ka(buf) + Lay::VEC_OFF, rec(c) + Rec::VEC, 512, bar);
        pending |= 2u << buf;
    };
    // this thread's part of the state slice: key row d, columns vb0 + c0 .. + HALF, exact fp32
    const int d = 32 * wq + lane;
    float s[HALF];
    {
        const float* src = nullptr;  // row-major [KD][VD] source of the entering state, or none (zeros)
        if (OUTS) src = NS == 1 ? (S0 ? S0 + (size_t)pair * KD * VD : nullptr) : carry_slot(seg == 0 ? NS - 1 : seg - 1, seg == 0 ? 0 : 1);
#pragma unroll
        for (int j = 0; j < HALF; j += 4) {
            float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)d * VD + vb0 + c0 + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            if (!OUTS && half == 0) {  // identity: row d has its 1 in column d
                const int col = vb0 + c0 + j;
                x = make_float4(col == d ? 1.f : 0.f, col + 1 == d ? 1.f : 0.f, col + 2 == d ? 1.f : 0.f,
                                col + 3 == d ? 1.f : 0.f);
            }
            s[j] = x.x;
            s[j + 1] = x.y;
            s[j + 2] = x.z;
            s[j + 3] = x.w;
        }
    }
    // the chunk records are written by the preceding prep kernel: wait for it (a no-op unless this
    // grid was launched as its programmatic dependent; the prep CTAs release it once their records
    // are complete, so only the launch itself overlaps their tail)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {
        load_wq(c_begin);
        load_ka(c_begin, 0);
        if (Lay::NKA == 2 && c_begin + 1 < c_end) load_ka(c_begin + 1, 1);
    }
    // tf32(S)^T into the B operand of M8; lanes sharing a bank store different columns
    auto write_sop = [&]() {
        uint32_t w[HALF];
#pragma unroll
        for (int j = 0; j < HALF; ++j) w[j] = to_tf32(s[j]);
        rotate_groups8(w, rot);
#pragma unroll
        for (int j = 0; j < HALF; ++j)
            *reinterpret_cast<uint32_t*>(smem + Lay::SOP + cm_off(c0 + (j & ~7) + ((j + rot) & 7), d, KD)) = w[j];
    };
    uint32_t ph_wq = 0, ph_mma = 0, ph_ka = 0, ph_out = 0;
    bool aborted = false;
    write_sop();
    fence_proxy_async();
    cta_sync_tc();
    for (int c = c_begin; c < c_end && !aborted; ++c) {
        const int buf = (Lay::NKA == 2) ? ((c - c_begin) & 1) : 0;
        const int n = min(CH, T - c * CH);
        // ---- M8: D1 = [Wtil; Qtil] S ------------------------------------------------------------
        bool ok = true;
        if (tid == 0) {
            ok = mbar_wait(bar_wq, ph_wq, WAIT_POLLS);
            if (ok) {
                pending &= ~1u;
                gemm_tf32(tmem + Lay::D1, s_base + Lay::WQ, KD / 4 * 128, s_base + Lay::SOP, KD / 4 * 128,
                          idesc_tf32(128, VB), KD / 8, false);
                mma_commit(bar_mma);
            }
        }
        ok = mbar_wait(bar_mma, ph_mma, WAIT_POLLS) && ok;
        ok = mbar_wait(bar_ka0 + 8 * buf, (ph_ka >> buf) & 1u, WAIT_POLLS) && ok;
        fence_after_sync();
        if (!__syncthreads_and(ok)) { aborted = true; break; }
        // phases advance only on success, so that on abort they name the operations still pending
        ph_wq ^= 1u;
        ph_mma ^= 1u;
        ph_ka ^= 1u << buf;
        // this chunk's e^{Gam_end}, read before a single KA buffer is refilled below
        const float eg = reinterpret_cast<const float*>(smem + Lay::ka(buf) + Lay::VEC_OFF)[d];
        if (tid == 0) {
            pending &= ~(2u << buf);
            if (c + 1 < c_end) load_wq(c + 1);  // M8 has read WQ
        }
        // ---- E = U - Wtil S (rows 0-63: lane quarters 0, 1) -> E^T tf32 operand ------------------
        const uint32_t ka = s_base + Lay::ka(buf);
        {
            uint32_t r[HALF];
            if (wq < 2) {
                const float* sU = reinterpret_cast<const float*>(smem + Lay::ka(buf) + Lay::UT_OFF);
                tmem_ld_row<HALF>(taddr(tmem, 32 * wq, Lay::D1 + c0), r);
                tmem_wait_ld();
#pragma unroll
                for (int vv = 0; vv < HALF; ++vv)
                    r[vv] = to_tf32((use_u ? sU[(c0 + vv) * CH + d] : 0.f) - __uint_as_float(r[vv]));
                rotate_groups8(r, rot);
            }
            if constexpr (Lay::ALIAS_E) __syncthreads();  // every U^T read done before E^T overwrites them
            if (wq < 2) {
#pragma unroll
                for (int vv = 0; vv < HALF; ++vv)
                    *reinterpret_cast<uint32_t*>(smem + Lay::EOP + cm_off(c0 + (vv & ~7) + ((vv + rot) & 7), d, CH)) =
                        r[vv];
            }
        }
        fence_proxy_async();
        cta_sync_tc();
        // ---- M10: D2 = Kend E (the state side), then M9: D1[64:] += A E (the outputs), each with its
        //      own commit, so that the state update starts after M10 while M9 still runs -------------
        if (tid == 0) {
            gemm_tf32(tmem + Lay::D2, ka, CH / 4 * 128, s_base + Lay::EOP, CH / 4 * 128, idesc_tf32(128, VB), CH / 8,
                      false);
            mma_commit(bar_mma);
            if (OUTS) {
                gemm_tf32(tmem + Lay::D1, ka + 16384, CH / 4 * 128, s_base + Lay::EOP, CH / 4 * 128,
                          idesc_tf32(128, VB), CH / 8, true);
                mma_commit(bar_out);
            }
        }
        ok = mbar_wait(bar_mma, ph_mma, WAIT_POLLS);
        fence_after_sync();
        if (!__syncthreads_and(ok)) { aborted = true; break; }
        ph_mma ^= 1u;
        // ---- state: S = e^{Gam_end} S + D2 --------------------------------------------------------
        {
            uint32_t r[HALF];
            tmem_ld_row<HALF>(taddr(tmem, 32 * wq, Lay::D2 + c0), r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < HALF; ++j) s[j] = fmaf(eg, s[j], __uint_as_float(r[j]));
        }
        bool ok_out = true;
        if constexpr (OUTS) {
            // ---- outputs (rows 64-127 of D1: lane quarters 2, 3), once M9 is done; thread 0 waits for
            //      it too before a KA buffer M9 reads is refilled -------------------------------------
            if (wq >= 2 || tid == 0) {
                ok_out = mbar_wait(bar_out, ph_out, WAIT_POLLS);
                fence_after_sync();
            }
            if (wq >= 2 && ok_out) {
                const int i = d - 64;
                uint32_t r[HALF];
                tmem_ld_row<HALF>(taddr(tmem, 32 * wq, Lay::D1 + c0), r);
                tmem_wait_ld();
                if (i < n) {
                    bf16* op = o + ((size_t)b * T + (size_t)c * CH + i) * v_row + (size_t)hv * VD + vb0 + c0;
#pragma unroll
                    for (int j = 0; j < HALF; j += 8) {
                        uint4 w;
                        __nv_bfloat162 p0 = __floats2bfloat162_rn(__uint_as_float(r[j]), __uint_as_float(r[j + 1]));
                        __nv_bfloat162 p1 = __floats2bfloat162_rn(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                        __nv_bfloat162 p3 = __floats2bfloat162_rn(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                        w.x = *reinterpret_cast<uint32_t*>(&p0);
                        w.y = *reinterpret_cast<uint32_t*>(&p1);
                        w.z = *reinterpret_cast<uint32_t*>(&p2);
                        w.w = *reinterpret_cast<uint32_t*>(&p3);
                        *reinterpret_cast<uint4*>(op + j) = w;
                    }
                }
            }
        }
        // a single KA buffer (and, with 128 columns, the E^T operand over its U^T rows) is refilled once
        // the products that read it (M10, and M9 when there are outputs) are done
        if (Lay::NKA == 1 && tid == 0 && ok_out && c + 1 < c_end) load_ka(c + 1, 0);
        // ---- the next chunk's S operand --------------------------------------------------------
        if (c + 1 < c_end) write_sop();
        fence_proxy_async();
        fence_before_sync();
        if (!__syncthreads_and(ok_out)) { aborted = true; break; }
        fence_after_sync();
        if (OUTS) ph_out ^= 1u;
        if (Lay::NKA == 2 && tid == 0 && c + 2 < c_end) load_ka(c + 2, buf);
    }

    if (aborted) {
        if (tid == 0) {
            atomicOr(status, STATUS_TIMEOUT);
            // bounded drain of copies and MMAs still in flight before shared memory and TMEM go away
            if (pending & 1u) mbar_wait(bar_wq, ph_wq, WAIT_POLLS);
            for (int bb = 0; bb < Lay::NKA; ++bb)
                if (pending & (2u << bb)) mbar_wait(bar_ka0 + 8 * bb, (ph_ka >> bb) & 1u, WAIT_POLLS);
            mbar_wait(bar_mma, ph_mma, WAIT_POLLS);
            if (OUTS) mbar_wait(bar_out, ph_out, WAIT_POLLS);
        }
    } else {
        float* dst = nullptr;
        if (!OUTS) dst = carry_slot(seg, half);
        else if (S_T && seg == NS - 1) dst = S_T + (size_t)pair * KD * VD;
        if (dst) {
#pragma unroll
            for (int j = 0; j < HALF; j += 4)
                *reinterpret_cast<float4*>(dst + (size_t)d * VD + vb0 + c0 + j) =
                    make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
    }
    cta_sync_tc();
    if (warp == 0) tmem_dealloc(tmem, Lay::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
// Between the two state passes: the segments of each pair in order, S_{s+1} = M_s S_s + b_s in fp32
// on the CUDA cores (value columns are independent: one CTA per (pair, block of 16 columns)).  The
// state entering segment s + 1 overwrites b_s in `carry`, where the STATE_OUT pass reads it.  The last
// segment's map M_{NS-1} is never applied, so its slot receives the state entering segment 0 (S0 or
// zeros): the output pass then reads no S0, and S_T may alias S0.
// ---------------------------------------------------------------------------------------------
constexpr int CHAIN_THREADS = 256, CHAIN_COLS = 16;

__global__ void __launch_bounds__(CHAIN_THREADS)
scan_chain_kernel(const float* __restrict__ S0, float* __restrict__ carry, int NS) {
    __shared__ __align__(16) float sS[KD][CHAIN_COLS];
    constexpr int NCB = VD / CHAIN_COLS;
    const int pair = blockIdx.x / NCB, col0 = (blockIdx.x % NCB) * CHAIN_COLS;
    const int tid = threadIdx.x, d = tid >> 1, cc = (tid & 1) * 8;  // row d, 8 columns from cc
    const float* s0 = S0 ? S0 + (size_t)pair * KD * VD : nullptr;
#pragma unroll
    for (int j = 0; j < 8; j += 4)
        *reinterpret_cast<float4*>(&sS[d][cc + j]) =
            s0 ? *reinterpret_cast<const float4*>(s0 + (size_t)d * VD + col0 + cc + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    {
        float* first = carry + ((size_t)pair * NS + NS - 1) * 2 * KD * VD + (size_t)d * VD + col0 + cc;
        *reinterpret_cast<float4*>(first) = *reinterpret_cast<const float4*>(&sS[d][cc]);
        *reinterpret_cast<float4*>(first + 4) = *reinterpret_cast<const float4*>(&sS[d][cc + 4]);
    }
    __syncthreads();
    for (int sg = 0; sg + 1 < NS; ++sg) {
        const float* M = carry + ((size_t)pair * NS + sg) * 2 * KD * VD;
        float* bs = carry + (((size_t)pair * NS + sg) * 2 + 1) * KD * VD + (size_t)d * VD + col0 + cc;
        float acc[8];
        {
            const float4 b0 = *reinterpret_cast<const float4*>(bs), b1 = *reinterpret_cast<const float4*>(bs + 4);
            acc[0] = b0.x; acc[1] = b0.y; acc[2] = b0.z; acc[3] = b0.w;
            acc[4] = b1.x; acc[5] = b1.y; acc[6] = b1.z; acc[7] = b1.w;
        }
        const float* Mrow = M + (size_t)d * VD;
#pragma unroll 4
        for (int e4 = 0; e4 < KD; e4 += 4) {
            const float4 m = __ldg(reinterpret_cast<const float4*>(Mrow + e4));
            const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float4 x0 = *reinterpret_cast<const float4*>(&sS[e4 + t][cc]);
                const float4 x1 = *reinterpret_cast<const float4*>(&sS[e4 + t][cc + 4]);
                acc[0] = fmaf(mv[t], x0.x, acc[0]); acc[1] = fmaf(mv[t], x0.y, acc[1]);
                acc[2] = fmaf(mv[t], x0.z, acc[2]); acc[3] = fmaf(mv[t], x0.w, acc[3]);
                acc[4] = fmaf(mv[t], x1.x, acc[4]); acc[5] = fmaf(mv[t], x1.y, acc[5]);
                acc[6] = fmaf(mv[t], x1.z, acc[6]); acc[7] = fmaf(mv[t], x1.w, acc[7]);
            }
        }
        __syncthreads();  // every row of the old state read
        *reinterpret_cast<float4*>(&sS[d][cc]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(&sS[d][cc + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        *reinterpret_cast<float4*>(bs) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(bs + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------------
// Segments of the state pass.  Cost model, in thousands of cycles of one CTA per SM: the unsplit pass is
// a chain of NC steps per wave of (pair, value block) CTAs, one step taking about 3.6K cycles with 16
// columns, 4.8K with 32 and 6K with 64 (as launch_chunk_split picks the block width); the split one runs
// 2 x pairs x (NS - 1) carry CTAs, then pairs x NS output CTAs, of L chunks each, in waves over the SMs,
// one 128-column step taking about 10.3K cycles, plus the segment chain at about 3K cycles per segment
// (measured on B200 with tf32 records).  The split therefore pays only where the unsplit pass leaves SMs
// idle: few (sequence, head) pairs and long sequences.  The number of SMs is a planning constant (a
// B200's 148), so that the workspace size does not depend on the device; the split is taken where the
// model gains at least a fifth.
ScanPlan chunk_scan_plan(long long pairs, int NC) {
    constexpr long long kPlanSMs = 148;
    const long long nvb = pairs * 8 <= kPlanSMs ? 8 : pairs * 4 <= kPlanSMs ? 4 : 2;
    const double t_unsplit = nvb == 8 ? 3.6 : nvb == 4 ? 4.8 : 6.0, t_split = 10.3, t_chain = 3.0;
    ScanPlan plan{NC, 1};
    double best = 0.8 * (double)NC * t_unsplit * (double)((pairs * nvb + kPlanSMs - 1) / kPlanSMs);
    for (int Lc : {8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256}) {
        if (Lc >= NC) break;
        const long long NS = (NC + Lc - 1) / Lc;
        const long long wa = (2 * pairs * (NS - 1) + kPlanSMs - 1) / kPlanSMs;
        const long long wc = (pairs * NS + kPlanSMs - 1) / kPlanSMs;
        const double cost = (double)(wa + wc) * Lc * t_split + t_chain * (double)NS;
        if (cost < best) {
            best = cost;
            plan = ScanPlan{Lc, (int)NS};
        }
    }
    return plan;
}

size_t chunk_split_workspace(int B, int T, int HV) {
    const size_t NC = ((size_t)T + CH - 1) / CH;
    const long long pairs = (long long)B * HV;
    const ScanPlan plan = chunk_scan_plan(pairs, (int)NC);
    const size_t carry = plan.NS > 1 ? (size_t)pairs * plan.NS * 2 * KD * VD * sizeof(float) : 0;
    return (size_t)pairs * NC * Rec::BYTES + carry;
}

namespace {
// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// Tensor map over a bf16 [B][T][heads][128] tensor whose box is 64 tokens of one head and `inner`
// entries of the last dimension: plain rows for inner = 128, 128-byte rows with the 128-byte swizzle
// for inner = 64.  Tokens past T read as zero.
cudaError_t make_token_tile_map(CUtensorMap* m, const void* base, int B, int T, int heads, int inner) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {128, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, (cuuint64_t)heads * 256, (cuuint64_t)T * heads * 256};  // bytes
    const cuuint32_t box[4] = {(cuuint32_t)inner, 1, (cuuint32_t)CH, 1};
    const cuuint32_t estride[4] = {1, 1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estride,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, inner == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_prep(const ChunkArgs& a, int NC, int ntasks, int grid) {
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PrepLayout::BYTES);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv, tg;
    if ((e = make_token_tile_map(&tq, a.q, a.B, a.T, a.H, 64)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&tk, a.k, a.B, a.T, a.H, 64)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&tv, a.v, a.B, a.T, a.HV, 128)) != cudaSuccess) return e;
    if ((e = make_token_tile_map(&tg, a.g, a.B, a.T, a.HV, 128)) != cudaSuccess) return e;
    chunk_prep_kernel<MODE><<<grid, PREP_THREADS, PrepLayout::BYTES, a.stream>>>(
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k), static_cast<const bf16*>(a.v),
        static_cast<const bf16*>(a.g), static_cast<const bf16*>(a.beta), a.A_log, a.dt_bias, a.T, a.H, a.HV, NC,
        ntasks, a.lower_bound, a.scale, a.flags, static_cast<unsigned char*>(a.scratch), a.status, tq, tk, tv, tg);
    return cudaGetLastError();
}

template <int VB, int MODE>
cudaError_t launch_state(const ChunkArgs& a, int NC, ScanPlan plan, float* carry, bool dependent) {
    using L = StateLayout<VB>;
    auto kern = chunk_state_kernel<VB, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    const long long nseg = MODE == STATE_OUT ? plan.NS : plan.NS - 1;
    cfg.gridDim = dim3((unsigned)((long long)a.B * a.HV * nseg * (MODE == STATE_OUT ? 1 : 2) * (VD / VB)));
    cfg.blockDim = dim3(STATE_THREADS);
    cfg.dynamicSmemBytes = L::BYTES;
    cfg.stream = a.stream;
    // programmatic dependent launch right after the prep kernel: the state kernel's set-up may overlap
    // the prep kernel's tail; it waits (griddepcontrol.wait) for the prep grid before reading a record
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const unsigned char*>(a.scratch), a.S0, a.T, a.HV, NC, plan.L,
                              plan.NS, static_cast<bf16*>(a.o), a.S_T, carry, a.status);
}
}  // namespace

cudaError_t launch_chunk_split(const ChunkArgs& a) {
    const int NC = (a.T + CH - 1) / CH;
    const int ntasks = a.B * a.HV * NC;  // < 2^30: checked by kda_chunk_fwd_schedule
    int dev = 0, nsm = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int grid = ntasks < nsm ? ntasks : nsm;
    e = a.gate_mode == KDA_GATE_SAFE       ? launch_prep<KDA_GATE_SAFE>(a, NC, ntasks, grid)
        : a.gate_mode == KDA_GATE_STANDARD ? launch_prep<KDA_GATE_STANDARD>(a, NC, ntasks, grid)
                                           : launch_prep<KDA_GATE_NONE>(a, NC, ntasks, grid);
    if (e != cudaSuccess) return e;
    const long long pairs = (long long)a.B * a.HV;
    const ScanPlan plan = chunk_scan_plan(pairs, NC);
    if (plan.NS == 1) {
        // value-block width: enough (pair, block) CTAs to cover the SMs, blocks as wide as that allows
        if (pairs * 8 <= nsm) return launch_state<16, STATE_OUT>(a, NC, plan, nullptr, true);
        if (pairs * 4 <= nsm) return launch_state<32, STATE_OUT>(a, NC, plan, nullptr, true);
        return launch_state<64, STATE_OUT>(a, NC, plan, nullptr, true);
    }
    // long sequences: carry [M | b] through every segment, chain the segments, then the outputs
    float* carry = reinterpret_cast<float*>(static_cast<unsigned char*>(a.scratch) + (size_t)pairs * NC * Rec::BYTES);
    if ((e = launch_state<128, STATE_CARRY>(a, NC, plan, carry, true)) != cudaSuccess) return e;
    scan_chain_kernel<<<(unsigned)(pairs * (VD / CHAIN_COLS)), CHAIN_THREADS, 0, a.stream>>>(a.S0, carry, plan.NS);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_state<128, STATE_OUT>(a, NC, plan, carry, false);
}

}  // namespace kda
