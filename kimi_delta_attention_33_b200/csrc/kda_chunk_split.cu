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
// M7 = [Tb; A] [Khat^T; V^T]^T -> W and U (rows 0-63), and the products that fold the delta errors
// into the record:
//   S_c+1 = e^{Gam_end} S_c + Kend (U - Wtil S_c) = e^{Gam_end} S_c - G S_c + KU,  G = Kend Wtil, KU = Kend U
//   O      = Qtil S_c + A (U - Wtil S_c)          = Q' S_c + A U,               Q' = Qtil - A Wtil
// M11 = Kend [Wtil^T; U^T]^T -> [G | KU] and M12 = [Tb; A] [Wtil^T; U^T]^T -> [A Wtil | A U] (rows 64-127),
// written to a per-chunk record in the workspace:
//   WQ  [G; Q']   192 x 128 fp16 in the K-major tiling of kda_tc_ptx.cuh (A operands of the state pass)
//   KU  128 x 128 fp16, AU 64 x 128 fp32, both by blocks of 16 value columns
//   VEC e^{Gam_end} (fp32, 128), then the scale block
// Every fp16 tile (G, Q', KU) is stored as tile * 2^-e with one power-of-two exponent e per tile, chosen
// from the tile's largest magnitude so that the scaled tile uses fp16's range (kda_tc_ptx.cuh,
// fp16_scale_exponent); the exponents sit in the scale block.  fp16 carries the same 10 fraction bits as
// tf32, and the powers of two come off exactly on the fp32 accumulators.  The decay e^{Gam_end} S stays
// an exact fp32 product: only the low-rank corrections G S and KU are rounded.
// Pass 2 (chunk_state_kernel, one CTA per (pair, block of VB value columns), chunks in order):
// the state slice S_c[:, block] lives in registers (thread d owns key row d, exact fp32);
// per chunk, with fp16(S_c 2^-sig)^T staged in shared memory as a B operand:
//   chain  D_S = G S_c                     -> S_c+1 = e^{Gam_end} S_c - D_S + KU, in registers
//   out    D_O = Q' S_c (M = 64)           -> O = Q' S_c + A U, read out while the next chunk's chain
//                                             product runs
// One tensor-core round trip per chunk is on the chunk-to-chunk path.  The state scale is not reduced over
// the CTA on the chain: it comes from a bound that all threads compute alike (see chunk_state_kernel).
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

// Per-chunk record in the workspace (bytes).  KU and AU are stored as 16-byte chunks of consecutive value
// columns, rows contiguous within a chunk column: a block of 16 value columns is one contiguous 4 KB range
// (one copy per block), and 16-byte accesses by consecutive rows touch consecutive banks.
struct Rec {
    static constexpr uint32_t WQ = 0;          // [192][128] fp16 tiles: G 2^-eg (rows 0-127), Q' 2^-eq (rows 128-191)
    static constexpr uint32_t WQ_BYTES = 49152;
    static constexpr uint32_t QP_OFF = 32768;  // row 128 of WQ
    static constexpr uint32_t KU = 49152;      // fp16 [16][128][8]: KU 2^-eu, 8 value columns per row chunk
    static constexpr uint32_t AU = 81920;      // fp32 [32][64][4]: A U, 4 value columns per row chunk
    static constexpr uint32_t VEC = 114688;    // [128] fp32 e^{Gam_end}, then the scale block at SCL
    static constexpr uint32_t SCL = VEC + 512; // int eg, eq, eu; float max e^{Gam_end}
    static constexpr uint32_t VEC_LOAD = 528;  // bytes of VEC the state pass reads
    static constexpr uint32_t BYTES = 115712;
    static_assert(SCL + 16 <= VEC + VEC_LOAD && VEC + 1024 <= BYTES && BYTES % 256 == 0, "record layout");
};
// slots of the per-chunk maxima in the prep kernel (PrepLayout::MX)
enum : int { MX_QT = 0, MX_K = 1, MX_A = 2, MX_W = 3, MX_U = 4, MX_EG = 5, MX_SLOTS = 8 };

struct PrepLayout {
    static constexpr uint32_t X1 = 0;        // [128][128] [-Khat; Qhat] (A of M1); once M1 is done X1 stages
                                             //   the next chunk's input tiles, bf16 [64][128] each: g, v
                                             //   (plain rows), q, k (two 64-column halves each, rows of 128
                                             //   bytes with the 128-byte swizzle)
    static constexpr uint32_t CK = 65536;    // [64][128] Kchk (B of M1); then R / T (pitch RP) + doubling
                                             //   scratch; then U^T [128][64] fp32 (record UT)
    static constexpr uint32_t XS = CK + 64 * RP * 4;
    static constexpr uint32_t KA = 98304;    // [256][64]: Kend^T rows 0-127 (A of M11), Tb in rows 128-191 and
                                             //   the masked A in rows 192-255 (A of M7 and M12)
    static constexpr uint32_t GM = 163840;   // Gam (fp32 [64][128]) -> Khat^T [128][64] (B rows 0-127 of M7)
    static constexpr uint32_t VT = 196608;   // V^T [128][64] (B rows 128-255 of M7); after M7 GM and VT hold
                                             //   BT = [Wtil^T; U^T] [256][64], the B operand of M11 and M12
    static constexpr uint32_t VEC = 229376;
    static constexpr uint32_t RHO = VEC, SIG = VEC + 512, BETA = VEC + 1024, ERHO = VEC + 1280, FEND = VEC + 1792;
    static constexpr uint32_t MBAR = VEC + 2304, MBAR_IN = MBAR + 8, TBASE = MBAR_IN + 8;
    static constexpr uint32_t SQQ = VEC + 2336, SQK = VEC + 2592;  // [64] row sums of squares of q, k
    static constexpr uint32_t MX = VEC + 2848;  // [MX_SLOTS] per-chunk maxima of the record tiles (float bits)
    static constexpr uint32_t QT = KA + 32768;    // record Qtil staging, in the Tb rows (free until the inverse)
    static constexpr uint32_t PART = KA + 49152;  // gate: per-channel quarter totals and Gam_0 (5 x [128] fp32),
                                                  //   in KA rows 192-255, free until M1 is read out and not
                                                  //   part of the record staging below
    // record staging at the end of a chunk (bulk stores, done reading before the next chunk's V^T step):
    // [G; Q'] fp16 in KA rows 0-191, KU in CK, AU in VT
    static constexpr uint32_t STG_G = X1, STG_V = X1 + 16384, STG_Q = X1 + 32768, STG_K = X1 + 49152;
    static constexpr uint32_t BYTES = MX + 4 * MX_SLOTS;
    static constexpr uint32_t TMEM_COLS = 512;  // D [128][64] for M1, [128][256] for M7, then [128][512] for M11, M12
    static_assert(XS + 1024 * 4 <= KA, "doubling scratch");
    static_assert(GM + 32768 == VT, "M7's B operand spans GM and VT");
    static_assert(BYTES <= 232448, "shared memory budget");
};

// What one state-pass CTA computes over its chunks (see chunk_state_kernel).
enum : int { STATE_OUT = 0, STATE_CARRY = 1 };

// Shared memory of one state-pass CTA.  Record slots hold, per chunk, [G; Q'] (G only without outputs), this
// block's columns of KU and AU, and VEC.  With outputs a slot stays in use until the step after its own (the
// outputs are read out then), so three slots keep the copies two chunks ahead; without, two.
template <int VB, int MODE>
struct StateLayout {
    static constexpr bool OUTS = MODE == STATE_OUT;
    static constexpr int NBUF = OUTS ? 3 : 2;
    static constexpr int NSOP = OUTS ? 2 : 1;                  // S operands: by chunk parity when the output
                                                               // product of a chunk may still read its own
    static constexpr uint32_t WQ_LOAD = OUTS ? Rec::WQ_BYTES : Rec::QP_OFF;
    static constexpr uint32_t KU_OFF = WQ_LOAD, AU_OFF = KU_OFF + VB * 256;
    static constexpr uint32_t VEC_OFF = AU_OFF + (OUTS ? VB * 256 : 0);
    static constexpr uint32_t SLOT = VEC_OFF + 1024;
    // fp16 S^T [VB][128] per buffer (B operand), in the padded tiling: K-adjacent core matrices 144 bytes
    // apart (SOP_LBO), 8-row groups 16 x 144 bytes apart (SOP_SBO)
    static constexpr uint32_t SOP_LBO = 144, SOP_SBO = 16 * SOP_LBO, SOP_BYTES = VB / 8 * SOP_SBO;
    static constexpr uint32_t SOP = NBUF * SLOT;
    static constexpr uint32_t MBAR = SOP + NSOP * SOP_BYTES;   // rec[NBUF], chain, out[2]
    static constexpr uint32_t TBASE = MBAR + 8 * (NBUF + 3);
    static constexpr uint32_t SMX = TBASE + 16;                // [2][8] per-warp max |S|, by chunk parity
    static constexpr uint32_t BYTES = SMX + 64;
    // D_S = G S (chain); D_O[2] = Q' S (M = 64, lanes 32 q + 0..15), by chunk parity
    static constexpr int D_S = 0, D_O = VB;
    static constexpr uint32_t NCOL = OUTS ? 3 * VB : VB;
    static constexpr uint32_t TMEM_COLS = NCOL <= 32 ? 32 : NCOL <= 64 ? 64 : NCOL <= 128 ? 128 : NCOL <= 256 ? 256 : 512;
    static __device__ __forceinline__ uint32_t slot(int k) { return k * SLOT; }
    static_assert(SLOT % 1024 == 0 && BYTES <= 232448, "shared memory budget");
};


constexpr int STATE_WARPS = 8;                         // warps that own the state slice
constexpr int STATE_THREADS = 32 * (STATE_WARPS + 2);  // and two that issue the chain and the output products
constexpr int ISSUER = 32 * STATE_WARPS, OUT_ISSUER = ISSUER + 32;
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

// Folds this thread's maximum magnitude into a shared slot (float bits; every lane of the warp calls).
__device__ __forceinline__ void max_into_slot(float m, unsigned int* slot, int lane) {
    m = warp_max_nonneg(m);
    if (lane == 0) atomicMax(slot, __float_as_uint(m));
}

__device__ __forceinline__ float slot_value(const unsigned int* slot) {
    return __uint_as_float(*reinterpret_cast<const volatile unsigned int*>(slot));
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
    unsigned int* sMx = reinterpret_cast<unsigned int*>(smem + L::MX);
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
    if (tid < MX_SLOTS) sMx[tid] = 0u;
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::TBASE);
    uint32_t phase = 0, phase_in = 0;
    bool aborted = false, in_pending = false;

    // Inputs of one chunk: the q, k, g and v tiles into X1 by six tensor-map copies issued by thread 32
    // (rows past T read as zero), completing on mbar_in; beta, this head's A_log and this thread's
    // dt_bias entry into registers.  q / k are read back in the operand pass as units u = tid + NT * it: row
    // i = 8 (u / 128) + u % 8, key group d8 = (u / 8) % 16.
    uint32_t beta_bits = 0;  // raw bf16 bits of beta for row tid (tid < 64), converted where used
    float alog_in = 0.f, bias_in = 0.f;
    auto load_inputs = [&](const Task& tk) {
        if (tid == 32) {
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
                const float eg = __expf(gend);
                reinterpret_cast<float*>(rec + Rec::VEC)[gd] = eg;
                max_into_slot(eg, sMx + MX_EG, lane);  // warps 0-3 are exactly the gq = 0 threads
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
            // the previous chunk's record stores must be done reading KA, CK and VT (their staging) before this
            // chunk rewrites them, and the staged tiles in X1 must all be read
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

        // ---- P3: [-Khat; Qhat] -> X1, Kchk -> CK, Kend^T -> KA rows 0-127 (A of M11); Qtil (fp32) -> QT;
        //      the largest magnitudes of Qtil and Kend ----------------------------------------------------
        uint32_t kh[2][8];  // tf32 bits of -Khat (rotated), kept for Khat^T once Gam is no longer needed
        float mq = 0.f, mk = 0.f;
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
                const float qtil = qh * ef[t], kend = kc * ff[t];
                mq = fmaxf(mq, fabsf(qtil));
                mk = fmaxf(mk, fabsf(kend));
                wq_[t] = to_tf32(qh);
                qt[t] = __float_as_uint(qtil);
                kh[it][t] = to_tf32(-kf[t] * e1);
                wc_[t] = to_tf32(kc);
                ke[t] = to_tf32(kend);
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
        max_into_slot(mq, sMx + MX_QT, lane);
        max_into_slot(mk, sMx + MX_K, lane);
        fence_proxy_async();
        cta_sync_tc();
        if (!slow && tid == 0) {
            gemm_tf32(tmem, s_base + L::X1, KD / 4 * 128, s_base + L::CK, KD / 4 * 128, idesc_tf32(128, 64), KD / 8,
                      false);
            mma_commit(mbar);
        }
        // Qtil (fp32) into TMEM rows 64-127, columns 256-383, and zeros into columns 384-511, while M1 runs: M12
        // accumulates [-A Wtil | -A U] onto them
        if (wq >= 2) {
            const int i = 32 * (wq - 2) + lane;
            uint32_t x[32];
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const uint4 v4 = *reinterpret_cast<const uint4*>(smem + L::QT + cm_off(i, 32 * wc + 4 * c4, KD));
                x[4 * c4] = v4.x;
                x[4 * c4 + 1] = v4.y;
                x[4 * c4 + 2] = v4.z;
                x[4 * c4 + 3] = v4.w;
            }
            tmem_st32(taddr(tmem, 32 * wq, 256 + 32 * wc), x);
#pragma unroll
            for (int t = 0; t < 32; ++t) x[t] = 0u;
            tmem_st32(taddr(tmem, 32 * wq, 384 + 32 * wc), x);
            tmem_wait_st();
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
            } else {  // rows 64-127 hold A (unmasked): masked, negated, tf32, into KA rows 192-255 (A of M12)
                const int i = 32 * (wq - 2) + lane;
                float m = 0.f;
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int j = 16 * wc + jj;
                    float a4[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        a4[t] = j + t <= i ? __uint_as_float(raw[jj + t]) : 0.f;
                        m = fmaxf(m, fabsf(a4[t]));
                    }
                    *reinterpret_cast<uint4*>(smem + L::KA + 49152 + cm_off(i, j, CH)) =
                        make_uint4(to_tf32(-a4[0]), to_tf32(-a4[1]), to_tf32(-a4[2]), to_tf32(-a4[3]));
                }
                max_into_slot(m, sMx + MX_A, lane);
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
            {
                float m = 0.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) m = fmaxf(m, fabsf(av[x]));
                max_into_slot(m, sMx + MX_A, lane);
            }
            __syncthreads();  // Gam fully read: GM becomes Khat^T
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int p = tid + NT * x;
                const int i = p >> 6, j = p & 63;
                *reinterpret_cast<uint32_t*>(smem + L::KA + 49152 + cm_off(i, j, CH)) = to_tf32(-av[x]);
                sRT[i * RP + j] = rr[x];
            }
            write_khat_t();
        }
        __syncthreads();

        // ---- T = (I + R)^{-1} in place; Tb = T diag(beta) -> KA rows 128-191 --------------------------
        tri_inverse_diag16(sRT, sX, tid);
        tri_inverse_step16(sRT, sX, tid);
        // Tb = T diag(beta) into KA rows 128-191: the diagonal blocks (final now) while step 32 -> 64 runs, which
        // writes the lower-left block itself
        tb_outside_lower_left(sRT, tid, sBeta, smem + L::KA + 32768);
        tri_inverse_step32_tb(sRT, sX, tid, sBeta, smem + L::KA + 32768);
        if (tid < 64) sSqQ[tid] = sSqK[tid] = 0.0f;  // read for the last time above; the next chunk's sums follow
        fence_proxy_async();
        cta_sync_tc();

        // ---- M7: D[:, 0:64] = Khat^T Tb^T = W^T and D[:, 64:128] = V^T Tb^T = U^T (rows d / v, columns i) ----
        if (tid == 0) {
            gemm_tf32(tmem, s_base + L::GM, CH / 4 * 128, s_base + L::KA + 32768, CH / 4 * 128, idesc_tf32(128, 64),
                      CH / 8, false);
            gemm_tf32(tmem + 64, s_base + L::VT, CH / 4 * 128, s_base + L::KA + 32768, CH / 4 * 128, idesc_tf32(128, 64),
                      CH / 8, false);
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }
        // BT = [Wtil^T; U^T] (tf32 [256][64] over GM and VT, which M7 has read), Wtil^T = diag(e^rho) W^T: warp
        // (wq, wc) stores 32 columns i of row 32 wq + lane of W^T (wc < 2) or of U^T (wc >= 2)
        {
            const int r = 32 * wq + lane;
            const bool isW = wc < 2;
            uint32_t x[32];
            tmem_ld32(taddr(tmem, 32 * wq, (isW ? 0 : 64) + 32 * (wc & 1)), x);
            tmem_wait_ld();
            const float sc = isW ? sERho[r] : 1.f;
            float m = 0.f;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const float v = __uint_as_float(x[t]) * sc;
                m = fmaxf(m, fabsf(v));
                x[t] = to_tf32(v);
            }
            max_into_slot(m, sMx + (isW ? MX_W : MX_U), lane);
            const int n = (isW ? 0 : 128) + r;
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
                *reinterpret_cast<uint4*>(smem + L::GM + cm_off(n, 32 * (wc & 1) + 4 * c4, CH)) =
                    make_uint4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
        }
        fence_proxy_async();
        cta_sync_tc();

        // ---- M11: D[:, 0:256] = Kend^T BT^T = [G | KU];  M12: D[:, 256:512] = [Tb; -A] BT^T, rows 64-127:
        //      Qtil - A Wtil = Q' (accumulated onto Qtil) and -A U -------------------------------------------
        if (tid == 0) {
            gemm_tf32(tmem, s_base + L::KA, CH / 4 * 128, s_base + L::GM, CH / 4 * 128, idesc_tf32(128, 256), CH / 8,
                      false);
            gemm_tf32(tmem + 256, s_base + L::KA + 32768, CH / 4 * 128, s_base + L::GM, CH / 4 * 128,
                      idesc_tf32(128, 256), CH / 8, true);  // B = BT rows 0-255 (GM, then VT)
            mma_commit(mbar);
        }
        {
            const bool ok = mbar_wait(mbar, phase, WAIT_POLLS);
            fence_after_sync();
            if (!__syncthreads_and(ok)) { aborted = true; break; }
            phase ^= 1u;
        }
        // ---- read-out to the record, staged in shared memory that M11 and M12 have read (KA, VT) or that is
        //      free since Tb (CK), then three bulk stores.  Every warp: 64 columns of [G | KU] (rows d = lane
        //      quarter); the warps of lane quarters 2, 3 also 64 columns of [Q' | -A U] (rows i = d - 64).  The
        //      fp16 exponents come from bounds on the tiles (64 products per entry, a factor 2 for the tf32
        //      operands), so that one pass converts. --------------------------------------------------------
        const float kmax = slot_value(sMx + MX_K), wmax = slot_value(sMx + MX_W);
        const int e_g = fp16_scale_exponent(128.f * kmax * wmax);
        const int e_u = fp16_scale_exponent(128.f * kmax * slot_value(sMx + MX_U));
        const int e_q = fp16_scale_exponent(slot_value(sMx + MX_QT) + 128.f * slot_value(sMx + MX_A) * wmax);
        {
            const int d = 32 * wq + lane;
            const bool isG = wc < 2;
            const float f = exp2i(-(isG ? e_g : e_u));
            uint32_t r[32];
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                tmem_ld32(taddr(tmem, 32 * wq, 64 * wc + 32 * h), r);
                tmem_wait_ld();
                uint4 w[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    w[c] = make_uint4(pack_f16x2(__uint_as_float(r[8 * c]) * f, __uint_as_float(r[8 * c + 1]) * f),
                                      pack_f16x2(__uint_as_float(r[8 * c + 2]) * f, __uint_as_float(r[8 * c + 3]) * f),
                                      pack_f16x2(__uint_as_float(r[8 * c + 4]) * f, __uint_as_float(r[8 * c + 5]) * f),
                                      pack_f16x2(__uint_as_float(r[8 * c + 6]) * f, __uint_as_float(r[8 * c + 7]) * f));
                if (isG) {  // G row d, columns 64 wc + 32 h + 8 c: operand tiling
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(smem + L::KA + cm_off16(d, 64 * wc + 32 * h + 8 * c, KD)) = w[c];
                } else {    // KU row d, value columns v = 64 (wc - 2) + 32 h + 8 c
                    const int v0 = 64 * (wc - 2) + 32 * h;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int v = v0 + 8 * c;
                        *reinterpret_cast<uint4*>(smem + L::CK + ((v >> 3) * KD + d) * 16) = w[c];
                    }
                }
            }
            if (wq >= 2) {
                const int i = d - 64;
                const float fq = exp2i(-e_q);
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    tmem_ld32(taddr(tmem, 32 * wq, 256 + 64 * wc + 32 * h), r);
                    tmem_wait_ld();
                    if (isG) {  // Q' row i, columns 64 wc + 32 h + 8 c: operand tiling, rows 128-191 of [G; Q']
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4*>(smem + L::KA + Rec::QP_OFF + cm_off16(i, 64 * wc + 32 * h + 8 * c, KD)) =
                                make_uint4(pack_f16x2(__uint_as_float(r[8 * c]) * fq, __uint_as_float(r[8 * c + 1]) * fq),
                                           pack_f16x2(__uint_as_float(r[8 * c + 2]) * fq, __uint_as_float(r[8 * c + 3]) * fq),
                                           pack_f16x2(__uint_as_float(r[8 * c + 4]) * fq, __uint_as_float(r[8 * c + 5]) * fq),
                                           pack_f16x2(__uint_as_float(r[8 * c + 6]) * fq, __uint_as_float(r[8 * c + 7]) * fq));
                    } else {    // A U row i (negated back), value columns 64 (wc - 2) + 32 h + 4 c: fp32
                        const int v0 = 64 * (wc - 2) + 32 * h;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int v = v0 + 4 * c;
                            *reinterpret_cast<uint4*>(smem + L::VT + ((v >> 2) * 64 + i) * 16) =
                                make_uint4(r[4 * c] ^ 0x80000000u, r[4 * c + 1] ^ 0x80000000u, r[4 * c + 2] ^ 0x80000000u,
                                           r[4 * c + 3] ^ 0x80000000u);
                        }
                    }
                }
            }
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (tid == 32) {
            bulk_store(rec + Rec::WQ, s_base + L::KA, Rec::WQ_BYTES);
            bulk_store(rec + Rec::KU, s_base + L::CK, 32768);
            bulk_store(rec + Rec::AU, s_base + L::VT, 32768);
            bulk_commit();
        }
        if (tid == 0) {  // the scale block; then the maxima start over for the next chunk
            int* sc = reinterpret_cast<int*>(rec + Rec::SCL);
            sc[0] = e_g;
            sc[1] = e_q;
            sc[2] = e_u;
            sc[3] = (int)sMx[MX_EG];
#pragma unroll
            for (int x = 0; x < MX_SLOTS; ++x) sMx[x] = 0u;
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

// Thread layout: warp w < 8 serves TMEM lane quarter w % 4 (rows 32 (w % 4) + lane of every
// accumulator) and column half w / 4 of the value block (HALF = VB / 2 columns); warp 8 issues the record
// copies and the tensor-core products (one thread), so that no state row waits while the products issue.
//
// One CTA runs chunks [seg L, min(NC, seg L + L)) of one (sequence, value head) pair for one block of
// VB state columns.  With NS = 1 that is the whole sequence.  For long sequences the chunks are split
// into NS segments: the chunk map S -> e^{Gam_end} S - G S + KU is affine in S, so a segment maps its
// entering state by S -> M S + b, and the segments can run in parallel (DeltaNet-family digest,
// "Chunkwise Triton pipeline": the state pass is the only traversal between chunks).
//   STATE_CARRY  two CTA halves per (pair, segment but the last) carry X = [M | b] through the segment
//                from [I | 0]: half 0 the M columns (identity start, no KU), half 1 the b columns (zero
//                start); X is written to `carry` at the end.  No outputs.
//   STATE_OUT    the chunks from the state entering the segment, with the outputs; the last segment
//                writes S_T.  Unsplit (NS = 1) the entering state is S0; split, every segment reads it
//                from `carry`, where scan_chain_kernel left it (so S_T may alias S0 in both cases).
//
// Per chunk c, one tensor-core round trip is on the chain: the issuer issues D_S = G S_c (and, with outputs,
// D_O = Q' S_c into the buffer of c's parity) on the S operand of c; every thread waits for D_S and
// updates its part of the state, S_c+1 = e^{Gam_end} S_c - D_S + KU, writes the next S operand, and meets
// the others at one barrier.  The outputs of chunk c are read out in step c + 1, before the state warps
// wait for that step's D_S.
//
// The state operand is fp16(S_c 2^-sig_c).  sig_c comes from a bound on |S_c| that every thread computes
// alike, with no reduction on the chain: at the start the exact maximum, then
//   bound_c+1 = max e^{Gam_end} max|S_c| + 256 * 2^(14+eg) max|S_c| + 2 * 2^(14+eu),
// where |G| <= 2^(14+eg) and |KU| <= 2^(14+eu) (128 terms in G S; a factor 2 for the fp16 roundings) and
// max|S_c| is the exact CTA maximum, reduced one step late through per-warp slots.
template <int VB, int MODE>
__global__ void __launch_bounds__(STATE_THREADS, 1)
chunk_state_kernel(const unsigned char* __restrict__ rec_base, const float* __restrict__ S0, int T, int HV, int NC,
                   int L, int NS, bf16* __restrict__ o, float* __restrict__ S_T, float* __restrict__ carry,
                   unsigned int* __restrict__ status) {
    using Lay = StateLayout<VB, MODE>;
    constexpr bool OUTS = MODE == STATE_OUT;
    constexpr int NVB = VD / VB;
    constexpr int NH = OUTS ? 1 : 2;
    constexpr int HALF = VB / 2;
    constexpr int NBUF = Lay::NBUF;
    extern __shared__ __align__(1024) unsigned char smem[];
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar_rec0 = s_base + Lay::MBAR, bar_chain = bar_rec0 + 8 * NBUF, bar_out0 = bar_chain + 8;
    volatile unsigned int* sMaxS = reinterpret_cast<volatile unsigned int*>(smem + Lay::SMX);  // [2][8]
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
    const size_t v_row = (size_t)HV * VD;
    const unsigned char* rec0 = rec_base + (size_t)pair * NC * Rec::BYTES;
    auto rec = [&](int c) { return rec0 + (size_t)c * Rec::BYTES; };
    // carry slots of (pair, segment): [2][KD][VD] fp32, M then b
    auto carry_slot = [&](int sg, int hf) { return carry + (((size_t)pair * NS + sg) * 2 + hf) * KD * VD; };
    auto slot_of = [&](int c) { return (c - c_begin) % NBUF; };

    if (tid == 0) {
        for (int k = 0; k < NBUF + 3; ++k) mbar_init(bar_rec0 + 8 * k, 1);
    }
    if (warp == 0) tmem_alloc(s_base + Lay::TBASE, Lay::TMEM_COLS);
    cta_sync_tc();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + Lay::TBASE);

    // record copies in flight (bit k: slot k), for the bounded drain on abort; per-slot phases
    uint32_t pending = 0, ph_rec = 0;
    auto load_rec = [&](int c) {
        const int k = slot_of(c);
        const uint32_t bar = bar_rec0 + 8 * k, dst = s_base + Lay::slot(k);
        mbar_expect_tx(bar, Lay::WQ_LOAD + (use_u ? VB * 256u : 0u) + (OUTS ? VB * 256u : 0u) + Rec::VEC_LOAD);
        bulk_load(dst, rec(c) + Rec::WQ, Lay::WQ_LOAD, bar);
        if (use_u) bulk_load(dst + Lay::KU_OFF, rec(c) + Rec::KU + (vb0 / 16) * 4096, VB * 256, bar);
        if (OUTS) bulk_load(dst + Lay::AU_OFF, rec(c) + Rec::AU + (vb0 / 16) * 4096, VB * 256, bar);
        bulk_load(dst + Lay::VEC_OFF, rec(c) + Rec::VEC, Rec::VEC_LOAD, bar);
        pending |= 1u << k;
    };
    // this thread's part of the state slice: key row d, columns vb0 + c0 .. + HALF, exact fp32 (state warps)
    const bool issuer = tid == ISSUER, out_issuer = tid == OUT_ISSUER, state_warp = warp < STATE_WARPS;
    // the record copies come from the output issuer: its products are read out a step later, so a copy issued after the
    // barrier delays nothing on the chain
    const bool loader = tid == OUT_ISSUER;
    const int d = 32 * wq + lane;
    float s[HALF];
    {
        const float* src = nullptr;  // row-major [KD][VD] source of the entering state, or none (zeros)
        if (OUTS && state_warp) src = NS == 1 ? (S0 ? S0 + (size_t)pair * KD * VD : nullptr) : carry_slot(seg == 0 ? NS - 1 : seg - 1, seg == 0 ? 0 : 1);
#pragma unroll
        for (int j = 0; j < HALF; j += 4) {
            float4 x = src ? *reinterpret_cast<const float4*>(src + (size_t)d * VD + vb0 + c0 + j)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            if (!OUTS && half == 0 && state_warp) {  // identity: row d has its 1 in column d
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
    if (loader) {  // two chunks ahead
        load_rec(c_begin);
        if (c_begin + 1 < c_end) load_rec(c_begin + 1);
    }
    // this warp's largest |S| into slot `par`
    auto warp_max_s = [&](int par) {
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < HALF; ++j) m = fmaxf(m, fabsf(s[j]));
        m = warp_max_nonneg(m);
        if (lane == 0) sMaxS[8 * par + warp] = __float_as_uint(m);
    };
    auto cta_max_s = [&](int par) {
        float m = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) m = fmaxf(m, __uint_as_float(sMaxS[8 * par + w]));
        return m;
    };
    // fp16(S 2^-sig)^T into S operand `buf`: element (v, d) of the padded tiling; the 32 lanes (d) of a
    // warp store one column v into 16 different banks
    const uint32_t sop_thread = (uint32_t)(c0 >> 3) * Lay::SOP_SBO + (uint32_t)(d >> 3) * Lay::SOP_LBO + (uint32_t)(d & 7) * 2;
    auto write_sop = [&](int buf, int sig) {
        const float f = exp2i(-sig);
        unsigned char* sop = smem + Lay::SOP + buf * Lay::SOP_BYTES + sop_thread;
#pragma unroll
        for (int j = 0; j < HALF; ++j)
            *reinterpret_cast<uint16_t*>(sop + (j >> 3) * Lay::SOP_SBO + (j & 7) * 16) = to_f16_bits(s[j] * f);
    };
    // outputs of chunk c: an M = 64 product puts row i in lane 32 (i / 16) + i % 16, so lanes 0-15 of every
    // state warp read 16 rows (i = 16 wq + lane), O = Q' S_c 2^(eq + sig_c) + A U
    uint32_t ph_out = 0;
    auto outputs = [&](int c, float f_q) -> bool {
        const int par = (c - c_begin) & 1;
        const bool ok = mbar_wait(bar_out0 + 8 * par, (ph_out >> par) & 1u, WAIT_POLLS);
        fence_after_sync();
        if (!ok) return false;
        ph_out ^= 1u << par;
        const int i = 16 * wq + lane, n = lane < 16 ? min(CH, T - c * CH) : 0;
        const float* sAU = reinterpret_cast<const float*>(smem + Lay::slot(slot_of(c)) + Lay::AU_OFF);
        constexpr int SUB = HALF < 16 ? HALF : 16;
#pragma unroll
        for (int j0 = 0; j0 < HALF; j0 += SUB) {
            uint32_t r[SUB];
            tmem_ld_row<SUB>(taddr(tmem, 32 * wq, Lay::D_O + par * VB + c0 + j0), r);
            tmem_wait_ld();
            if (i < n) {
                bf16* op = o + ((size_t)b * T + (size_t)c * CH + i) * v_row + (size_t)hv * VD + vb0 + c0 + j0;
#pragma unroll
                for (int j = 0; j < SUB; j += 8) {
                    const int v = c0 + j0 + j;  // column within the block; AU by blocks of 16 columns
                    const float4 a0 = *reinterpret_cast<const float4*>(sAU + ((v >> 2) * 64 + i) * 4);
                    const float4 a1 = *reinterpret_cast<const float4*>(sAU + (((v >> 2) + 1) * 64 + i) * 4);
                    const float au[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                    uint32_t w[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        __nv_bfloat162 pr = __floats2bfloat162_rn(fmaf(__uint_as_float(r[j + 2 * t]), f_q, au[2 * t]),
                                                                  fmaf(__uint_as_float(r[j + 2 * t + 1]), f_q, au[2 * t + 1]));
                        w[t] = *reinterpret_cast<uint32_t*>(&pr);
                    }
                    *reinterpret_cast<uint4*>(op + j) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        return true;
    };
    uint32_t ph_chain = 0, out_commits = 0;
    int last_out_par = -1;
    bool aborted = false;
    if (state_warp) warp_max_s(0);
    __syncthreads();
    int sig = fp16_scale_exponent(cta_max_s(0));  // exact max |S| of the entering state
    float fq_prev = 0.f;      // output scale of the previous chunk
    if (state_warp) write_sop(0, sig);
    fence_proxy_async();
    cta_sync_tc();
    for (int c = c_begin; c < c_end && !aborted; ++c) {
        const int par = (c - c_begin) & 1, k = slot_of(c);
        const uint32_t sl = s_base + Lay::slot(k);
        const uint32_t sop = s_base + Lay::SOP + (Lay::NSOP == 2 ? par : 0) * Lay::SOP_BYTES;
        // ---- chain (and output) products on the S operand of chunk c ---------------------------------
        bool ok = mbar_wait(bar_rec0 + 8 * k, (ph_rec >> k) & 1u, WAIT_POLLS);
        ph_rec ^= 1u << k;
        if (loader && ok) pending &= ~(1u << k);
        // two issuing threads on different schedulers: an MMA takes a thread about 100 cycles to issue here, and
        // the chain's products should not queue behind the output's in one thread
        if (issuer && ok) {
            gemm_f16_bpad(tmem + Lay::D_S, sl, KD / 8 * 128, sop, Lay::SOP_LBO, Lay::SOP_SBO, idesc_f16(128, VB),
                          KD / 16, false);
            mma_commit(bar_chain);
        }
        if (OUTS && out_issuer && ok) {  // M = 64 on the Q' rows: row i of D_O = Q' S sits in TMEM lane 32 (i / 16) + i % 16
            gemm_f16_bpad(tmem + Lay::D_O + par * VB, sl + Rec::QP_OFF, KD / 8 * 128, sop, Lay::SOP_LBO, Lay::SOP_SBO,
                          idesc_f16(64, VB), KD / 16, false);
            mma_commit(bar_out0 + 8 * par);
            out_commits += 1u << (16 * par);  // commits per parity, for the drain on abort
            last_out_par = par;
        }
        fence_after_sync();
        const unsigned char* vec = smem + Lay::slot(k) + Lay::VEC_OFF;
        const float eg = reinterpret_cast<const float*>(vec)[d];
        const int* scl = reinterpret_cast<const int*>(vec + (Rec::SCL - Rec::VEC));
        const int e_g = scl[0], e_q = scl[1], e_u = scl[2];
        const float egmax = __int_as_float(scl[3]);
        // scales: this chunk's outputs (sig_c), and the bound on S_c+1 that sets sig_c+1 (max |S_c| exact)
        const float mS = cta_max_s(par);
        const float fq = exp2i(e_q) * exp2i(sig);
        const float f_g = exp2i(e_g) * exp2i(sig), f_u = exp2i(e_u);
        const int sig_next = fp16_scale_exponent(egmax * mS + 256.f * exp2i(14 + e_g) * mS +
                                                 (use_u ? 2.f * exp2i(14 + e_u) : 0.f));
        // ---- the previous chunk's outputs, while D_S runs -------------------------------------------
        if (OUTS && state_warp && c > c_begin) ok = outputs(c - 1, fq_prev) && ok;
        // ---- state: S = e^{Gam_end} S - G S + KU ------------------------------------------------------
        const unsigned char* sKU = smem + Lay::slot(k) + Lay::KU_OFF;
        constexpr int PIECE = HALF < 32 ? HALF : 32;
        uint4 ku_first[PIECE / 8];  // this thread's KU of the first piece, read while D_S runs
#pragma unroll
        for (int j = 0; j < PIECE; j += 8) {
            const int v = c0 + j;
            ku_first[j / 8] = use_u && state_warp ? *reinterpret_cast<const uint4*>(sKU + ((v >> 3) * KD + d) * 16)
                                                   : make_uint4(0u, 0u, 0u, 0u);
        }
        if (state_warp) ok = mbar_wait(bar_chain, ph_chain, WAIT_POLLS) && ok;
        ph_chain ^= 1u;
        fence_after_sync();
        if (ok && state_warp) {
#pragma unroll
            for (int j0 = 0; j0 < HALF; j0 += PIECE) {
                uint32_t r[PIECE];
                tmem_ld_row<PIECE>(taddr(tmem, 32 * wq, Lay::D_S + c0 + j0), r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < PIECE; j += 8) {
                    float ku[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (use_u) {
                        const int v = c0 + j0 + j;
                        const uint4 u4 = j0 == 0 ? ku_first[j / 8]
                                                 : *reinterpret_cast<const uint4*>(sKU + ((v >> 3) * KD + d) * 16);
                        f16x2_to_f32(u4.x, ku[0], ku[1]);
                        f16x2_to_f32(u4.y, ku[2], ku[3]);
                        f16x2_to_f32(u4.z, ku[4], ku[5]);
                        f16x2_to_f32(u4.w, ku[6], ku[7]);
                    }
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        s[j0 + j + t] = fmaf(ku[t], f_u, fmaf(eg, s[j0 + j + t], -__uint_as_float(r[j + t]) * f_g));
                }
            }
            // ---- the next chunk's S operand (its buffer is free: the products of chunk c - 1 that read it
            //      are complete, since D_S of chunk c completes after them); max |S_c+1| for the next bound --
            if (c + 1 < c_end) write_sop(Lay::NSOP == 2 ? par ^ 1 : 0, sig_next);
            warp_max_s(par ^ 1);
        }
        sig = sig_next;
        fence_proxy_async();
        fence_before_sync();
        if (!__syncthreads_and(ok)) { aborted = true; break; }
        fence_after_sync();
        if (loader && c + 2 < c_end) load_rec(c + 2);  // into the slot of chunk c - 1 (outputs) or c (no outputs)
        fq_prev = fq;
    }
    if (OUTS && !aborted && state_warp && c_end > c_begin) aborted = !outputs(c_end - 1, fq_prev);
    aborted = __syncthreads_or(aborted) != 0;

    if (aborted) {
        // bounded drain of copies and MMAs still in flight before shared memory and TMEM go away
        if (loader) {
            atomicOr(status, STATUS_TIMEOUT);
            for (int bb = 0; bb < NBUF; ++bb)
                if (pending & (1u << bb)) mbar_wait(bar_rec0 + 8 * bb, (ph_rec >> bb) & 1u, WAIT_POLLS);
        }
        if (issuer) mbar_wait(bar_chain, ph_chain, WAIT_POLLS);
        if (OUTS && out_issuer && last_out_par >= 0)  // the output products: their last commit tracks them all
            mbar_wait(bar_out0 + 8 * last_out_par, ((out_commits >> (16 * last_out_par)) - 1u) & 1u, WAIT_POLLS);
    } else if (state_warp) {
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
// a chain of NC steps per wave of (pair, value block) CTAs, T_UNSPLIT16 / T_UNSPLIT32 per step with 16 / 32
// columns (as launch_chunk_split picks the block width); the split one runs 4 x pairs x (NS - 1) carry
// CTAs (64 columns, T_CARRY per step), then 4 x pairs x NS output CTAs (32 columns), of L chunks each, in
// waves over the SMs, plus the segment chain at T_CHAIN per segment.  The split therefore pays only where
// the unsplit pass leaves SMs idle: few (sequence, head) pairs and long sequences.  The number of SMs is a
// planning constant (a B200's 148), so that the workspace size does not depend on the device; the split is
// taken where the model gains at least a fifth.
constexpr double T_UNSPLIT16 = 1.3, T_UNSPLIT32 = 1.4, T_CARRY = 1.5, T_CHAIN = 3.0;

ScanPlan chunk_scan_plan(long long pairs, int NC) {
    constexpr long long kPlanSMs = 148;
    const bool narrow = pairs * 8 <= kPlanSMs;
    const long long nvb = narrow ? 8 : 4;
    ScanPlan plan{NC, 1};
    double best = 0.8 * (double)NC * (narrow ? T_UNSPLIT16 : T_UNSPLIT32) *
                  (double)((pairs * nvb + kPlanSMs - 1) / kPlanSMs);
    for (int Lc : {8, 12, 16, 24, 32, 48, 64, 96, 128, 192, 256}) {
        if (Lc >= NC) break;
        const long long NS = (NC + Lc - 1) / Lc;
        const long long wa = (4 * pairs * (NS - 1) + kPlanSMs - 1) / kPlanSMs;
        const long long wc = (4 * pairs * NS + kPlanSMs - 1) / kPlanSMs;
        const double cost = (double)wa * Lc * T_CARRY + (double)wc * Lc * T_UNSPLIT32 + T_CHAIN * (double)NS;
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
    using L = StateLayout<VB, MODE>;
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
        // value-block width: 16 columns while the (pair, block) CTAs still fit on the SMs, else 32
        if (pairs * 8 <= nsm) return launch_state<16, STATE_OUT>(a, NC, plan, nullptr, true);
        return launch_state<32, STATE_OUT>(a, NC, plan, nullptr, true);
    }
    // long sequences: carry [M | b] through every segment, chain the segments, then the outputs
    float* carry = reinterpret_cast<float*>(static_cast<unsigned char*>(a.scratch) + (size_t)pairs * NC * Rec::BYTES);
    if ((e = launch_state<64, STATE_CARRY>(a, NC, plan, carry, true)) != cudaSuccess) return e;
    scan_chain_kernel<<<(unsigned)(pairs * (VD / CHAIN_COLS)), CHAIN_THREADS, 0, a.stream>>>(a.S0, carry, plan.NS);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_state<32, STATE_OUT>(a, NC, plan, carry, false);
}

}  // namespace kda
