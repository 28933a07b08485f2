// kda_mla.cu -- absorbed MLA decode: one query token per sequence against its cached latent vectors.
//
// KDA ledger, derivation DER2 ("MLA 矩阵吸收推导", claim C4): the query absorbs the key up-projection
// and meets the latent cache directly, so K and V are never decompressed:
//   1. q_abs = q . W_UK                   [B, H, r]      (W_UK [H, d_q, r])
//   2. score = q_abs . c^T                 [B, H, T]      (c [B, T, r], shared by every head)
//   3. o_lat = softmax(scale score) . c    [B, H, r]
//   4. o     = o_lat . W_UV^T              [B, H, d_v]    (W_UV [H, d_v, r])
// (the K3 MLA layer: global softmax attention without positional encoding).  Three kernels:
//   mla_qabs_kernel    step 1 with bf16 tensor-core MMAs; q_abs is kept as two bf16 terms, hi + lo, so that
//                      the tensor-core scores carry about 16 mantissa bits of it;
//   mla_attend_kernel  steps 2-3 with bf16 tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation):
//                      one CTA per (sequence, group of 48 heads, split of the positions) streams its
//                      latent tiles once through shared memory, with an online softmax;
//   mla_out_kernel     merges the splits and applies step 4 with bf16 MMAs on the hi + lo terms of o_lat.
// Every head reads the same latent vectors, so the CTA covers as many heads as its registers allow and
// the cache crosses HBM once per head group.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
using bf16 = __nv_bfloat16;

namespace {

constexpr int MLA_GH = 48;              // heads per CTA: three m16 tiles
constexpr int MLA_TP = 32;              // positions per latent tile
constexpr int MLA_WARPS = 12;           // (3 head tiles) x (4 position / value quarters)
constexpr int MLA_THREADS = 32 * MLA_WARPS;

template <int R>
struct MlaSmem {
    static constexpr int PITCH = R + 8;  // bf16 elements per row: conflict-free fragment loads
    static constexpr int PP = MLA_TP + 8;
    static constexpr size_t QA = 0;                                      // hi, lo: [48][PITCH] bf16 each
    static constexpr size_t CT = QA + 2 * (size_t)MLA_GH * PITCH * 2;    // latent tiles: 2 x [32][PITCH] bf16
    static constexpr size_t PB = CT + 2 * (size_t)MLA_TP * PITCH * 2;    // probabilities: 2 x [48][PP] bf16
    static constexpr int SPP = MLA_TP + 8;                                // score partial row pitch (floats)
    static constexpr size_t SP = PB + 2 * (size_t)MLA_GH * PP * 2;       // score partials: [4][48][SPP] fp32
    static constexpr size_t ST = SP + 4 * (size_t)MLA_GH * SPP * 4;      // row statistics (floats)
    // ST: max partials 2 x [4][48], sum partials 2 x [4][48], running max 2 x [48], running sum [48]
    static constexpr size_t BYTES = ST + (2 * 4 * MLA_GH + 2 * 4 * MLA_GH + 2 * MLA_GH + MLA_GH) * 4;
    static_assert(BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t ld_u32(const bf16* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices, lane l giving the address of row l % 8 of matrix l / 8; thread t receives
// (row t / 4, columns 2 (t % 4) and 2 (t % 4) + 1) of each matrix.
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Two 8x8 b16 matrices from rows k0 .. k0 + 15 of a row-major [K][N] shared tile (lanes 0-15 give the
// row addresses), transposed into the B fragment of an m16n8k16 MMA.
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& b0, uint32_t& b1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n" : "=r"(b0), "=r"(b1) : "r"(addr));
}

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool ok) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(ok ? 16u : 0u) : "memory");
}

}  // namespace

// ---- step 1: q_abs = q W_UK per head, as bf16 hi + lo ------------------------------------------
// Grid (H, ceil(B / 32)), 256 threads.  q (32 sequences x DQ) and W_UK[h] (DQ x R) go to shared memory by
// 16-byte cp.async; the product runs on bf16 MMAs (m16n8k16, fp32 accumulation; both operands are bf16,
// so the sums are those of the CUDA-core product up to their order).  Warp w: sequences 16 (w % 2) ..,
// latent columns (w / 2) R / 4 ..; W_UK's rows are k, so its B fragments come from transposing loads.
constexpr int QABS_B = 32;
constexpr int PROJ_THREADS = 256;

template <int DQ, int R>
struct QabsSmem {
    static constexpr int PQ = DQ + 8, PW = R + 8;  // row pitches (bf16): conflict-free fragment loads
    static constexpr size_t SQ = 0, SW = SQ + (size_t)QABS_B * PQ * 2;
    static constexpr size_t BYTES = SW + (size_t)DQ * PW * 2;
    static_assert(BYTES <= 232448, "shared memory budget");
};

template <int DQ, int R>
__global__ void __launch_bounds__(PROJ_THREADS)
mla_qabs_kernel(const bf16* __restrict__ q, const bf16* __restrict__ W_UK, int B, int H, bf16* __restrict__ qa_hi,
                bf16* __restrict__ qa_lo) {
    using Sm = QabsSmem<DQ, R>;
    constexpr int PQ = Sm::PQ, PW = Sm::PW, NT8 = R / 4 / 8;  // n8 tiles per warp
    extern __shared__ __align__(16) unsigned char qsm[];
    const uint32_t sq = (uint32_t)__cvta_generic_to_shared(qsm + Sm::SQ), sw = (uint32_t)__cvta_generic_to_shared(qsm + Sm::SW);
    const int h = blockIdx.x, b0 = blockIdx.y * QABS_B, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < QABS_B * (DQ / 8); i += PROJ_THREADS) {  // rows past B read as zeros
        const int bb = i / (DQ / 8), ch = i - bb * (DQ / 8);
        const bool ok = b0 + bb < B;
        cp_async16_zfill(sq + (uint32_t)((bb * PQ + 8 * ch) * 2),
                         ok ? (const void*)(q + ((size_t)(b0 + bb) * H + h) * DQ + 8 * ch) : (const void*)q, ok);
    }
    const bf16* w = W_UK + (size_t)h * DQ * R;
    for (int i = tid; i < DQ * (R / 8); i += PROJ_THREADS) {
        const int d = i / (R / 8), ch = i - d * (R / 8);
        cp_async16_zfill(sw + (uint32_t)((d * PW + 8 * ch) * 2), w + (size_t)d * R + 8 * ch, true);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    const int mt = warp & 1, n0 = (warp >> 1) * (R / 4), g = lane >> 2, t4 = lane & 3;
    float acc[NT8][4];
#pragma unroll
    for (int j = 0; j < NT8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const uint32_t a_off = (uint32_t)(((16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1)) * PQ + 8 * (lane >> 4)) * 2);
    const uint32_t b_off = (uint32_t)(((lane & 15) * PW + n0) * 2);  // rows k0 + (lane % 16) of [k][n]
#pragma unroll
    for (int k = 0; k < DQ; k += 16) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(a0, a1, a2, a3, sq + a_off + (uint32_t)(k * 2));
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
            uint32_t b0f, b1f;
            ldmatrix_x2_trans(b0f, b1f, sw + b_off + (uint32_t)((k * PW + 8 * j) * 2));
            mma_bf16(acc[j], a0, a1, a2, a3, b0f, b1f);
        }
    }
    // D fragment: rows 16 mt + g (+ 8), columns n0 + 8 j + 2 t4 (+ 1)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int b = b0 + 16 * mt + g + 8 * half;
        if (b >= B) continue;
        const size_t row = ((size_t)b * H + h) * R;
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
            const float x0 = acc[j][2 * half], x1 = acc[j][2 * half + 1];
            const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
            const float2 hf = __bfloat1622float2(hi);
            const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
            const int col = n0 + 8 * j + 2 * t4;
            *reinterpret_cast<__nv_bfloat162*>(qa_hi + row + col) = hi;
            *reinterpret_cast<__nv_bfloat162*>(qa_lo + row + col) = lo;
        }
    }
}

// ---- steps 2-3: scores, online softmax, weighted latent sum -------------------------------------
// Grid (B, ceil(H / 48), NSPLIT).  Warp w: head tile m = w / 4 (16 heads) and quarter w % 4.  For the scores
// the quarter is a quarter of the latent columns: the warp computes partial scores of its 16 heads for all
// 32 positions of the tile (four independent accumulators; every q_abs fragment is read from shared memory
// once per tile), and the four partials meet in shared memory.  For the softmax the quarter is 8 positions,
// for the weighted sum it is a quarter of the latent columns again.  Writes the unnormalised o_lat, the
// running max and the running sum of its split to the workspace.
template <int R>
__global__ void __launch_bounds__(MLA_THREADS, 1)
mla_attend_kernel(const bf16* __restrict__ qa_hi, const bf16* __restrict__ qa_lo, const bf16* __restrict__ c,
                  const int* __restrict__ lengths, int T, int H, int nsplit, int split_len, float scale_log2,
                  float* __restrict__ part_o, float* __restrict__ part_ml) {
    using Sm = MlaSmem<R>;
    constexpr int P = Sm::PITCH, PP = Sm::PP, SPP = Sm::SPP;
    constexpr int NC = R / 4;       // latent columns per warp in the weighted sum
    constexpr int NT8 = NC / 8;     // n8 tiles per warp
    extern __shared__ __align__(16) unsigned char msm[];
    bf16* sQh = reinterpret_cast<bf16*>(msm + Sm::QA);
    bf16* sQl = sQh + MLA_GH * P;
    bf16* sC = reinterpret_cast<bf16*>(msm + Sm::CT);
    bf16* sP = reinterpret_cast<bf16*>(msm + Sm::PB);
    float* sSP = reinterpret_cast<float*>(msm + Sm::SP);    // [4][48][SPP] partial scores
    float* sMaxP = reinterpret_cast<float*>(msm + Sm::ST);  // 2 x [4][48]
    float* sSumP = sMaxP + 2 * 4 * MLA_GH;                   // 2 x [4][48]
    float* sM = sSumP + 2 * 4 * MLA_GH;                      // 2 x [48]
    float* sL = sM + 2 * MLA_GH;                             // [48]

    const int b = blockIdx.x, hg = blockIdx.y, split = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m = warp >> 2, quarter = warp & 3;
    const int g = lane >> 2, t4 = lane & 3;
    const int len = lengths ? min(max(lengths[b], 0), T) : T;
    const int p0 = split * split_len, p1 = min(len, p0 + split_len);
    const int ntiles = p1 > p0 ? (p1 - p0 + MLA_TP - 1) / MLA_TP : 0;
    const uint32_t c_base = (uint32_t)__cvta_generic_to_shared(sC);

    // q_abs of this head group (rows past H are zero)
    for (int i = tid; i < MLA_GH * (R / 8); i += MLA_THREADS) {
        const int row = i / (R / 8), ch = i - row * (R / 8);
        const int h = hg * MLA_GH + row;
        uint4 vh = make_uint4(0u, 0u, 0u, 0u), vl = vh;
        if (h < H) {
            vh = *reinterpret_cast<const uint4*>(qa_hi + ((size_t)b * H + h) * R + 8 * ch);
            vl = *reinterpret_cast<const uint4*>(qa_lo + ((size_t)b * H + h) * R + 8 * ch);
        }
        *reinterpret_cast<uint4*>(sQh + row * P + 8 * ch) = vh;
        *reinterpret_cast<uint4*>(sQl + row * P + 8 * ch) = vl;
    }
    if (tid < MLA_GH) {
        sM[tid] = -INFINITY;
        sM[MLA_GH + tid] = -INFINITY;
        sL[tid] = 0.f;
    }
    auto load_tile = [&](int tile, int buf) {  // positions past len read as zeros (masked below)
        const int pos0 = p0 + tile * MLA_TP;
        for (int i = tid; i < MLA_TP * (R / 8); i += MLA_THREADS) {
            const int row = i / (R / 8), ch = i - row * (R / 8);
            const int pos = pos0 + row;
            const bool ok = pos < p1;
            cp_async16_zfill(c_base + (uint32_t)(((buf * MLA_TP + row) * P + 8 * ch) * 2),
                             ok ? (const void*)(c + ((size_t)b * T + pos) * R + 8 * ch) : (const void*)c, ok);
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    if (ntiles > 0) load_tile(0, 0);

    float acc[NT8][4];
#pragma unroll
    for (int j = 0; j < NT8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    for (int tile = 0; tile < ntiles; ++tile) {
        const int buf = tile & 1, par = tile & 1;
        // the next tile streams into the other buffer (the previous tile's, released by the barrier that
        // ended the previous iteration) while this one is computed
        if (tile + 1 < ntiles) {
            load_tile(tile + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;\n" ::: "memory");
        }
        __syncthreads();  // this tile has landed for every thread
        // ---- partial scores: 16 heads x 32 positions over this warp's quarter of the latent columns,
        //      (q_hi + q_lo) . c with bf16 MMAs ----------------------------------------------------------
        {
            float sp[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) sp[j][0] = sp[j][1] = sp[j][2] = sp[j][3] = 0.f;
            const uint32_t qh_base = (uint32_t)__cvta_generic_to_shared(sQh), ql_base = (uint32_t)__cvta_generic_to_shared(sQl);
            const uint32_t ct_base = c_base + (uint32_t)(buf * MLA_TP * P * 2);
            // A fragment addresses: lane l -> row 16 m + (l % 8) + 8 ((l / 8) % 2), column + 8 (l / 16)
            const uint32_t a_off = (uint32_t)(((16 * m + (lane & 7) + 8 * ((lane >> 3) & 1)) * P + 8 * (lane >> 4)) * 2);
            // B fragment addresses: lane l -> position 8 j + (l % 8), column + 8 (l / 8) (two k16 steps per load)
            const uint32_t b_off = (uint32_t)(((lane & 7) * P + 8 * (lane >> 3)) * 2);
            const int k_begin = quarter * (R / 4);
#pragma unroll
            for (int k = k_begin; k < k_begin + R / 4; k += 32) {
                uint32_t ah[2][4], al[2][4];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    ldmatrix_x4(ah[h2][0], ah[h2][1], ah[h2][2], ah[h2][3], qh_base + a_off + (uint32_t)((k + 16 * h2) * 2));
                    ldmatrix_x4(al[h2][0], al[h2][1], al[h2][2], al[h2][3], ql_base + a_off + (uint32_t)((k + 16 * h2) * 2));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t b[4];
                    ldmatrix_x4(b[0], b[1], b[2], b[3], ct_base + b_off + (uint32_t)((8 * j * P + k) * 2));
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        mma_bf16(sp[j], ah[h2][0], ah[h2][1], ah[h2][2], ah[h2][3], b[2 * h2], b[2 * h2 + 1]);
                        mma_bf16(sp[j], al[h2][0], al[h2][1], al[h2][2], al[h2][3], b[2 * h2], b[2 * h2 + 1]);
                    }
                }
            }
            float* dst = sSP + (size_t)quarter * MLA_GH * SPP;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                *reinterpret_cast<float2*>(dst + (16 * m + g) * SPP + 8 * j + 2 * t4) = make_float2(sp[j][0], sp[j][1]);
                *reinterpret_cast<float2*>(dst + (16 * m + g + 8) * SPP + 8 * j + 2 * t4) = make_float2(sp[j][2], sp[j][3]);
            }
        }
        __syncthreads();
        // the scores of 16 heads x this warp's 8 positions: the four partials summed
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
            const float* src = sSP + (size_t)kq * MLA_GH * SPP;
            const float2 x0 = *reinterpret_cast<const float2*>(src + (16 * m + g) * SPP + 8 * quarter + 2 * t4);
            const float2 x1 = *reinterpret_cast<const float2*>(src + (16 * m + g + 8) * SPP + 8 * quarter + 2 * t4);
            s[0] += x0.x;
            s[1] += x0.y;
            s[2] += x1.x;
            s[3] += x1.y;
        }
        // scale into the log2 domain, mask positions past the split's end
        const int posc = p0 + tile * MLA_TP + 8 * quarter + 2 * t4;
        const bool v0 = posc < p1, v1 = posc + 1 < p1;
        s[0] = v0 ? s[0] * scale_log2 : -INFINITY;
        s[1] = v1 ? s[1] * scale_log2 : -INFINITY;
        s[2] = v0 ? s[2] * scale_log2 : -INFINITY;
        s[3] = v1 ? s[3] * scale_log2 : -INFINITY;
        // row maxima over this warp's 8 positions (rows g and g + 8 of the head tile)
        float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const int r0 = 16 * m + g, r1 = r0 + 8;
        float* maxp = sMaxP + par * 4 * MLA_GH;
        float* sump = sSumP + par * 4 * MLA_GH;
        if (t4 == 0) {
            maxp[quarter * MLA_GH + r0] = mx0;
            maxp[quarter * MLA_GH + r1] = mx1;
        }
        __syncthreads();
        // new running maxima (every warp computes the same values), probabilities to shared memory
        const float* mold = sM + par * MLA_GH;
        auto new_max = [&](int r) {
            return fmaxf(mold[r], fmaxf(fmaxf(maxp[r], maxp[MLA_GH + r]), fmaxf(maxp[2 * MLA_GH + r], maxp[3 * MLA_GH + r])));
        };
        const float mn0 = new_max(r0), mn1 = new_max(r1);
        const float e0 = exp2f(s[0] - mn0), e1 = exp2f(s[1] - mn0), e2 = exp2f(s[2] - mn1), e3 = exp2f(s[3] - mn1);
        bf16* Pt = sP + par * MLA_GH * PP;
        *reinterpret_cast<__nv_bfloat162*>(Pt + r0 * PP + 8 * quarter + 2 * t4) = __floats2bfloat162_rn(e0, e1);
        *reinterpret_cast<__nv_bfloat162*>(Pt + r1 * PP + 8 * quarter + 2 * t4) = __floats2bfloat162_rn(e2, e3);
        float sm0 = e0 + e1, sm1 = e2 + e3;
        sm0 += __shfl_xor_sync(0xffffffffu, sm0, 1);
        sm0 += __shfl_xor_sync(0xffffffffu, sm0, 2);
        sm1 += __shfl_xor_sync(0xffffffffu, sm1, 1);
        sm1 += __shfl_xor_sync(0xffffffffu, sm1, 2);
        if (t4 == 0) {
            sump[quarter * MLA_GH + r0] = sm0;
            sump[quarter * MLA_GH + r1] = sm1;
        }
        __syncthreads();
        // ---- rescale the accumulators and add P . c for this warp's latent columns -----------------
        const float a0 = exp2f(mold[r0] - mn0), a1 = exp2f(mold[r1] - mn1);
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
            acc[j][0] *= a0;
            acc[j][1] *= a0;
            acc[j][2] *= a1;
            acc[j][3] *= a1;
        }
        if (quarter == 0 && t4 == 0) {  // running sums and maxima for the next tile (other parity)
            sL[r0] = a0 * sL[r0] + sump[r0] + sump[MLA_GH + r0] + sump[2 * MLA_GH + r0] + sump[3 * MLA_GH + r0];
            sL[r1] = a1 * sL[r1] + sump[r1] + sump[MLA_GH + r1] + sump[2 * MLA_GH + r1] + sump[3 * MLA_GH + r1];
            sM[(par ^ 1) * MLA_GH + r0] = mn0;
            sM[(par ^ 1) * MLA_GH + r1] = mn1;
        }
        const bf16* pa = Pt + (16 * m) * PP;
#pragma unroll
        for (int kk = 0; kk < MLA_TP; kk += 16) {
            const uint32_t a_0 = ld_u32(pa + g * PP + kk + 2 * t4), a_1 = ld_u32(pa + (g + 8) * PP + kk + 2 * t4);
            const uint32_t a_2 = ld_u32(pa + g * PP + kk + 2 * t4 + 8), a_3 = ld_u32(pa + (g + 8) * PP + kk + 2 * t4 + 8);
            // lanes 0-15 address rows kk .. kk + 15 of the latent tile at this warp's column block
            const int lrow = kk + (lane & 15);
#pragma unroll
            for (int j = 0; j < NT8; ++j) {
                uint32_t b0, b1;
                const uint32_t addr = c_base + (uint32_t)(((buf * MLA_TP + lrow) * P + NC * quarter + 8 * j) * 2);
                ldmatrix_x2_trans(b0, b1, addr);
                mma_bf16(acc[j], a_0, a_1, a_2, a_3, b0, b1);
            }
        }
        __syncthreads();  // every warp is done with this tile's buffers before they are refilled
    }
    // ---- this split's unnormalised o_lat, running max (log2 domain) and sum ---------------------------
    const int par_end = ntiles & 1;
#pragma unroll
    for (int j = 0; j < NT8; ++j) {
        const int col = NC * quarter + 8 * j + 2 * t4;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int row = 16 * m + g + 8 * half, h = hg * MLA_GH + row;
            if (h >= H) continue;
            float* dst = part_o + (((size_t)blockIdx.x * nsplit + split) * H + h) * R + col;
            *reinterpret_cast<float2*>(dst) = make_float2(acc[j][2 * half], acc[j][2 * half + 1]);
        }
    }
    if (tid < MLA_GH) {
        const int h = hg * MLA_GH + tid;
        if (h < H) {
            float* ml = part_ml + (((size_t)blockIdx.x * nsplit + split) * H + h) * 2;
            ml[0] = sM[par_end * MLA_GH + tid];
            ml[1] = sL[tid];
        }
    }
}

// ---- merge the splits and step 4: o = (o_lat / l) W_UV^T ---------------------------------------
// Grid (H, ceil(B / 32)), 256 threads.  The merged o_lat of 32 sequences is split into bf16 hi + lo terms
// (about 16 mantissa bits) in shared memory; W_UV[h] (DV x R, rows v, k contiguous) arrives by 16-byte
// cp.async while the merge runs.  o = (hi + lo) W_UV^T on bf16 MMAs (m16n8k16, fp32 accumulation).
// Warp w: sequences 16 (w % 2) .., value columns (w / 2) DV / 4 ...
constexpr int OUT_B = 32;

template <int DV, int R>
struct MlaOutSmem {
    static constexpr int PA = R + 8;  // row pitch (bf16) of the o_lat terms and of W_UV
    static constexpr size_t SH = 0, SL = SH + (size_t)OUT_B * PA * 2, SW = SL + (size_t)OUT_B * PA * 2;
    static constexpr size_t BYTES = SW + (size_t)DV * PA * 2;
    static_assert(BYTES <= 232448, "shared memory budget");
};

template <int DV, int R>
__global__ void __launch_bounds__(PROJ_THREADS)
mla_out_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, const bf16* __restrict__ W_UV,
               int B, int H, int nsplit, bf16* __restrict__ o) {
    using Sm = MlaOutSmem<DV, R>;
    constexpr int PA = Sm::PA, NT8 = DV / 4 / 8;  // n8 tiles per warp
    extern __shared__ __align__(16) unsigned char osm[];
    bf16* sH = reinterpret_cast<bf16*>(osm + Sm::SH);
    bf16* sL = reinterpret_cast<bf16*>(osm + Sm::SL);
    const uint32_t sh = (uint32_t)__cvta_generic_to_shared(sH), sl = (uint32_t)__cvta_generic_to_shared(sL);
    const uint32_t sw = (uint32_t)__cvta_generic_to_shared(osm + Sm::SW);
    const int h = blockIdx.x, b0 = blockIdx.y * OUT_B, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bf16* w = W_UV + (size_t)h * DV * R;
    for (int i = tid; i < DV * (R / 8); i += PROJ_THREADS) {
        const int v = i / (R / 8), ch = i - v * (R / 8);
        cp_async16_zfill(sw + (uint32_t)((v * PA + 8 * ch) * 2), w + (size_t)v * R + 8 * ch, true);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    // merge: o_lat = sum_s 2^{m_s - M} o_s / sum_s 2^{m_s - M} l_s, four columns per item
    for (int i = tid; i < OUT_B * (R / 4); i += PROJ_THREADS) {
        const int bb = i / (R / 4), col = 4 * (i - bb * (R / 4)), b = b0 + bb;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (b < B) {
            float M = -INFINITY;
            for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, part_ml[(((size_t)b * nsplit + sp) * H + h) * 2]);
            float den = 0.f;
            for (int sp = 0; sp < nsplit; ++sp) {
                const float* ml = part_ml + (((size_t)b * nsplit + sp) * H + h) * 2;
                if (ml[0] == -INFINITY) continue;  // an empty split
                const float wt = exp2f(ml[0] - M);
                const float4 x = *reinterpret_cast<const float4*>(part_o + (((size_t)b * nsplit + sp) * H + h) * R + col);
                val.x += wt * x.x;
                val.y += wt * x.y;
                val.z += wt * x.z;
                val.w += wt * x.w;
                den += wt * ml[1];
            }
            const float inv = 1.f / den;
            val = make_float4(val.x * inv, val.y * inv, val.z * inv, val.w * inv);
        }
        const __nv_bfloat162 h01 = __floats2bfloat162_rn(val.x, val.y), h23 = __floats2bfloat162_rn(val.z, val.w);
        const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
        const __nv_bfloat162 l01 = __floats2bfloat162_rn(val.x - f01.x, val.y - f01.y);
        const __nv_bfloat162 l23 = __floats2bfloat162_rn(val.z - f23.x, val.w - f23.y);
        *reinterpret_cast<uint2*>(sH + bb * PA + col) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
        *reinterpret_cast<uint2*>(sL + bb * PA + col) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    const int mt = warp & 1, n0 = (warp >> 1) * (DV / 4), g = lane >> 2, t4 = lane & 3;
    float acc[NT8][4];
#pragma unroll
    for (int j = 0; j < NT8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const uint32_t a_off = (uint32_t)(((16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1)) * PA + 8 * (lane >> 4)) * 2);
    // B fragment addresses: lane l -> row (value column) n0 + 8 j + (l % 8), column k + 8 (l / 8): two k16 steps
    const uint32_t b_off = (uint32_t)(((n0 + (lane & 7)) * PA + 8 * (lane >> 3)) * 2);
#pragma unroll 2
    for (int k = 0; k < R; k += 32) {
        uint32_t ah[2][4], al[2][4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            ldmatrix_x4(ah[h2][0], ah[h2][1], ah[h2][2], ah[h2][3], sh + a_off + (uint32_t)((k + 16 * h2) * 2));
            ldmatrix_x4(al[h2][0], al[h2][1], al[h2][2], al[h2][3], sl + a_off + (uint32_t)((k + 16 * h2) * 2));
        }
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
            uint32_t bf[4];
            ldmatrix_x4(bf[0], bf[1], bf[2], bf[3], sw + b_off + (uint32_t)((8 * j * PA + k) * 2));
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                mma_bf16(acc[j], ah[h2][0], ah[h2][1], ah[h2][2], ah[h2][3], bf[2 * h2], bf[2 * h2 + 1]);
                mma_bf16(acc[j], al[h2][0], al[h2][1], al[h2][2], al[h2][3], bf[2 * h2], bf[2 * h2 + 1]);
            }
        }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int b = b0 + 16 * mt + g + 8 * half;
        if (b >= B) continue;
#pragma unroll
        for (int j = 0; j < NT8; ++j)
            *reinterpret_cast<__nv_bfloat162*>(o + ((size_t)b * H + h) * DV + n0 + 8 * j + 2 * t4) =
                __floats2bfloat162_rn(acc[j][2 * half], acc[j][2 * half + 1]);
    }
}

// ---------------------------------------------------------------------------------------------
int mla_nsplit(int B, int T, int H) {
    // as many (sequence, head group, split) CTAs as a B200 has SMs at most (one wave of one CTA per SM),
    // splits of at least 256 positions
    const long long groups = (long long)B * ((H + MLA_GH - 1) / MLA_GH);
    int ns = (int)(148 / groups);
    const int maxs = (T + 255) / 256;
    if (ns > maxs) ns = maxs;
    return ns < 1 ? 1 : ns;
}

size_t mla_workspace(int B, int T, int H, int R) {
    const int ns = mla_nsplit(B, T, H);
    return 2 * (size_t)B * H * R * sizeof(bf16) + (size_t)B * ns * H * R * sizeof(float) +
           (size_t)B * ns * H * 2 * sizeof(float);
}

namespace {
template <int DQ, int DV, int R>
cudaError_t launch_mla_t(const MlaArgs& a) {
    const int ns = mla_nsplit(a.B, a.T, a.H);
    const int split_len = (a.T + ns - 1) / ns;
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    bf16* qa_hi = reinterpret_cast<bf16*>(ws);
    bf16* qa_lo = qa_hi + (size_t)a.B * a.H * R;
    float* part_o = reinterpret_cast<float*>(qa_lo + (size_t)a.B * a.H * R);
    float* part_ml = part_o + (size_t)a.B * ns * a.H * R;
    const bf16* q = static_cast<const bf16*>(a.q);
    using QSm = QabsSmem<DQ, R>;
    cudaError_t e = cudaFuncSetAttribute(mla_qabs_kernel<DQ, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QSm::BYTES);
    if (e != cudaSuccess) return e;
    mla_qabs_kernel<DQ, R><<<dim3(a.H, (a.B + QABS_B - 1) / QABS_B), PROJ_THREADS, QSm::BYTES, a.stream>>>(
        q, static_cast<const bf16*>(a.W_UK), a.B, a.H, qa_hi, qa_lo);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using Sm = MlaSmem<R>;
    e = cudaFuncSetAttribute(mla_attend_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sm::BYTES);
    if (e != cudaSuccess) return e;
    const float scale_log2 = a.scale * 1.4426950408889634f;  // softmax with exp2: scores times log2(e)
    mla_attend_kernel<R><<<dim3(a.B, (a.H + MLA_GH - 1) / MLA_GH, ns), MLA_THREADS, Sm::BYTES, a.stream>>>(
        qa_hi, qa_lo, static_cast<const bf16*>(a.c), a.lengths, a.T, a.H, ns, split_len, scale_log2, part_o, part_ml);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using OSm = MlaOutSmem<DV, R>;
    e = cudaFuncSetAttribute(mla_out_kernel<DV, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OSm::BYTES);
    if (e != cudaSuccess) return e;
    mla_out_kernel<DV, R><<<dim3(a.H, (a.B + OUT_B - 1) / OUT_B), PROJ_THREADS, OSm::BYTES, a.stream>>>(
        part_o, part_ml, static_cast<const bf16*>(a.W_UV), a.B, a.H, ns, static_cast<bf16*>(a.o));
    return cudaGetLastError();
}

template <int DQ, int DV>
cudaError_t mla_r(const MlaArgs& a) {
    switch (a.R) {
        case 128: return launch_mla_t<DQ, DV, 128>(a);
        case 256: return launch_mla_t<DQ, DV, 256>(a);
        case 512: return launch_mla_t<DQ, DV, 512>(a);
    }
    return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_mla_decode(const MlaArgs& a) {
    if (a.d_q == 64 && a.d_v == 64) return mla_r<64, 64>(a);
    if (a.d_q == 128 && a.d_v == 128) return mla_r<128, 128>(a);
    if (a.d_q == 64 && a.d_v == 128) return mla_r<64, 128>(a);
    if (a.d_q == 128 && a.d_v == 64) return mla_r<128, 64>(a);
    return cudaErrorInvalidValue;
}

}  // namespace kda
