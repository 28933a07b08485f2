// kda_chunk64.cuh -- pieces shared by the tensor-core prefill kernels for K = V = 128, chunk 64:
// sizes, the swizzled fp32 index of the in-chunk cumulative decay tile, bf16 unpacking, the
// CTA barrier with tcgen05 fences, and the in-place unit-lower-triangular inverse by doubling
// (DeltaNet-family digest, "Chunkwise KDA": T = (I + R)^{-1} for the in-chunk delta coupling R).
#pragma once
#include "kda_common.cuh"
#include "kda_tc_ptx.cuh"

namespace kda {
namespace c64 {
using namespace tc;

constexpr int INV_THREADS = 512;  // threads of the kernels that run the triangular inverse
constexpr int KD = 128;          // key dimension
constexpr int VD = 128;          // value dimension
constexpr int CH = 64;           // chunk length
constexpr int RP = 68;           // row pitch (floats) of the R / T scratch: 16-byte aligned rows
constexpr float SPAN_LIMIT = 40.0f;        // widest per-channel in-chunk log-decay span of the factorised path
constexpr uint32_t WAIT_POLLS = 1u << 26;  // polls before a bounded mbarrier wait gives up

__device__ __forceinline__ int gidx(int i, int d) { return i * KD + ((((d >> 2) ^ (i & 7)) << 2) | (d & 3)); }

__device__ __forceinline__ void cta_sync_tc() {
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 x = __bfloat1622float2(hp[t]);
        f[2 * t] = x.x;
        f[2 * t + 1] = x.y;
    }
}

// Gate values of one key channel for 16 consecutive rows as their running sum in registers.
template <int MODE>
__device__ __forceinline__ float gate_rows16_regs(const __nv_bfloat16* col, int stride, int nn, float bias, float rate,
                                                  float lower_bound, float (&gv)[16]) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float gr = __bfloat162float(col[r * stride]);
        gv[r] = (r < nn) ? gate_value_fast(gr, bias, rate, MODE, lower_bound) : 0.f;
    }
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        acc += gv[r];
        gv[r] = acc;
    }
    return acc;
}

// KDA_INPUT_L2NORM_QK: the sums of squares of this thread's two q / k operand units (8 channels of
// row i = 8 (u / 128) + u % 8, u = tid + 512 it) added into per-row totals.  Lanes that share a row
// differ in lane bits 3 and 4, so two shuffles sum four units and lanes 0-7 add them in shared memory
// (four warps per row).  The totals must start at zero and are complete after the next barrier.
__device__ __forceinline__ void add_row_sumsq(const uint4 (&qr)[2], const uint4 (&kr)[2], float* sSqQ, float* sSqK,
                                              int tid, int lane) {
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        float qf[8], kf[8];
        bf16x8_to_f32(qr[it], qf);
        bf16x8_to_f32(kr[it], kf);
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            sq = fmaf(qf[t], qf[t], sq);
            sk = fmaf(kf[t], kf[t], sk);
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 8);
        sk += __shfl_xor_sync(0xffffffffu, sk, 8);
        sq += __shfl_xor_sync(0xffffffffu, sq, 16);
        sk += __shfl_xor_sync(0xffffffffu, sk, 16);
        if (lane < 8) {
            const int u = tid + INV_THREADS * it;
            const int i = ((u >> 7) << 3) + (u & 7);
            atomicAdd(sSqQ + i, sq);
            atomicAdd(sSqK + i, sk);
        }
    }
}

// Divides 8 channels of one q row and one k row by their norms, given their sums of squares.
__device__ __forceinline__ void scale_row8(float (&qf)[8], float (&kf)[8], float sumsq_q, float sumsq_k) {
    const float iq = inv_l2norm(sumsq_q), ik = inv_l2norm(sumsq_k);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        qf[t] *= iq;
        kf[t] *= ik;
    }
}

__device__ __forceinline__ float bf16_bits_to_f32(unsigned short u) { return __uint_as_float((uint32_t)u << 16); }

// The doubling steps with blocks of 2, 4, 8 and 16 rows never cross a 16 x 16 diagonal block, so
// one warp can take one such block through all four with warp-level syncs only: warp w < 4 inverts
// the diagonal block at rows / columns 16 w .. 16 w + 15 (scratch: 64 floats of sX per warp).
template <int HS>
__device__ __forceinline__ void tri_inverse_diag16_step(float* sRT, float* sXw, int b16, int lane) {
    constexpr int CNT = 8 * HS;  // entries of the HS x HS lower-left blocks inside one 16 x 16 block
#pragma unroll
    for (int e = lane; e < CNT; e += 32) {  // X = C Ta
        const int c = e % HS, r = (e / HS) % HS, base = b16 + (e / (HS * HS)) * 2 * HS;
        const float* Crow = sRT + (base + HS + r) * RP + base;
        float acc = Crow[c];
#pragma unroll
        for (int m = 1; m < HS; ++m)
            if (m > c) acc += Crow[m] * sRT[(base + m) * RP + base + c];
        sXw[e] = acc;
    }
    __syncwarp();
#pragma unroll
    for (int e = lane; e < CNT; e += 32) {  // C <- -Td X
        const int c = e % HS, r = (e / HS) % HS, blk = e / (HS * HS), base = b16 + blk * 2 * HS;
        const float* Drow = sRT + (base + HS + r) * RP + base + HS;
        const float* Xb = sXw + blk * HS * HS;
        float acc = Xb[r * HS + c];
#pragma unroll
        for (int m = 0; m < HS - 1; ++m)
            if (m < r) acc += Drow[m] * Xb[m * HS + c];
        sRT[(base + HS + r) * RP + base + c] = -acc;
    }
    __syncwarp();
}

__device__ __forceinline__ void tri_inverse_diag16(float* sRT, float* sX, int tid) {
    const int w = tid >> 5, lane = tid & 31;
    if (w < 4) {
        float* sXw = sX + 64 * w;
        tri_inverse_diag16_step<1>(sRT, sXw, 16 * w, lane);
        tri_inverse_diag16_step<2>(sRT, sXw, 16 * w, lane);
        tri_inverse_diag16_step<4>(sRT, sXw, 16 * w, lane);
        tri_inverse_diag16_step<8>(sRT, sXw, 16 * w, lane);
    }
    __syncthreads();
}

// The last two doubling steps, for CTAs of INV_THREADS = 512 threads.  With T's strictly-lower
// part stored in place and its unit diagonal implicit, a block [[Ta, 0], [C, Td]] of the matrix being
// inverted, whose diagonal blocks Ta, Td are already inverted, becomes [[Ta, 0], [-Td C Ta, Td]]:
// first X = C Ta (the m = c term of Ta is the unit diagonal), then C <- -(X + Td' X) with Td' the
// strictly-lower part of Td.
// Step 16 -> 32 (two 32 x 32 blocks, at 0 and 32): thread (blk, r, c) = (tid / 256, (tid / 16) % 16,
// tid % 16) owns entry (r, c) of its block's 16 x 16 lower-left part.
__device__ __forceinline__ void tri_inverse_step16(float* sRT, float* sX, int tid) {
    const int blk = tid >> 8, r = (tid >> 4) & 15, c = tid & 15, base = 32 * blk;
    const float* Crow = sRT + (base + 16 + r) * RP + base;
    float acc = Crow[c];
#pragma unroll
    for (int m4 = 0; m4 < 16; m4 += 4) {
        const float4 cr = *reinterpret_cast<const float4*>(Crow + m4);
        const float cm[4] = {cr.x, cr.y, cr.z, cr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
            if (m4 + t > c) acc += cm[t] * sRT[(base + m4 + t) * RP + base + c];
    }
    float* Xb = sX + blk * 256;
    Xb[r * 16 + c] = acc;
    __syncthreads();
    const float* Drow = sRT + (base + 16 + r) * RP + base + 16;
    acc = Xb[r * 16 + c];
#pragma unroll
    for (int m4 = 0; m4 < 16; m4 += 4) {
        const float4 dr = *reinterpret_cast<const float4*>(Drow + m4);
        const float dm[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
            if (m4 + t < r) acc += dm[t] * Xb[(m4 + t) * 16 + c];
    }
    sRT[(base + 16 + r) * RP + base + c] = -acc;
    __syncthreads();
}

// Step 32 -> 64 (one 64 x 64 block): thread (r, c) = (tid / 16, tid % 16) owns entries (r, c) and
// (r, c + 16) of the 32 x 32 lower-left part.
__device__ __forceinline__ void tri_inverse_step32(float* sRT, float* sX, int tid) {
    const int r = tid >> 4, c = tid & 15;
    const float* Crow = sRT + (32 + r) * RP;
    float acc0 = Crow[c], acc1 = Crow[c + 16];
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        const float4 cr = *reinterpret_cast<const float4*>(Crow + m4);
        const float cm[4] = {cr.x, cr.y, cr.z, cr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int m = m4 + t;
            if (m > c) acc0 += cm[t] * sRT[m * RP + c];
            if (m4 >= 16 && m > c + 16) acc1 += cm[t] * sRT[m * RP + c + 16];
        }
    }
    sX[r * 32 + c] = acc0;
    sX[r * 32 + c + 16] = acc1;
    __syncthreads();
    const float* Drow = sRT + (32 + r) * RP + 32;
    acc0 = sX[r * 32 + c];
    acc1 = sX[r * 32 + c + 16];
    const int rmax = 2 * (tid >> 5) + 1;  // largest row of this warp: rows m < r <= rmax contribute
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        if (m4 >= rmax) break;  // warp-uniform
        const float4 dr = *reinterpret_cast<const float4*>(Drow + m4);
        const float dm[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int m = m4 + t;
            if (m < r) {
                acc0 += dm[t] * sX[m * 32 + c];
                acc1 += dm[t] * sX[m * 32 + c + 16];
            }
        }
    }
    sRT[(32 + r) * RP + c] = -acc0;
    sRT[(32 + r) * RP + c + 16] = -acc1;
    __syncthreads();
}

// The same last doubling step, writing its lower-left entries straight into Tb = T diag(beta), a [64][64]
// tf32 operand tile in the tiling of cm_off (tb: its shared-memory base), instead of back into sRT.  The
// other entries of Tb (the diagonal blocks, final after step 16 -> 32, and the zero upper-right block)
// are written by tb_outside_lower_left, before this; the caller's barrier completes Tb.
__device__ __forceinline__ void tri_inverse_step32_tb(const float* sRT, float* sX, int tid, const float* sBeta,
                                                      unsigned char* tb) {
    const int r = tid >> 4, c = tid & 15;
    const float* Crow = sRT + (32 + r) * RP;
    float acc0 = Crow[c], acc1 = Crow[c + 16];
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        const float4 cr = *reinterpret_cast<const float4*>(Crow + m4);
        const float cm[4] = {cr.x, cr.y, cr.z, cr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int m = m4 + t;
            if (m > c) acc0 += cm[t] * sRT[m * RP + c];
            if (m4 >= 16 && m > c + 16) acc1 += cm[t] * sRT[m * RP + c + 16];
        }
    }
    sX[r * 32 + c] = acc0;
    sX[r * 32 + c + 16] = acc1;
    __syncthreads();
    const float* Drow = sRT + (32 + r) * RP + 32;
    acc0 = sX[r * 32 + c];
    acc1 = sX[r * 32 + c + 16];
    const int rmax = 2 * (tid >> 5) + 1;  // largest row of this warp: rows m < r <= rmax contribute
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        if (m4 >= rmax) break;  // warp-uniform
        const float4 dr = *reinterpret_cast<const float4*>(Drow + m4);
        const float dm[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int m = m4 + t;
            if (m < r) {
                acc0 += dm[t] * sX[m * 32 + c];
                acc1 += dm[t] * sX[m * 32 + c + 16];
            }
        }
    }
    *reinterpret_cast<uint32_t*>(tb + tc::cm_off(32 + r, c, 64)) = to_tf32(-acc0 * sBeta[c]);
    *reinterpret_cast<uint32_t*>(tb + tc::cm_off(32 + r, c + 16, 64)) = to_tf32(-acc1 * sBeta[c + 16]);
}

// Tb entries outside the lower-left 32 x 32 block, from T after step 16 -> 32: the two diagonal blocks (strictly
// lower part from sRT, unit diagonal, zeros above) and the zero upper-right block.  Units of four columns.
__device__ __forceinline__ void tb_outside_lower_left(const float* sRT, int tid, const float* sBeta, unsigned char* tb) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int u = tid + INV_THREADS * x;
        const int i = ((u >> 7) << 3) + (u & 7), j4 = (u >> 3) & 15;
        if (i >= 32 && j4 < 8) continue;  // the lower-left block: step 32 -> 64 writes it
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if ((i >> 5) == (j4 >> 3)) {  // a diagonal block
            const float4 t4 = *reinterpret_cast<const float4*>(sRT + i * RP + 4 * j4);
            const float tr[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = 4 * j4 + t;
                w[t] = to_tf32(((j < i) ? tr[t] : (j == i ? 1.f : 0.f)) * sBeta[j]);
            }
        }
        *reinterpret_cast<uint4*>(tb + tc::cm_off(i, 4 * j4, 64)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace c64
}  // namespace kda
