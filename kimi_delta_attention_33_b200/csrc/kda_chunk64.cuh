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

constexpr int TC_THREADS = 256;  // threads of the kernels that run the triangular inverse
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

// The same for 16 rows (CTAs with four threads per key channel).
template <int MODE, typename Idx>
__device__ __forceinline__ float gate_rows16_to(const __nv_bfloat16* col, int stride, int nn, float bias, float rate,
                                                float lower_bound, float* dst, Idx idx) {
    float acc = 0.f;
#pragma unroll
    for (int r0 = 0; r0 < 16; r0 += 8) {
        float x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const float gr = __bfloat162float(col[(r0 + r) * stride]);
            x[r] = (r0 + r < nn) ? gate_value_fast(gr, bias, rate, MODE, lower_bound) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            acc += x[r];
            dst[idx(r0 + r)] = acc;
        }
    }
    return acc;
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

__device__ __forceinline__ float gate_rows16_regs(int mode, const __nv_bfloat16* col, int stride, int nn, float bias,
                                                  float rate, float lower_bound, float (&gv)[16]) {
    if (mode == KDA_GATE_SAFE) return gate_rows16_regs<KDA_GATE_SAFE>(col, stride, nn, bias, rate, lower_bound, gv);
    if (mode == KDA_GATE_STANDARD)
        return gate_rows16_regs<KDA_GATE_STANDARD>(col, stride, nn, bias, rate, lower_bound, gv);
    return gate_rows16_regs<KDA_GATE_NONE>(col, stride, nn, bias, rate, lower_bound, gv);
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

// The last two doubling steps with one column per lane and four rows per thread: X = C Ta and the
// new block -Td X, accumulating over m with loads of four consecutive row entries at a time.
// Step 16 -> 32 (two blocks, at 0 and 32): warp w serves block w / 4 and rows 4 (w % 4) .. + 3 of its
// 16 x 16 lower-left block; lane = column (lane % 16) and row pair (lane / 16).
__device__ __forceinline__ void tri_inverse_step16(float* sRT, float* sX, int tid) {
    const bool active = tid < TC_THREADS;  // larger CTAs: threads past the first 256 only join the barriers
    const int w = (tid >> 5) & 7, lane = tid & 31;
    const int base = 32 * (w >> 2), c = lane & 15;
    const int r0 = 4 * (w & 3) + 2 * (lane >> 4);  // rows r0, r0 + 1 of the 16 x 16 lower-left block
    float acc[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) acc[x] = sRT[(base + 16 + r0 + x) * RP + base + c];
#pragma unroll
    for (int m4 = 0; m4 < 16; m4 += 4) {
        float a[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) a[t] = (m4 + t > c) ? sRT[(base + m4 + t) * RP + base + c] : 0.f;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const float4 cr = *reinterpret_cast<const float4*>(sRT + (base + 16 + r0 + x) * RP + base + m4);
            acc[x] += cr.x * a[0] + cr.y * a[1] + cr.z * a[2] + cr.w * a[3];
        }
    }
    if (active) {
#pragma unroll
        for (int x = 0; x < 2; ++x) sX[(w >> 2) * 256 + (r0 + x) * 16 + c] = acc[x];
    }
    __syncthreads();
    const float* Xb = sX + (w >> 2) * 256;
#pragma unroll
    for (int x = 0; x < 2; ++x) acc[x] = Xb[(r0 + x) * 16 + c];
#pragma unroll
    for (int m4 = 0; m4 < 16; m4 += 4) {
        float xm[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) xm[t] = Xb[(m4 + t) * 16 + c];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const float4 dr = *reinterpret_cast<const float4*>(sRT + (base + 16 + r0 + x) * RP + base + 16 + m4);
            const int r = r0 + x;
            acc[x] += (m4 + 0 < r ? dr.x * xm[0] : 0.f) + (m4 + 1 < r ? dr.y * xm[1] : 0.f) +
                      (m4 + 2 < r ? dr.z * xm[2] : 0.f) + (m4 + 3 < r ? dr.w * xm[3] : 0.f);
        }
    }
    if (active) {
#pragma unroll
        for (int x = 0; x < 2; ++x) sRT[(base + 16 + r0 + x) * RP + base + c] = -acc[x];
    }
    __syncthreads();
}

// Step 32 -> 64 (one block): warp w serves rows 4 w + {0..3}, lane = column.
__device__ __forceinline__ void tri_inverse_step32(float* sRT, float* sX, int tid) {
    const bool active = tid < TC_THREADS;  // larger CTAs: threads past the first 256 only join the barriers
    const int w = (tid >> 5) & 7, c = tid & 31, r0 = 4 * w;
    float acc[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[x] = sRT[(32 + r0 + x) * RP + c];
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        float a[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) a[t] = (m4 + t > c) ? sRT[(m4 + t) * RP + c] : 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float4 cr = *reinterpret_cast<const float4*>(sRT + (32 + r0 + x) * RP + m4);
            acc[x] += cr.x * a[0] + cr.y * a[1] + cr.z * a[2] + cr.w * a[3];
        }
    }
    if (active) {
#pragma unroll
        for (int x = 0; x < 4; ++x) sX[(r0 + x) * 32 + c] = acc[x];
    }
    __syncthreads();
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[x] = sX[(r0 + x) * 32 + c];
#pragma unroll
    for (int m4 = 0; m4 < 32; m4 += 4) {
        if (m4 >= r0 + 3) break;  // warp-uniform: no row of this warp reaches these m
        float xm[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) xm[t] = sX[(m4 + t) * 32 + c];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float4 dr = *reinterpret_cast<const float4*>(sRT + (32 + r0 + x) * RP + 32 + m4);
            const int r = r0 + x;
            acc[x] += (m4 + 0 < r ? dr.x * xm[0] : 0.f) + (m4 + 1 < r ? dr.y * xm[1] : 0.f) +
                      (m4 + 2 < r ? dr.z * xm[2] : 0.f) + (m4 + 3 < r ? dr.w * xm[3] : 0.f);
        }
    }
    if (active) {
#pragma unroll
        for (int x = 0; x < 4; ++x) sRT[(32 + r0 + x) * RP + c] = -acc[x];
    }
    __syncthreads();
}

}  // namespace c64
}  // namespace kda
