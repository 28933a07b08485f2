// kda_tc_ptx.cuh -- thin inline-PTX wrappers for the sm_100a tensor-core path:
// tcgen05.mma (kind::tf32, A and B from shared memory, fp32 accumulator in TMEM),
// tcgen05.commit -> mbarrier, TMEM allocation, tcgen05.ld / tcgen05.st, and the
// proxy / thread-sync fences that order them.
//
// Operand layout used everywhere (no swizzle, "K-major"): an operand with `rows`
// rows (its M or N index) and KD elements along the contraction is tiled into
// 8-row x 16-byte core matrices of 128 contiguous bytes; core matrix (row/8, k/4)
// sits at ((row/8) * KD/4 + k/4) * 128 bytes.  In descriptor terms: the two
// 16-byte K-chunks one MMA step reads are 128 B apart (leading byte offset) and
// successive 8-row groups are KD/4 * 128 B apart (stride byte offset).  One
// kind::tf32 MMA step covers K = 8, i.e. 256 bytes of that tiling.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of element (r, k) in a [rows][KD] fp32/tf32 operand tile.
__device__ __forceinline__ uint32_t cm_off(int r, int k, int KD) {
    return ((uint32_t)((r >> 3) * (KD >> 2) + (k >> 2)) << 7) + ((uint32_t)(r & 7) << 4) + ((uint32_t)(k & 3) << 2);
}

// Shared-memory matrix descriptor: start address, leading byte offset 128, stride byte offset
// `sbo`, descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) |
           (1ull << 46);
}

// Instruction descriptor for kind::tf32 with fp32 accumulation, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// Same MMA with the A operand read from TMEM (row m in lane m, contraction index along columns;
// the tensor core takes the top 19 bits of each fp32 word, i.e. truncates it to tf32).
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

// The products below build each shared-memory descriptor once and step it along K by adding to its
// start-address field (address / 16 in bits 0-13: shared memory stays below 256 KB, so the field does not
// carry): the issuing thread then spends a few instructions per MMA, not a descriptor build.

// D[M x N] (+)= A_tmem[M x 8*ksteps] * B[N x 8*ksteps]^T: one K = 8 step per 8 TMEM columns of A.
__device__ __forceinline__ void gemm_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_addr, uint32_t b_sbo,
                                             uint32_t idesc, int ksteps, bool accumulate) {
    const uint64_t b0 = smem_desc(b_addr, b_sbo);
#pragma unroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_tf32_ts(d_tmem, a_tmem + 8u * ks, b0 + (uint64_t)(16 * ks), idesc, (ks > 0 || accumulate) ? 1u : 0u);
}

// D[M x N] (+)= A[M x 8*ksteps] * B[N x 8*ksteps]^T, operands in the tiling above.
__device__ __forceinline__ void gemm_tf32(uint32_t d_tmem, uint32_t a_addr, uint32_t a_sbo, uint32_t b_addr,
                                          uint32_t b_sbo, uint32_t idesc, int ksteps, bool accumulate) {
    const uint64_t a0 = smem_desc(a_addr, a_sbo), b0 = smem_desc(b_addr, b_sbo);
#pragma unroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_tf32(d_tmem, a0 + (uint64_t)(16 * ks), b0 + (uint64_t)(16 * ks), idesc, (ks > 0 || accumulate) ? 1u : 0u);
}

// ---- kind::f16 with fp16 operands (both A and B fp16), fp32 accumulation ----------------------------
// Operand tiling for 16-bit elements: 8-row x 16-byte core matrices hold 8 x 8 elements; core matrix
// (row/8, k/8) sits at ((row/8) * KD/8 + k/8) * 128 bytes, so one K = 16 MMA step reads 256 bytes of it
// (leading byte offset 128) and 8-row groups are KD/8 * 128 bytes apart (stride byte offset).
__device__ __forceinline__ uint32_t cm_off16(int r, int k, int KD) {
    return ((uint32_t)((r >> 3) * (KD >> 3) + (k >> 3)) << 7) + ((uint32_t)(r & 7) << 4) + ((uint32_t)(k & 7) << 1);
}

// Shared-memory matrix descriptor with a leading byte offset `lbo` (the distance between K-adjacent
// core matrices; a multiple of 16), stride byte offset `sbo`, descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t smem_desc_lbo(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor for kind::f16 with fp16 A and B, fp32 accumulation, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// D[M x N] (+)= A[M x 16*ksteps] * B[N x 16*ksteps]^T, fp16 operands in the tiling of cm_off16.
__device__ __forceinline__ void gemm_f16(uint32_t d_tmem, uint32_t a_addr, uint32_t a_sbo, uint32_t b_addr,
                                         uint32_t b_sbo, uint32_t idesc, int ksteps, bool accumulate) {
    const uint64_t a0 = smem_desc(a_addr, a_sbo), b0 = smem_desc(b_addr, b_sbo);
#pragma unroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_f16(d_tmem, a0 + (uint64_t)(16 * ks), b0 + (uint64_t)(16 * ks), idesc, (ks > 0 || accumulate) ? 1u : 0u);
}

// gemm_f16 with a B operand whose K-adjacent core matrices are `b_lbo` bytes apart (a padded tiling:
// with b_lbo = 144 the eight rows of a core matrix and the next core matrix along K fall in different
// banks, so stores of one column by 32 consecutive K indices do not conflict).
__device__ __forceinline__ void gemm_f16_bpad(uint32_t d_tmem, uint32_t a_addr, uint32_t a_sbo, uint32_t b_addr,
                                              uint32_t b_lbo, uint32_t b_sbo, uint32_t idesc, int ksteps,
                                              bool accumulate) {
    const uint64_t a0 = smem_desc(a_addr, a_sbo), b0 = smem_desc_lbo(b_addr, b_lbo, b_sbo);
    const uint64_t b_step = (2u * b_lbo) >> 4;
#pragma unroll
    for (int ks = 0; ks < ksteps; ++ks)
        mma_f16(d_tmem, a0 + (uint64_t)(16 * ks), b0 + b_step * (uint64_t)ks, idesc, (ks > 0 || accumulate) ? 1u : 0u);
}

// 2^e as a float, for -126 <= e <= 127 (exact).
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// The power-of-two exponent e with max_abs * 2^-e in [2^13, 2^14): operands scaled by 2^-e keep fp16's
// 10 mantissa bits and stay four times below its largest finite value.  0 for a zero or NaN bound, the
// upper clamp for an infinite one; the result is clamped to [-100, 100] so that 2^e, 2^-e and the
// product of two such factors with a small power of two are normal floats.
__device__ __forceinline__ int fp16_scale_exponent(float max_abs) {
    if (!(max_abs > 0.f)) return 0;
    if (!(max_abs < 3.0e38f)) return 100;
    // IEEE single: a normal value with biased exponent b lies in [2^(b-127), 2^(b-126))
    const int b = (int)((__float_as_uint(max_abs) >> 23) & 0xFFu);
    const int e = (b == 0 ? -126 : b - 126) - 14;
    return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// Round two floats to fp16 (nearest, ties to even) and pack them, the first in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Unpack two fp16 values (low half first) to floats.
__device__ __forceinline__ void f16x2_to_f32(uint32_t x, float& lo, float& hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}" : "=f"(lo), "=f"(hi) : "r"(x));
}

__device__ __forceinline__ uint16_t to_f16_bits(float x) {
    uint16_t r;
    asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// Warp-wide maximum of non-negative floats (their bit patterns order like unsigned integers).
__device__ __forceinline__ float warp_max_nonneg(float x) {
    return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(x)));
}

// Barrier over `nthreads` threads (whole warps) that use the same id; id 0 is __syncthreads.
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Bounded wait for the mbarrier phase with the given parity to complete.  Returns false if it
// did not complete within `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, uint32_t limit) {
    uint32_t done = 0;
    for (uint32_t it = 0; it < limit; ++it) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// TMEM allocation (one full warp executes these).
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) { return base + ((uint32_t)lane << 16) + (uint32_t)col; }

// 32 lanes x 32-bit, 16 / 32 consecutive columns per thread (thread t <-> lane base + t).
__device__ __forceinline__ void tmem_ld16(uint32_t a, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(a));
}
__device__ __forceinline__ void tmem_ld8(uint32_t a, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(a));
}
__device__ __forceinline__ void tmem_ld32(uint32_t a, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(a));
}
__device__ __forceinline__ void tmem_st16(uint32_t a, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(a),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]));
}
__device__ __forceinline__ void tmem_st32(uint32_t a, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(a),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16-byte asynchronous global -> shared copy; src_bytes < 16 zero-fills the rest (0: all zeros).
__device__ __forceinline__ void cp_async16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Bulk (non-tensor) asynchronous copies between global and this CTA's shared memory.  Both
// addresses 16-byte aligned, size a multiple of 16.  No cluster multicast anywhere.
// The mbarrier completes its phase once `bytes` of announced transactions have landed.
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_smem),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}
// Tiled 4-D tensor copy global -> shared through a tensor map (a __grid_constant__ kernel parameter),
// completing on an mbarrier as transaction bytes.  Coordinates innermost first; the innermost one
// times the element size must be a multiple of 16 bytes.  Elements outside the tensor read as zero.
__device__ __forceinline__ void tma_load_4d(uint32_t dst_smem, const void* tmap, int c0, int c1, int c2, int c3,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src_smem), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the committed bulk stores of this thread have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until the committed bulk stores of this thread are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// fp32 -> operand word for a kind::tf32 MMA.  The tensor core reads the top 19 bits of each word
// (sign, exponent, 10 mantissa bits) and ignores the low 13; adding half a unit of the 10th
// mantissa bit to the magnitude first makes that truncation a round to nearest (ties away from
// zero; a carry into the exponent gives the correctly rounded next binade).  One integer add.
__device__ __forceinline__ uint32_t to_tf32(float x) { return __float_as_uint(x) + 0x1000u; }

// Rotation inside aligned groups of 8: a[g + k] <- a[g + ((k + r) & 7)] for r in 0..7, by three
// conditional rotations (no dynamic register indexing).  Used to give the 8 lanes that would store
// to the same shared-memory bank 8 different words of their group, so that transposed stores into
// the operand tiling are free of bank conflicts.
template <int N>
__device__ __forceinline__ void rotate_groups8(uint32_t (&a)[N], int r) {
    static_assert(N % 8 == 0, "groups of 8");
#pragma unroll
    for (int sh = 1; sh < 8; sh <<= 1) {
        const bool on = (r & sh) != 0;
#pragma unroll
        for (int g = 0; g < N; g += 8) {
            uint32_t t[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) t[k] = a[g + ((k + sh) & 7)];
#pragma unroll
            for (int k = 0; k < 8; ++k) a[g + k] = on ? t[k] : a[g + k];
        }
    }
}

// Row-of-TMEM loader: N columns (16 or 32) starting at `col` for this warp's 32 lanes.
template <int N>
struct TmemRow;
template <>
struct TmemRow<16> {
    uint32_t r[16];
    __device__ __forceinline__ void load(uint32_t a) { tmem_ld16(a, r); }
    __device__ __forceinline__ void store(uint32_t a) { tmem_st16(a, r); }
};
template <>
struct TmemRow<32> {
    uint32_t r[32];
    __device__ __forceinline__ void load(uint32_t a) { tmem_ld32(a, r); }
    __device__ __forceinline__ void store(uint32_t a) { tmem_st32(a, r); }
};

}  // namespace tc
}  // namespace kda
