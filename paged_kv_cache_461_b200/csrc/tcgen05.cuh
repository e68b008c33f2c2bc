// tcgen05.cuh -- inline-PTX wrappers for the 5th-generation tensor cores (TMEM
// allocation, tcgen05.mma with shared-memory descriptors or a TMEM A operand,
// commit to an mbarrier, TMEM loads and stores), packed fp32x2 arithmetic and
// the shared-memory / instruction descriptor encodings.  Used by the prefill
// kernel only.
#pragma once

#include "ptx.cuh"

namespace pa {

// ---------------------------------------------------------------- tcgen05 (prefill)
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The tcgen05.mma / tcgen05.commit wrappers below are warp-collective: all 32 lanes of one
// warp call them with the same arguments and one lane, picked by elect.sync, issues.  Keeping
// the whole warp on the issuing path lets the operands stay warp-uniform, which measured about
// 10% more MMA issue rate than a single-lane branch.

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, pe;\n\t.reg .b32 re;\n\t"
        "elect.sync re|pe, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A is read from TMEM (lane = row of A,
// each 32-bit column holds two consecutive K elements, lower K index in the low half)
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, pe;\n\t.reg .b32 re;\n\t"
        "elect.sync re|pe, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Eight back-to-back kind::f16 MMAs into one accumulator, operands from shared memory:
// MMA i uses descriptors a + A_OFF(i) and b + B_OF(i) (16-byte units), offsets given as a
// compile-time table.  The first MMA overwrites D unless accumulate is set; the rest add.
template <uint32_t A0, uint32_t A1, uint32_t A2, uint32_t A3, uint32_t A4, uint32_t A5, uint32_t A6, uint32_t A7>
__device__ __forceinline__ void umma_f16_x8_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p0, pe;\n\t.reg .b64 ra, rb;\n\t.reg .b32 re;\n\t"
        "elect.sync re|pe, 0xffffffff;\n\t"
        "setp.ne.b32 p0, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n\t"
        "add.s64 ra, %1, %5;\n\tadd.s64 rb, %2, %5;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %6;\n\tadd.s64 rb, %2, %6;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %7;\n\tadd.s64 rb, %2, %7;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %8;\n\tadd.s64 rb, %2, %8;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %9;\n\tadd.s64 rb, %2, %9;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %10;\n\tadd.s64 rb, %2, %10;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %11;\n\tadd.s64 rb, %2, %11;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "n"((uint64_t)A1), "n"((uint64_t)A2),
          "n"((uint64_t)A3), "n"((uint64_t)A4), "n"((uint64_t)A5), "n"((uint64_t)A6), "n"((uint64_t)A7)
        : "memory");
    (void)A0;
}

// Four back-to-back kind::f16 MMAs into one accumulator, operands from shared memory, MMA i at
// descriptors a + A_OFF(i) and b + A_OFF(i) (16-byte units, A_OFF(0) = 0); the first overwrites D.
template <uint32_t A1, uint32_t A2, uint32_t A3>
__device__ __forceinline__ void umma_f16_x4_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc)
{
    asm volatile(
        "{\n\t.reg .pred pe;\n\t.reg .b64 ra, rb;\n\t.reg .b32 re;\n\t"
        "elect.sync re|pe, 0xffffffff;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 0;\n\t"
        "add.s64 ra, %1, %4;\n\tadd.s64 rb, %2, %4;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %5;\n\tadd.s64 rb, %2, %5;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t"
        "add.s64 ra, %1, %6;\n\tadd.s64 rb, %2, %6;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], ra, rb, %3, 1;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "n"((uint64_t)A1), "n"((uint64_t)A2), "n"((uint64_t)A3)
        : "memory");
}

// Eight back-to-back kind::f16 MMAs, A from TMEM (columns a_tmem + 8i), B from shared memory
// (descriptor b + i * B_STEP in 16-byte units).
template <uint32_t B_STEP>
__device__ __forceinline__ void umma_f16_x8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                               uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p0, pe;\n\t.reg .b64 rb;\n\t.reg .b32 ra, re;\n\t"
        "elect.sync re|pe, 0xffffffff;\n\t"
        "setp.ne.b32 p0, %4, 0;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
        "add.u32 ra, %1, 8;\n\tadd.s64 rb, %2, %5;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 16;\n\tadd.s64 rb, %2, %6;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 24;\n\tadd.s64 rb, %2, %7;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 32;\n\tadd.s64 rb, %2, %8;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 40;\n\tadd.s64 rb, %2, %9;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 48;\n\tadd.s64 rb, %2, %10;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t"
        "add.u32 ra, %1, 56;\n\tadd.s64 rb, %2, %11;\n\t"
        "@pe tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], rb, %3, 1;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "n"((uint64_t)B_STEP),
          "n"((uint64_t)(2 * B_STEP)), "n"((uint64_t)(3 * B_STEP)), "n"((uint64_t)(4 * B_STEP)),
          "n"((uint64_t)(5 * B_STEP)), "n"((uint64_t)(6 * B_STEP)), "n"((uint64_t)(7 * B_STEP))
        : "memory");
}

// arrive on an mbarrier once all tcgen05 ops issued so far by the issuing lane are done
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("{\n\t.reg .pred pe;\n\t.reg .b32 re;\n\t"
                 "elect.sync re|pe, 0xffffffff;\n\t"
                 "@pe tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 32 lanes x 32 consecutive 32-bit columns into r[0..31] of a register array (constant indices only):
// thread i of the warp gets lane (base + i), columns col .. col + 31
__device__ __forceinline__ void tmem_ld32p(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// ---------------------------------------------------------------- warpgroup register budgets
// setmaxnreg moves registers between the warpgroups of a CTA: every warp of a warpgroup executes
// the same instruction.  A raise waits until lowered warpgroups have returned enough registers to
// the CTA's pool (threads x registers per thread at launch), so the budgets of all warpgroups
// must add up to at most that pool; the host checks this against the compiled kernel before
// every launch.
template <uint32_t N>
__device__ __forceinline__ void wg_reg_raise()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <uint32_t N>
__device__ __forceinline__ void wg_reg_lower()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- packed fp32 pairs (sm_100)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Shared-memory matrix descriptor for tcgen05.mma (sm_100 format):
// start address >> 4 in bits [0,14), leading byte offset >> 4 in [16,30),
// stride byte offset >> 4 in [32,46), version 1 in [46,48), swizzle mode in
// [61,64) (2 = 128-byte swizzle).  Base offset 0: every operand tile starts on
// a 1024-byte boundary (advancing the start inside a swizzle atom along K is
// done by adding the byte offset, as the hardware applies the XOR pattern to
// the final address bits).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D, dense.
// a_mn / b_mn: 1 if the operand is MN-major in shared memory.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn)
{
    return (1u << 4)                                  // D format: f32
           | (1u << 7)                                // A format: bf16
           | (1u << 10)                               // B format: bf16
           | (static_cast<uint32_t>(a_mn) << 15)      // A major
           | (static_cast<uint32_t>(b_mn) << 16)      // B major
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

} // namespace pa
