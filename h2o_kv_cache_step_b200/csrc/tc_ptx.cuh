// tc_ptx.cuh -- inline-PTX wrappers for the sm_100a tensor-core path:
// TMEM allocation, tcgen05.mma (kind::f16, bf16 in / fp32 accumulate) and its
// commit, TMEM <-> register moves, TMA tile loads, and the shared-memory
// matrix descriptors of the 128-byte-swizzled operand layouts.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace h2o {
namespace tc {

// ---- TMEM -----------------------------------------------------------------
// Allocate ncols (power of two >= 32) TMEM columns; the base address lands in
// *slot (shared memory). Warp-collective: one whole warp calls it.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- MMA ------------------------------------------------------------------
// D[tmem] (+)= A[smem] * B[smem]^T, one instruction of shape M x N x 16.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// mma_bf16_ss issued by a whole converged warp: elect.sync picks one lane
// (the lowest active one, the same every time under a full mask), which
// issues the instruction. The warp never diverges around the issue, so its
// operands can stay in uniform registers.
__device__ __forceinline__ void mma_bf16_ss_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A is read from TMEM (M rows on the lanes,
// K packed two bf16 per 32-bit column, K-major).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on the mbarrier when every tcgen05 operation this thread has
// issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// mma_commit by a whole converged warp through the lane elect.sync picks
// (the lane that issued the warp's mma_bf16_ss_warp instructions).
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator.
// b_mn_major: B stored N-contiguous (MN-major) rather than K-contiguous.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((b_mn_major ? 1u : 0u) << 16)   // B major-ness
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle, K-major: rows of 128 B
// (64 bf16 of K), groups of 8 rows 1024 B apart. The start address may be
// advanced by 32 B steps to select the 16-element K slice inside the row.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address >> 4
    d |= (uint64_t)1 << 16;                    // leading offset (unused for this layout)
    d |= (uint64_t)(1024u >> 4) << 32;         // stride offset: 8-row groups
    d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

// Same swizzle, MN-major: 64 contiguous MN elements per 128-B row, rows are
// consecutive K indices; 8-row K groups 1024 B apart; further 64-element MN
// blocks `mn_block_bytes` apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t mn_block_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16;  // leading offset: MN blocks
    d |= (uint64_t)(1024u >> 4) << 32;                      // stride offset: 8-row K groups
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// ---- TMEM <-> registers ----------------------------------------------------
// Each thread of the warp reads 32 consecutive 32-bit columns of its lane
// (lane = 32 * (warp % 4) + laneid, encoded in taddr's upper half).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
          "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Orders every later use of v after the preceding tmem_ld_wait(): each
// register passes through an empty volatile asm, and volatile asm statements
// keep their order, so no read of a tcgen05.ld destination is scheduled
// before the wait that completes it.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(v[i]));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- TMA --------------------------------------------------------------------
// 2-D tiled load of the box at (x = column, y = row) into shared memory; the
// mbarrier receives the byte count. x * 2 bytes must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Contiguous global -> shared copy on the TMA unit (bytes a multiple of 16,
// both addresses 16-byte aligned); completes on the mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- register reallocation between warpgroups ----------------------------------
// Executed by all four warps of a warpgroup. The per-thread counts of all
// warpgroups must add up to at most the registers the block was launched with.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---- misc -------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA/ALU pipes instead of the MUFU unit, for x <= ~126. Results
// below 2^-125 are flushed to 0 (ex2.approx.ftz flushes below 2^-126; the
// extra binade keeps the exponent field of the constructed float >= 1).
// Range reduction x = n + f with n = round(x): adding 1.5 * 2^23 rounds x to
// an integer held in the low mantissa bits of t; f = x - n lies in
// [-1/2, 1/2]; 2^f comes from a polynomial fitted (relative error) at
// Chebyshev nodes of [-1/2, 1/2] by csrc/gen_exp2_poly.py; n is then added to
// the exponent field ((bits(t) << 23) == n << 23 modulo 2^32).
// Max relative error of the float32 evaluation: 7.7e-5 (degree 3),
// 2.7e-6 (degree 4).
__device__ __forceinline__ float exp2_reduce(float x, float& f) {
    x = fmaxf(x, -125.0f);
    const float t = x + 12582912.0f;
    const float n = t - 12582912.0f;
    f = x - n;
    return t;
}
__device__ __forceinline__ float exp2_poly3(float x) {
    float f;
    const float t = exp2_reduce(x, f);
    const float p = fmaf(fmaf(fmaf(5.508868396e-02f, f, 2.426040471e-01f), f, 6.932762265e-01f), f,
                         9.999289513e-01f);
    const float r = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
    return x >= -125.0f ? r : 0.0f;
}
__device__ __forceinline__ float exp2_poly4(float x) {
    float f;
    const float t = exp2_reduce(x, f);
    const float p =
        fmaf(fmaf(fmaf(fmaf(9.560510516e-03f, f, 5.591703951e-02f), f, 2.402498126e-01f), f, 6.931219697e-01f),
             f, 9.999991655e-01f);
    const float r = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
    return x >= -125.0f ? r : 0.0f;
}

// ---- packed fp32 pairs (one instruction for two lanes of data) -------------
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// a + b with subnormal inputs and results flushed to zero.
__device__ __forceinline__ float fadd_ftz(float a, float b) {
    float d;
    asm("add.rn.ftz.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ float2 fadd2_ftz(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.ftz.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two 2^x at once on the FMA pipe (degree-3 or degree-4 polynomial, same
// range reduction and flush as exp2_poly3 / exp2_poly4).
template <int DEG>
__device__ __forceinline__ float2 exp2_poly_x2(float2 x) {
    const float2 xc = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
    const float2 magic = make_float2(12582912.0f, 12582912.0f);
    const float2 t = fadd2(xc, magic);
    const float2 n = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = fadd2(xc, make_float2(-n.x, -n.y));
    float2 p;
    if (DEG == 3) {
        p = ffma2(make_float2(5.508868396e-02f, 5.508868396e-02f), f, make_float2(2.426040471e-01f, 2.426040471e-01f));
        p = ffma2(p, f, make_float2(6.932762265e-01f, 6.932762265e-01f));
        p = ffma2(p, f, make_float2(9.999289513e-01f, 9.999289513e-01f));
    } else {
        p = ffma2(make_float2(9.560510516e-03f, 9.560510516e-03f), f, make_float2(5.591703951e-02f, 5.591703951e-02f));
        p = ffma2(p, f, make_float2(2.402498126e-01f, 2.402498126e-01f));
        p = ffma2(p, f, make_float2(6.931219697e-01f, 6.931219697e-01f));
        p = ffma2(p, f, make_float2(9.999991655e-01f, 9.999991655e-01f));
    }
    float2 r;
    r.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
    r.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
    r.x = x.x >= -125.0f ? r.x : 0.0f;
    r.y = x.y >= -125.0f ? r.y : 0.0f;
    return r;
}

// Two 2^x at once, degree-3 polynomial, with the range reduction clamped at
// -126 and no explicit flush: for x <= -126 (and just above it, where
// 2^x < 2^-126) the result is a subnormal float, which every consumer reads
// through flush-to-zero arithmetic (fadd2_ftz), exactly like ex2.approx.ftz.
// About 5.5 issue slots per value instead of ~7 with the explicit flush.
__device__ __forceinline__ float2 exp2_poly3_x2_ftz(float2 x) {
    const float2 xc = make_float2(fmaxf(x.x, -126.0f), fmaxf(x.y, -126.0f));
    const float2 t = fadd2(xc, make_float2(12582912.0f, 12582912.0f));
    const float2 n = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = fadd2(xc, make_float2(-n.x, -n.y));
    float2 p = ffma2(make_float2(5.508868396e-02f, 5.508868396e-02f), f,
                     make_float2(2.426040471e-01f, 2.426040471e-01f));
    p = ffma2(p, f, make_float2(6.932762265e-01f, 6.932762265e-01f));
    p = ffma2(p, f, make_float2(9.999289513e-01f, 9.999289513e-01f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Sync of the `count` threads of named barrier `id` (id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
    return *reinterpret_cast<uint32_t*>(&t);
}

}  // namespace tc

// ---- role synchronisation shared by the tensor-core kernels -----------------
// Bounded wait that also gives up once another role has given up.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const WaitBound& wb, int code,
                                         volatile int* abort_flag) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        for (int i = 0; i < 8; ++i)
            if (mbar_try_wait_sleep(addr, parity, 20000u)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > wb.ns) {
            record_error(wb, code);
            *abort_flag = 1;
            return false;
        }
    }
}

// Every lane waits; the outcome is made warp-uniform so that a give-up never
// leaves part of a warp behind at a warp-collective instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitBound& wb, int code,
                                          volatile int* abort_flag) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, wb, code, abort_flag));
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

}  // namespace h2o
