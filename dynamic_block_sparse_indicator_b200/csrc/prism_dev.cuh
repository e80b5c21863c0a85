// prism_dev.cuh -- sm_100a device primitives used by the attention kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// UMMA issue/commit, TMEM loads/stores) and shared-memory matrix descriptors.
//
// Every wait is bounded: after kWaitLimit polls it records PRISM_ERR_TIMEOUT
// in the plan's device error word and returns false, and the caller unwinds.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "prism_internal.h"

namespace prism {

constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s of wall-clock per wait before giving up
#ifndef PRISM_WAIT_SUSPEND
#define PRISM_WAIT_SUSPEND 1
#endif

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes (it is woken at once) or about `ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(ns) : "memory");
    return ok != 0;
}
// Bounded wait for the phase of parity `parity`; false (and the error word
// set, with `where` in err[1]) if it did not complete within kWaitNs.  The
// first poll is inline; the polling loop is an out-of-line call, which keeps
// the inline code of every wait short (the MMA issuer is a single warp whose
// instructions must stay in the instruction cache next to busy softmax warps).
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, int* err, int where) {
    const uint64_t t0 = globaltimer_ns();
#if PRISM_WAIT_SUSPEND
    for (;;) {
        if (mbar_try_suspend(bar, parity, 20000)) return true;
        if (*(volatile int*)err != 0) return false;              // someone else gave up
        if (globaltimer_ns() - t0 > kWaitNs) break;
    }
#else
    for (uint32_t i = 0;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if (i > 16) __nanosleep(128);
        if ((i & 255) == 0) {
            if (*(volatile int*)err != 0) return false;          // someone else gave up
            if (globaltimer_ns() - t0 > kWaitNs) break;
        }
    }
#endif
    if (atomicCAS(err, 0, PRISM_ERR_TIMEOUT) == 0) {
        err[1] = where;
        err[2] = (int)blockIdx.x;
        err[3] = (int)threadIdx.x;
    }
    return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int where = 0) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, err, where);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)),
           "r"(x), "r"(y) : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Element-wise add of a shared-memory tile into global memory (TMA reduce).
__device__ __forceinline__ void tma_reduce_add_2d(const void* tmap, const void* src, int32_t x, int32_t y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];"
                 :: "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(src)), "r"(x), "r"(y) : "memory");
}
// Running maximum magnitude over a 16-byte chunk of 16- or 32-bit floats: a
// magnitude is the value's bits with the sign cleared, so the maximum is an
// integer maximum (per 16-bit half for bf16; a NaN's bits exceed infinity's).
// abs_bits turns the result into fp32 bits (a bf16's bits shifted left by 16).
template <typename T>
__device__ __forceinline__ uint32_t fold_abs(uint32_t m, const uint4& x) {
    static_assert(sizeof(T) == 2 || sizeof(T) == 4, "16- or 32-bit values");
    if (sizeof(T) == 2) {
        constexpr uint32_t mask = 0x7fff7fffu;
        m = __vmaxu2(m, x.x & mask);
        m = __vmaxu2(m, x.y & mask);
        m = __vmaxu2(m, x.z & mask);
        return __vmaxu2(m, x.w & mask);
    }
    constexpr uint32_t mask = 0x7fffffffu;
    return max(max(m, x.x & mask), max(max(x.y & mask, x.z & mask), x.w & mask));
}
template <typename T>
__device__ __forceinline__ uint32_t abs_bits(uint32_t m) {
    return sizeof(T) == 2 ? max(m & 0xffffu, m >> 16) << 16 : m;
}

// Fire-and-forget fp32 add into global memory, performed in L2.
__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" :: "l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Named barrier among `count` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, 16-bit in, fp32 accumulate.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T: A (M x K, 16-bit) held in TMEM, lane = row,
// two K elements per 32-bit column (even K in the low half).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// Arrive once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

#define PRISM_TMEM_LD32(taddr, r)                                                          \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"                                  \
                 " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"               \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];" \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),   \
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), \
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),          \
                   "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),          \
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]),          \
                   "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])           \
                 : "r"(taddr))

#define PRISM_TMEM_ST32(taddr, r)                                                          \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32"                                  \
                 " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"         \
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"       \
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]),      \
                    "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]),      \
                    "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), \
                    "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), \
                    "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), \
                    "r"(r[29]), "r"(r[30]), "r"(r[31]) : "memory")

#define PRISM_TMEM_ST16(taddr, r)                                                          \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32"                                  \
                 " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"        \
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]),      \
                    "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]),      \
                    "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory")

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------- shared-memory descriptors
// Operand tiles live in shared memory in the 128-byte-swizzled layout that a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes: rows of 128 bytes (64 bf16),
// 8-row / 1024-byte swizzle atoms, the 16-byte chunk c of row r stored at
// chunk position c ^ (r & 7).  A tile wider than 64 elements is split into
// "slabs" of 64 columns, each slab = rows x 128 bytes.
//
// Descriptor fields (sm_100): start address >> 4 in bits 0-13, leading byte
// offset >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45, version 1
// in bits 46-47, swizzle mode (2 = 128B) in bits 61-63.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// K-major operand (rows = M or N, the contraction dim contiguous): the k-th
// 16-element step starts 32*k bytes into the row (inside a slab) or in the
// next slab.  SBO = 1024 (next 8-row group); LBO unused for swizzled K-major.
// The same descriptors split into a constant high word (SBO 1024 B, version 1,
// 128-byte swizzle) and a low word (start address, LBO).  Within one tile the
// K steps only add an immediate to the low word (the start field is 14 bits of
// a shared address below 256 KB, so the add never carries out of it), which
// keeps the MMA issuer's instruction stream short.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr >> 4) & 0x3FFFu) | ((lbo >> 4) << 16);
}
__device__ __forceinline__ uint64_t desc_from_lo(uint32_t lo) {
    return ((uint64_t)kDescHi << 32) | lo;
}
// low-word offset of K step k16 of a K-major tile of 64-column slabs
__host__ __device__ constexpr uint32_t kmajor_step(int k16, uint32_t slab_bytes) {
    return ((uint32_t)(k16 >> 2) * slab_bytes + (uint32_t)(k16 & 3) * 32u) >> 4;
}
// low-word offset of K step k16 of an MN-major tile
__host__ __device__ constexpr uint32_t mnmajor_step(int k16) { return (uint32_t)k16 * (2048u >> 4); }
// K-major tile of 64-column slabs: K step k16 moves 32 B inside a slab, a new
// slab every 4 steps.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_saddr, int k16, uint32_t slab_bytes) {
    return desc_from_lo(desc_lo(tile_saddr, 16) + kmajor_step(k16, slab_bytes));
}
// MN-major tile (MN contiguous, 64-element slabs slab_bytes apart): K step
// k16 moves 16 rows of 128 B.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile_saddr, int k16, uint32_t slab_bytes) {
    return desc_from_lo(desc_lo(tile_saddr, slab_bytes) + mnmajor_step(k16));
}

// One accumulation chain of n MMAs (K = 16 each) with the loop kept rolled:
// A and B are shared-memory tiles given by descriptor low words, K-major
// (slab bytes apart every 4 steps) or MN-major.  A short loop keeps the MMA
// issuer's instruction stream small.
template <bool A_KMAJOR, bool B_KMAJOR>
__device__ __forceinline__ void umma_chain(uint32_t d_tmem, uint32_t a_lo, uint32_t a_slab, uint32_t b_lo,
                                           uint32_t b_slab, uint32_t idesc, int n, bool acc) {
    #pragma unroll 1
    for (int kk = 0; kk < n; ++kk) {
        const uint32_t ao = A_KMAJOR ? kmajor_step(kk, a_slab) : mnmajor_step(kk);
        const uint32_t bo = B_KMAJOR ? kmajor_step(kk, b_slab) : mnmajor_step(kk);
        umma_f16(d_tmem, desc_from_lo(a_lo + ao), desc_from_lo(b_lo + bo), idesc, (acc || kk > 0) ? 1u : 0u);
    }
}
// The same with A (M x K, 16-bit) in TMEM: 8 columns per K step.
template <bool B_KMAJOR>
__device__ __forceinline__ void umma_chain_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_slab,
                                              uint32_t idesc, int n, bool acc) {
    #pragma unroll 1
    for (int kk = 0; kk < n; ++kk) {
        const uint32_t bo = B_KMAJOR ? kmajor_step(kk, b_slab) : mnmajor_step(kk);
        umma_f16_ts(d_tmem, a_tmem + 8 * kk, desc_from_lo(b_lo + bo), idesc, (acc || kk > 0) ? 1u : 0u);
    }
}

// Instruction descriptor, kind::f16 with fp16 A/B and fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4)                     // D format: f32
         | (0u << 7)                     // A format: f16
         | (0u << 10)                    // B format: f16
         | ((uint32_t)a_mn_major << 15)
         | ((uint32_t)b_mn_major << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Byte offset, inside a 128B-swizzled slab, of the 16-byte chunk `c` (0..7) of row `r`.
__device__ __forceinline__ uint32_t swz128(int r, int c) {
    return (uint32_t)r * 128u + (uint32_t)((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 :: "r"(saddr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Packed fp32 pairs (sm_100 f32x2 instructions): one instruction for two lanes
// of arithmetic, round-to-nearest like the scalar forms.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace prism
