// prism_attn_fwd.cu -- block-sparse attention forward on sm_100a tensor cores.
//
// Algorithm 1 stages 4-5 of "Prism: Dynamic Sparse Attention for Native 2K
// Joint Video-Audio Generation Model Training" (page paper.rainbus.top, section
// "方法步骤详情"): the whole query tile stays on chip, only the key blocks of
// S_i are visited, the softmax is online (running max xi and running sum
// zeta), and the output is scattered back to the original token order.
//
// Design (B200): one CTA per 128-token query tile.  The plan's tile list gives,
// for the tile, the 128-token key tiles to visit with a 4-bit mask (which
// 64-token query half attends to which 64-token key half).  Per key tile:
//   TMA (128B swizzle) K (2-stage ring) and V (one buffer), fp16 block-ordered copies
//   tcgen05.mma S = Q K^T into TMEM (double-buffered, 2 x 128 columns)
//   8 softmax warps (2 per TMEM lane quarter, 64 keys each) read S, mask, update the
//     running max (rescaling O in TMEM only when it grows by more than 2^8),
//     write P = 2^(s - m) as fp16 into TMEM
//   tcgen05.mma O += P V (P read from TMEM, V from shared memory) into TMEM
// Warp roles: 0-7 softmax/epilogue (two warpgroups, one per 64-key half),
// 8 TMA producer (and TMEM allocator), 9 MMA issuer.  Every barrier wait is bounded (PRISM_ERR_TIMEOUT).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "prism_dev.cuh"
#include "prism_internal.h"

namespace prism {

constexpr int FWD_STAGES = 2;
#ifndef PRISM_RESCALE_LOG2
#define PRISM_RESCALE_LOG2 0.0f
#endif
// O is rescaled whenever a row max grows by more than this (log2 units).
// A lazy threshold (P up to 2^8 between rescales) measured ~3x the output
// error of exact rescaling on these kernels, so the default is exact.
constexpr float kRescaleLog2 = PRISM_RESCALE_LOG2;
constexpr float kPScaleLog2 = 15.f;   // P operand scale 2^15 (<= 32768 < fp16 max)
constexpr int SLAB = 128 * 64 * 2;   // bytes of a 128-row x 64-column fp16 slab

template <int HD>
struct FwdSmem {
    static constexpr int NSL = HD / 64;
    alignas(1024) uint8_t q[NSL][SLAB];
    alignas(1024) uint8_t k[FWD_STAGES][NSL][SLAB];
    alignas(1024) uint8_t v[NSL][SLAB];           // one V tile: PV_j runs long after QK_j+1
    alignas(1024) uint8_t p[2][2][SLAB];          // [buffer][64-key slab]
    uint64_t bar_q;
    uint64_t k_full[FWD_STAGES], k_empty[FWD_STAGES];
    uint64_t v_full, v_empty;
    uint64_t s_full[2], p_full[2], pv_done[2];
    float pmax[2][2][128];                        // [step parity][warpgroup][row] partial max
    float psum[2][128];                           // [warpgroup][row] partial sum (epilogue)
    uint32_t tmem_base;
    int abort;
};

struct FwdArgs {
    const int* qt_ptr;     // [heads][NT + 1]
    const int* qt_ent;     // [heads][NT * NT]
    const int* src;        // [heads][N]
    void* O;               // [heads][N][HD] raster order
    float* lse;            // [heads][N]
    int64_t N;
    int NT;
    int out_f32;
    float scale_log2;      // log2(e) / sqrt(HD)
    int* err;
};

template <int HD>
__global__ void __launch_bounds__(320, 1)
k_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, FwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<HD>& sm = *reinterpret_cast<FwdSmem<HD>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSL = HD / 64;
    const int t = blockIdx.x, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int* ents = a.qt_ent + (size_t)h * a.NT * a.NT;
    const int e0 = a.qt_ptr[(size_t)h * (a.NT + 1) + t];
    const int n = a.qt_ptr[(size_t)h * (a.NT + 1) + t + 1] - e0;
    ents += e0;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < FWD_STAGES; ++s) { mbar_init(&sm.k_full[s], 1); mbar_init(&sm.k_empty[s], 1); }
        mbar_init(&sm.v_full, 1);
        mbar_init(&sm.v_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], 256);
            mbar_init(&sm.pv_done[b], 1);
        }
        sm.abort = 0;
        mbar_fence_init();
    }
    // warps 0-7: two softmax warpgroups (same 128 query rows; warpgroup g takes
    // the 64 keys of key half g of every tile); warp 8: TMA producer + TMEM
    // allocator; warp 9: MMA issuer.
    constexpr int W_PROD = 8, W_MMA = 9;
    if (warp == W_PROD) {
        __syncwarp();
        tmem_alloc(&sm.tmem_base, 512);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // TMEM columns: S double-buffered at 0 and 128, O at 256 (HD columns)
    constexpr uint32_t TS = 0, TO = 256;
    const int64_t qrow0 = (int64_t)h * a.N + (int64_t)t * 128;

    if (warp == W_PROD) {
        // ------------------------------------------------ TMA producer
        // lane 0 streams Q and the K ring, lane 1 the V ring
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&sm.bar_q, NSL * SLAB);
            for (int c = 0; c < NSL; ++c) tma_load_2d(sm.q[c], &tm_q, &sm.bar_q, 64 * c, (int)qrow0);
            for (int j = 0; j < n; ++j) {
                const int s = j % FWD_STAGES;
                if (j >= FWD_STAGES &&
                    !mbar_wait(&sm.k_empty[s], ((j / FWD_STAGES) - 1) & 1, a.err, 401)) break;
                const int krow = (int)((int64_t)h * a.N + (int64_t)(ents[j] >> 4) * 128);
                mbar_expect_tx(&sm.k_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_2d(sm.k[s][c], &tm_k, &sm.k_full[s], 64 * c, krow);
            }
        } else if (lane == 1 && n > 0) {
            for (int j = 0; j < n; ++j) {
                if (j >= 1 && !mbar_wait(&sm.v_empty, (j - 1) & 1, a.err, 402)) break;
                const int krow = (int)((int64_t)h * a.N + (int64_t)(ents[j] >> 4) * 128);
                mbar_expect_tx(&sm.v_full, NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_2d(sm.v[c], &tm_v, &sm.v_full, 64 * c, krow);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_qk = idesc_f16(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_f16(128, HD, 0, 1);
            // descriptor low words; every K step below adds an immediate
            const uint32_t qA = desc_lo(smem_u32(sm.q[0]), 16);
            const uint32_t vT = desc_lo(smem_u32(sm.v[0]), SLAB);
            bool ok = mbar_wait(&sm.bar_q, 0, a.err, 501);
            for (int j = 0; ok && j <= n; ++j) {
                if (j < n) {
                    const int s = j % FWD_STAGES, b = j & 1;
                    if (!mbar_wait(&sm.k_full[s], (j / FWD_STAGES) & 1, a.err, 502)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kB = desc_lo(smem_u32(sm.k[s][0]), 16);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + TS + 128 * b, desc_from_lo(qA + kmajor_step(kk, SLAB)),
                                 desc_from_lo(kB + kmajor_step(kk, SLAB)), idesc_qk, kk > 0);
                    umma_commit(&sm.s_full[b]);
                    umma_commit(&sm.k_empty[s]);
                }
                if (j >= 1) {
                    const int jj = j - 1, b = jj & 1;
                    if (!mbar_wait(&sm.p_full[b], (jj >> 1) & 1, a.err, 503)) { ok = false; break; }
                    if (!mbar_wait(&sm.v_full, jj & 1, a.err, 504)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t pA = desc_lo(smem_u32(sm.p[b][0]), 16);
                    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + TO, desc_from_lo(pA + kmajor_step(kk, SLAB)),
                                 desc_from_lo(vT + mnmajor_step(kk)), idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.pv_done[b]);
                    umma_commit(&sm.v_empty);
                }
            }
            if (!ok) sm.abort = 1;
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // tcgen05.ld/st are warp-collective (.sync.aligned): every decision that
        // guards one is made warp-uniform (__all_sync / __any_sync).  The two
        // warps sharing a TMEM lane quarter (w and w + 4) combine their row maxima
        // through shared memory and a 64-thread named barrier, so both take the
        // same rescaling decisions.
        const int wg = warp >> 2;                  // key half handled by this warpgroup
        const int r = (warp & 3) * 32 + lane;      // query row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int pair_bar = 1 + (warp & 3);
        const int qh = r >> 6;                     // uniform per warp (32 | 64)
        constexpr int OC = HD / 2;                 // O columns rescaled / written per warpgroup
        const uint32_t ocol = TO + OC * wg;
        float m_ref = -INFINITY, l = 0.f;          // l: this warpgroup's share of the row sum
        bool ok = true;
        int nbar = 0;                              // pair barriers taken in the loop
        for (int j = 0; j < n; ++j) {
            const int b = j & 1;
            const int msk = ents[j] & 15;
            const bool valid = (msk >> (qh * 2 + wg)) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (j >> 1) & 1, a.err, 1))) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            PRISM_TMEM_LD32(tmem + lane_off + TS + 128 * b + 64 * wg, (sr + 0));
            PRISM_TMEM_LD32(tmem + lane_off + TS + 128 * b + 64 * wg + 32, (sr + 32));
            tmem_wait_ld();
            float mx = -INFINITY;
            if (valid) {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                #pragma unroll
                for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sr[c]));
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            }
            mx *= a.scale_log2;
            sm.pmax[j & 1][wg][r] = mx;
            named_bar(pair_bar, 64);
            ++nbar;
            mx = fmaxf(mx, sm.pmax[j & 1][wg ^ 1][r]);
            const float m_new = fmaxf(m_ref, mx);
            const bool first = (j == 0) || (m_ref == -INFINITY);
            const bool need = !first && (m_new > m_ref + kRescaleLog2);
            if (first) m_ref = m_new;
            const bool rescale = __any_sync(0xffffffffu, need);
            if (rescale) {
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err, 2))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = need ? ex2(m_ref - m_new) : 1.f;
                #pragma unroll
                for (int c = 0; c < OC / 32; ++c) {
                    uint32_t o[32];
                    PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * c, o);
                    tmem_wait_ld();
                    #pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    PRISM_TMEM_ST32(tmem + lane_off + ocol + 32 * c, o);
                }
                if (need) { l *= f; m_ref = m_new; }
            }
            if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[b], ((j - 2) >> 1) & 1, a.err, 3))) {
                ok = false;
                break;
            }
            // P is formed as 2^15 * 2^(s - m): the fp16 operand of the PV product then
            // holds probabilities down to 2^-29 as normal numbers (the near-uniform rows
            // of a 1M-token head sit near 1e-6, fp16's subnormal range), and the
            // 2^15 cancels in O = acc / l because l sums the same scaled values.
            const float neg = kPScaleLog2 - m_ref;
            const uint32_t p_s = smem_u32(sm.p[b][wg]);
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
            #pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t w[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = ch * 8 + 2 * e;
                    float p0 = 0.f, p1 = 0.f;
                    if (valid) {
                        p0 = ex2(fmaf(__uint_as_float(sr[c]), a.scale_log2, neg));
                        p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), a.scale_log2, neg));
                    }
                    l4[e] += p0 + p1;
                    w[e] = pack_f16(p0, p1);
                }
                st_shared_v4(p_s + swz128(r, ch), w[0], w[1], w[2], w[3]);
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            fence_proxy_async_smem();
            if (rescale) tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
        }
        // epilogue: both warpgroups add their row sums, each writes half of O
        const int row_perm = t * 128 + r;
        const int dst = a.src[(size_t)h * a.N + row_perm];
        const size_t orow = (size_t)h * a.N + (size_t)dst;
        // A warp that left the loop on a failed wait still takes the pair barriers
        // its partner will take (one per tile, then the epilogue's), so the
        // partner is never left at a barrier.
        for (; nbar < n; ++nbar) named_bar(pair_bar, 64);
        bool fin = false;
        if (ok && n > 0)
            fin = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, a.err, 4));
        sm.psum[wg][r] = l;
        named_bar(pair_bar, 64);
        if (fin) {
            const float lt = sm.psum[0][r] + sm.psum[1][r];
            tc_fence_after();
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            #pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
                uint32_t o[32];
                PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * c, o);
                tmem_wait_ld();
                const int c0 = OC * wg + 32 * c;
                if (a.out_f32) {
                    float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow * HD + c0);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e)
                        op[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                            __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
                } else {
                    uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) + orow * HD + c0);
                    #pragma unroll
                    for (int e = 0; e < 4; ++e)
                        op[e] = make_uint4(pack_bf16(__uint_as_float(o[8 * e]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
                }
            }
            if (wg == 0)
                a.lse[orow] = lt > 0.f ? (m_ref - kPScaleLog2) * 0.69314718055994531f + logf(lt) : -INFINITY;
        } else if (n == 0) {
            for (int c = OC * wg; c < OC * wg + OC; ++c) {
                if (a.out_f32) static_cast<float*>(a.O)[orow * HD + c] = 0.f;
                else static_cast<__nv_bfloat16*>(a.O)[orow * HD + c] = __float2bfloat16(0.f);
            }
            if (wg == 0) a.lse[orow] = -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == W_PROD) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing
// ever arrives at.  The bounded wait gives up after kWaitNs, records
// PRISM_ERR_TIMEOUT (site 9001) in the error word and the kernel returns.
__global__ void k_selftest_wait(int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, err, 9001);
}

template <int HD>
static int launch_fwd(prism_plan_s* P, void* O, float* lse, cudaStream_t s) {
    const Geom& g = P->g;
    FwdArgs a;
    char* b = P->ws;
    a.qt_ptr = (const int*)(b + P->L.qt_ptr);
    a.qt_ent = (const int*)(b + P->L.qt_ent);
    a.src = (const int*)(b + P->L.src);
    a.O = O;
    a.lse = lse;
    a.N = g.N;
    a.NT = g.NT;
    a.out_f32 = P->p.out_dtype == PRISM_F32;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
    a.err = (int*)(b + P->L.err);
    const int smem = (int)sizeof(FwdSmem<HD>) + 1024;
    if (cudaFuncSetAttribute(k_attn_fwd<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PRISM_ERR_CUDA;
    {
        PrismProf prof(P, PRISM_STAGE_FWD, s);
        k_attn_fwd<HD><<<dim3(g.NT, g.heads), 320, smem, s>>>(P->tm_q, P->tm_k, P->tm_v, a);
    }
    P->launches += 1;
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

}  // namespace prism

int prism_launch_selftest_wait(prism_plan_s* P, void* stream) {
    prism::k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((int*)(P->ws + P->L.err));
    P->launches += 1;
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_launch_attn_fwd(prism_plan_s* P, void* O, float* lse, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return P->g.D == 128 ? prism::launch_fwd<128>(P, O, lse, s) : prism::launch_fwd<64>(P, O, lse, s);
}
