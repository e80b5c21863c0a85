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
//   TMA (128B swizzle) K, V (fp16 block-ordered copies) -> shared memory (2-stage ring)
//   tcgen05.mma S = Q K^T into TMEM (double-buffered, 2 x 128 columns)
//   4 softmax warps (thread = query row = TMEM lane) read S, mask, update the
//     running max (rescaling O in TMEM only when it grows by more than 2^8),
//     write P = 2^(s - m) as fp16 to shared memory
//   tcgen05.mma O += P V into TMEM (128 + head_dim columns)
// Warp roles: 0-3 softmax/epilogue, 4 TMA producer (and TMEM allocator),
// 5 MMA issuer.  Every barrier wait is bounded (PRISM_ERR_TIMEOUT).
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
    alignas(1024) uint8_t v[FWD_STAGES][NSL][SLAB];
    alignas(1024) uint8_t p[2][2][SLAB];          // [buffer][64-key slab]
    uint64_t bar_q;
    uint64_t kv_full[FWD_STAGES], kv_empty[FWD_STAGES];
    uint64_t s_full[2], p_full[2], pv_done[2];
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
__global__ void __launch_bounds__(192, 1)
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
        for (int s = 0; s < FWD_STAGES; ++s) { mbar_init(&sm.kv_full[s], 1); mbar_init(&sm.kv_empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], 128);
            mbar_init(&sm.pv_done[b], 1);
        }
        sm.abort = 0;
        mbar_fence_init();
    }
    if (warp == 4) {
        __syncwarp();
        tmem_alloc(&sm.tmem_base, 512);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int64_t qrow0 = (int64_t)h * a.N + (int64_t)t * 128;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&sm.bar_q, NSL * SLAB);
            for (int c = 0; c < NSL; ++c) tma_load_2d(sm.q[c], &tm_q, &sm.bar_q, 64 * c, (int)qrow0);
            for (int j = 0; j < n; ++j) {
                const int s = j % FWD_STAGES;
                if (j >= FWD_STAGES &&
                    !mbar_wait(&sm.kv_empty[s], ((j / FWD_STAGES) - 1) & 1, a.err, 401)) break;
                const int kt = ents[j] >> 4;
                const int krow = (int)((int64_t)h * a.N + (int64_t)kt * 128);
                mbar_expect_tx(&sm.kv_full[s], 2 * NSL * SLAB);
                for (int c = 0; c < NSL; ++c) {
                    tma_load_2d(sm.k[s][c], &tm_k, &sm.kv_full[s], 64 * c, krow);
                    tma_load_2d(sm.v[s][c], &tm_v, &sm.kv_full[s], 64 * c, krow);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_qk = idesc_f16(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_f16(128, HD, 0, 1);
            const uint32_t q_s = smem_u32(sm.q[0]);
            bool ok = mbar_wait(&sm.bar_q, 0, a.err, 501);
            for (int j = 0; ok && j <= n; ++j) {
                if (j < n) {
                    const int s = j % FWD_STAGES, b = j & 1;
                    if (!mbar_wait(&sm.kv_full[s], (j / FWD_STAGES) & 1, a.err, 502)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t k_s = smem_u32(sm.k[s][0]);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + 128 * b, desc_kmajor(q_s, kk, SLAB), desc_kmajor(k_s, kk, SLAB),
                                  idesc_qk, kk > 0);
                    umma_commit(&sm.s_full[b]);
                }
                if (j >= 1) {
                    const int jj = j - 1, b = jj & 1, s = jj % FWD_STAGES;
                    if (!mbar_wait(&sm.p_full[b], (jj >> 1) & 1, a.err, 503)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t p_s = smem_u32(sm.p[b][0]);
                    const uint32_t v_s = smem_u32(sm.v[s][0]);
                    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + 256, desc_kmajor(p_s, kk, SLAB), desc_mnmajor(v_s, kk, SLAB),
                                  idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.pv_done[b]);
                    umma_commit(&sm.kv_empty[s]);
                }
            }
            if (!ok) sm.abort = 1;
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // tcgen05.ld/st are warp-collective (.sync.aligned): every decision that
        // guards one is made warp-uniform (__all_sync / __any_sync).
        const int r = threadIdx.x;                 // query row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int qh = r >> 6;                     // uniform per warp (32 | 64)
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int b = j & 1;
            const int msk = ents[j] & 15;
            const bool v0 = (msk >> (qh * 2)) & 1, v1 = (msk >> (qh * 2 + 1)) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (j >> 1) & 1, a.err, 1))) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[128];
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 0, (sr + 0));
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 32, (sr + 32));
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 64, (sr + 64));
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 96, (sr + 96));
            tmem_wait_ld();
            float mx = -INFINITY;
            if (v0) {
                #pragma unroll
                for (int c = 0; c < 64; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
            }
            if (v1) {
                #pragma unroll
                for (int c = 64; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
            }
            mx *= a.scale_log2;
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
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    PRISM_TMEM_LD32(tmem + lane_off + 256 + 32 * c, o);
                    tmem_wait_ld();
                    #pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    PRISM_TMEM_ST32(tmem + lane_off + 256 + 32 * c, o);
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
            const uint32_t p_s = smem_u32(sm.p[b][0]);
            #pragma unroll
            for (int half = 0; half < 2; ++half) {
                const bool valid = half ? v1 : v0;
                #pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t w[4];
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = half * 64 + ch * 8 + 2 * e;
                        float p0 = 0.f, p1 = 0.f;
                        if (valid) {
                            p0 = ex2(fmaf(__uint_as_float(sr[c]), a.scale_log2, neg));
                            p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), a.scale_log2, neg));
                        }
                        l += p0 + p1;
                        w[e] = pack_f16(p0, p1);
                    }
                    st_shared_v4(p_s + half * SLAB + swz128(r, ch), w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            if (rescale) tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
        }
        // epilogue: O / l, scattered to raster order
        const int row_perm = t * 128 + r;
        const int dst = a.src[(size_t)h * a.N + row_perm];
        const size_t orow = (size_t)h * a.N + (size_t)dst;
        bool fin = false;
        if (ok && n > 0)
            fin = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, a.err, 4));
        if (fin) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            #pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                PRISM_TMEM_LD32(tmem + lane_off + 256 + 32 * c, o);
                tmem_wait_ld();
                if (a.out_f32) {
                    float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.O) + orow * HD + 32 * c);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e)
                        op[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                            __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
                } else {
                    uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.O) + orow * HD + 32 * c);
                    #pragma unroll
                    for (int e = 0; e < 4; ++e)
                        op[e] = make_uint4(pack_bf16(__uint_as_float(o[8 * e]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
                                           pack_bf16(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
                }
            }
            a.lse[orow] = l > 0.f ? (m_ref - kPScaleLog2) * 0.69314718055994531f + logf(l) : -INFINITY;
        } else if (n == 0) {
            for (int c = 0; c < HD; ++c) {
                if (a.out_f32) static_cast<float*>(a.O)[orow * HD + c] = 0.f;
                else static_cast<__nv_bfloat16*>(a.O)[orow * HD + c] = __float2bfloat16(0.f);
            }
            a.lse[orow] = -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 4) {
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
        k_attn_fwd<HD><<<dim3(g.NT, g.heads), 192, smem, s>>>(P->tm_q, P->tm_k, P->tm_v, a);
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
