// prism_av_norm.cu -- the guidance map's producer on sm_100a tensor cores.
//
// a_{t,h,w} = || h_hat_{t,h,w} ||_2 with h_hat = CrossAttn(h, K_a, V_a): per
// head, softmax(q K_a^T / sqrt(D)) V_a over the audio tokens, the heads
// concatenated, before the output projection ("Prism: Dynamic Sparse Attention
// for Native 2K Joint Video-Audio Generation Model Training", page
// paper.rainbus.top, section "前置知识", the dual-branch DiT paragraph; page
// xyznot.com/id, section "Metode" 1, where the next layer's plan reads the map
// cached from this one).  The audio sequence is short (under 1K tokens: page
// xyznot.com/th, section "คำถามที่พบบ่อย"), the video sequence about 1M tokens,
// so the work is a dense contraction of 4 N M D flops per head, tensor-bound.
//
// Design (B200): one CTA per 128 video tokens walks every head and every
// 128-token tile of the audio keys ("steps" j = head * MT + key tile); the sum
// of squares of the normalised outputs accumulates in registers over the heads,
// so the map is written once per token with no atomics and no second pass.
//   TMA (128B swizzle, 3-D maps [heads][rows][D] whose out-of-range rows read
//     as zeros): Q of the head (two buffers: the next head's Q loads while this
//     head's keys stream), K and V tiles (two-stage rings each);
//   tcgen05.mma S = Q K^T into TMEM (two buffers of 128 columns);
//   8 softmax warps (two warpgroups, one per 64-key half; TMEM lane = video
//     token) mask the keys past M, keep a running max per row (O is rescaled
//     in TMEM only when the max grows by more than 2^8), write P = 2^(s - m)
//     as bf16 into TMEM over the S columns they have read;
//   tcgen05.mma O += P V with P read from TMEM, V from shared memory, into one
//     of two O accumulators (heads alternate), so the softmax warps normalise
//     and square one head's O while the next head's products run.
// Warp roles: 0-7 softmax and epilogue, 8 TMA producer (and TMEM allocator),
// 9 MMA issuer.  Every barrier wait is bounded (PRISM_ERR_TIMEOUT with a site).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "prism_dev.cuh"
#include "prism_internal.h"

namespace prism {
namespace av {

constexpr int STAGES = 2;               // K and V ring depth
constexpr int SLAB = 128 * 64 * 2;      // 128 rows x 64 bf16 columns (128-byte rows)
constexpr float kRescaleLog2 = 8.f;     // bf16 P holds 2^8 without loss of relative precision

// 3-D TMA tile load: coordinates (x = column, y = row, z = head).
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)),
           "r"(x), "r"(y), "r"(z) : "memory");
}

__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Instruction descriptor, kind::f16 with bf16 A and B, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int HD>
struct Smem {
    static constexpr int NSL = HD / 64;
    alignas(1024) uint8_t q[2][NSL][SLAB];
    alignas(1024) uint8_t k[STAGES][NSL][SLAB];
    alignas(1024) uint8_t v[STAGES][NSL][SLAB];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[STAGES], k_empty[STAGES];
    uint64_t v_full[STAGES], v_empty[STAGES];
    uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
    float pmax[2][2][128];     // [step parity][warpgroup][row] partial row max
    float psum[2][128];        // [warpgroup][row] partial row sum of the finished head
    float pn[2][128];          // [warpgroup][row] partial sum of squares over the heads
    uint32_t tmem_base;
};

struct Args {
    float* amap;        // [N] fp32
    void* hhat;         // [heads][N][HD] or null
    int64_t N;
    int M, MT, heads;
    int hhat_f32;
    float scale_log2;   // log2(e) / sqrt(HD)
    int* err;
};

template <int HD>
__global__ void __launch_bounds__(320, 1)
k_av_norm(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, Args a) {
    extern __shared__ uint8_t smem_raw[];
    Smem<HD>& sm = *reinterpret_cast<Smem<HD>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSL = HD / 64;
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MT = a.MT, J = a.heads * a.MT;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 256);
            mbar_init(&sm.pv_done[i], 1);
            mbar_init(&sm.o_free[i], 256);
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_fence_init();
    }
    constexpr int W_PROD = 8, W_MMA = 9;
    if (warp == W_PROD) {
        __syncwarp();
        tmem_alloc(&sm.tmem_base, 512);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // TMEM columns: S (then P over its first 64 columns) at 0 and 128; O at 256 and 256 + HD
    constexpr uint32_t TO = 256;

    if (warp == W_PROD) {
        // ------------------------------------------------ TMA producer
        // lane 0 streams Q (at each head's first step) and the K ring, lane 1 the V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
            for (int j = 0; j < J; ++j) {
                const int h = j / MT, kt = j - h * MT;
                if (kt == 0) {
                    const int qb = h & 1;
                    if (h >= 2 && !mbar_wait(&sm.q_empty[qb], ((h >> 1) - 1) & 1, a.err, 2401)) break;
                    mbar_expect_tx(&sm.q_full[qb], NSL * SLAB);
                    for (int c = 0; c < NSL; ++c) tma_load_3d(sm.q[qb][c], &tm_q, &sm.q_full[qb], 64 * c, 128 * t, h);
                }
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&sm.k_empty[s], ((j / STAGES) - 1) & 1, a.err, 2402)) break;
                mbar_expect_tx(&sm.k_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_3d(sm.k[s][c], &tm_k, &sm.k_full[s], 64 * c, 128 * kt, h);
            }
        } else if (lane == 1) {
            for (int j = 0; j < J; ++j) {
                const int h = j / MT, kt = j - h * MT;
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&sm.v_empty[s], ((j / STAGES) - 1) & 1, a.err, 2403)) break;
                mbar_expect_tx(&sm.v_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_3d(sm.v[s][c], &tm_v, &sm.v_full[s], 64 * c, 128 * kt, h);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------ MMA issuer
        // Iteration j issues S(j) = Q K(j)^T, then O += P(j-1) V(j-1).  One thread's
        // MMAs run in issue order, so S(j + 1) overwrites the P(j - 1) columns only
        // after O += P(j - 1) V has read them.
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t id_pv = idesc_bf16(128, HD, 0, 1);
            for (int j = 0; j <= J; ++j) {
                if (j < J) {
                    const int h = j / MT, kt = j - h * MT;
                    const int s = j % STAGES, b = j & 1, qb = h & 1;
                    if (kt == 0 && !mbar_wait(&sm.q_full[qb], (h >> 1) & 1, a.err, 2501)) break;
                    if (!mbar_wait(&sm.k_full[s], (j / STAGES) & 1, a.err, 2502)) break;
                    tc_fence_after();
                    const uint32_t qA = desc_lo(smem_u32(sm.q[qb][0]), 16);
                    const uint32_t kB = desc_lo(smem_u32(sm.k[s][0]), 16);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + 128 * b, desc_from_lo(qA + kmajor_step(kk, SLAB)),
                                 desc_from_lo(kB + kmajor_step(kk, SLAB)), id_qk, kk > 0);
                    umma_commit(&sm.s_full[b]);
                    umma_commit(&sm.k_empty[s]);
                    if (kt == MT - 1) umma_commit(&sm.q_empty[qb]);
                }
                if (j >= 1) {
                    const int jj = j - 1, hh = jj / MT, kt = jj - hh * MT;
                    const int s = jj % STAGES, b = jj & 1, ob = hh & 1;
                    if (!mbar_wait(&sm.p_full[b], (jj >> 1) & 1, a.err, 2503)) break;
                    if (!mbar_wait(&sm.v_full[s], (jj / STAGES) & 1, a.err, 2504)) break;
                    // the first product of head hh overwrites the O of head hh - 2
                    if (kt == 0 && hh >= 2 && !mbar_wait(&sm.o_free[ob], ((hh >> 1) - 1) & 1, a.err, 2505)) break;
                    tc_fence_after();
                    const uint32_t vT = desc_lo(smem_u32(sm.v[s][0]), SLAB);
                    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ts(tmem + TO + HD * ob, tmem + 128 * b + 8 * kk, desc_from_lo(vT + mnmajor_step(kk)),
                                    id_pv, (kt > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.pv_done[b]);
                    umma_commit(&sm.v_empty[s]);
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // tcgen05.ld/st are warp-collective: every decision guarding one is
        // warp-uniform.  The two warps sharing a TMEM lane quarter (w, w + 4)
        // exchange row maxima and sums through shared memory and a 64-thread
        // named barrier.
        const int wg = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int pair_bar = 1 + (warp & 3);
        constexpr int OC = HD / 2;                 // O columns per warpgroup
        const int64_t row = (int64_t)t * 128 + r;
        const bool row_ok = row < a.N;
        float m_ref = -INFINITY, l = 0.f, nsq = 0.f;
        bool ok = true;
        int nbar = 0;                              // pair barriers taken so far

        // Normalise head hp's O (buffer hp & 1, complete once PV of step jl is
        // done), add its squares to nsq, write h_hat if asked, free the buffer.
        auto epilogue = [&](int hp, int jl, float l_hp) {
            bool fin = ok && __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[jl & 1], (jl >> 1) & 1, a.err, 2001));
            sm.psum[wg][r] = l_hp;
            named_bar(pair_bar, 64);
            ++nbar;
            if (!fin) { ok = false; return; }
            tc_fence_after();
            const float lt = sm.psum[0][r] + sm.psum[1][r];
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const uint32_t ocol = TO + HD * (hp & 1) + OC * wg;
            float acc = 0.f;
            #pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
                uint32_t o[32];
                PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * c, o);
                tmem_wait_ld();
                float x[32];
                #pragma unroll
                for (int e = 0; e < 32; ++e) {
                    x[e] = __uint_as_float(o[e]) * inv;
                    acc = fmaf(x[e], x[e], acc);
                }
                if (a.hhat && row_ok) {
                    const size_t base = ((size_t)hp * a.N + (size_t)row) * HD + OC * wg + 32 * c;
                    if (a.hhat_f32) {
                        float4* op = reinterpret_cast<float4*>(static_cast<float*>(a.hhat) + base);
                        #pragma unroll
                        for (int e = 0; e < 8; ++e) op[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    } else {
                        uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.hhat) + base);
                        #pragma unroll
                        for (int e = 0; e < 4; ++e)
                            op[e] = make_uint4(pack_bf16(x[8 * e], x[8 * e + 1]), pack_bf16(x[8 * e + 2], x[8 * e + 3]),
                                               pack_bf16(x[8 * e + 4], x[8 * e + 5]), pack_bf16(x[8 * e + 6], x[8 * e + 7]));
                    }
                }
            }
            nsq += acc;
            tc_fence_before();
            mbar_arrive(&sm.o_free[hp & 1]);
        };

        for (int j = 0; j < J; ++j) {
            const int h = j / MT, kt = j - h * MT, b = j & 1;
            const int kvalid = a.M - kt * 128 - 64 * wg;     // valid keys of this half (warp-uniform)
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (j >> 1) & 1, a.err, 2002))) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 64 * wg, (sr + 0));
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 64 * wg + 32, (sr + 32));
            tmem_wait_ld();
            float mx = -INFINITY;
            if (kvalid >= 64) {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                #pragma unroll
                for (int c = 0; c < 64; c += 2)
                    m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
            } else {
                #pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c < kvalid) mx = fmaxf(mx, __uint_as_float(sr[c]));
            }
            mx *= a.scale_log2;
            sm.pmax[j & 1][wg][r] = mx;
            // both warpgroups have read their S columns past this barrier, so P may
            // overwrite the first 64 of them
            named_bar(pair_bar, 64);
            ++nbar;
            mx = fmaxf(mx, sm.pmax[j & 1][wg ^ 1][r]);
            float l_done = 0.f;
            if (kt == 0) {                 // a new head: its first tile sets the reference
                l_done = l;
                l = 0.f;
                m_ref = mx;
            } else {
                const float m_new = fmaxf(m_ref, mx);
                const bool need = m_new > m_ref + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err, 2003))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float f = need ? ex2(m_ref - m_new) : 1.f;
                    const uint32_t ocol = TO + HD * (h & 1) + OC * wg;
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
            }
            const float neg = -m_ref;
            uint32_t pk[32];
            float l4[4] = {0.f, 0.f, 0.f, 0.f};      // two packed pairs of partial sums
            if (kvalid >= 64) {
                #pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float x0, x1;
                    ffma2(x0, x1, __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]), a.scale_log2,
                          a.scale_log2, neg, neg);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    const int q = (e & 1) * 2;
                    add2(l4[q], l4[q + 1], l4[q], l4[q + 1], p0, p1);
                    pk[e] = pack_bf16(p0, p1);
                }
            } else {
                #pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float p0 = 2 * e < kvalid ? ex2(fmaf(__uint_as_float(sr[2 * e]), a.scale_log2, neg)) : 0.f;
                    const float p1 = 2 * e + 1 < kvalid ? ex2(fmaf(__uint_as_float(sr[2 * e + 1]), a.scale_log2, neg)) : 0.f;
                    l4[e & 3] += p0 + p1;
                    pk[e] = pack_bf16(p0, p1);
                }
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            PRISM_TMEM_ST32(tmem + lane_off + 128 * b + 32 * wg, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
            if (kt == 0 && h > 0) epilogue(h - 1, j - 1, l_done);
            if (!ok) break;
        }
        // A warp that left the loop on a failed wait still takes every pair
        // barrier its partner will take: one per step, one per head epilogue.
        const int nbar_loop = J + a.heads - 1;
        for (; nbar < nbar_loop; ++nbar) named_bar(pair_bar, 64);
        epilogue(a.heads - 1, J - 1, l);           // the last head (takes one more barrier)
        sm.pn[wg][r] = nsq;
        named_bar(pair_bar, 64);
        if (ok && wg == 0 && row_ok) a.amap[row] = sqrtf(sm.pn[0][r] + sm.pn[1][r]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == W_PROD) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// [heads][rows][D] bf16 as a 3-D map with 64-column x 128-row x 1-head boxes
// (128-byte swizzle); rows past `rows` read as zeros.
static int make_map(CUtensorMap* m, const void* base, int64_t rows, int heads, int D) {
    auto enc = encode_fn();
    if (!enc) return PRISM_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

template <int HD>
static int launch(int64_t N, int M, int heads, const void* Qv, const void* Ka, const void* Va, float* amap,
                  void* hhat, int hhat_f32, int* err, cudaStream_t s) {
    CUtensorMap tq, tk, tv;
    int st = make_map(&tq, Qv, N, heads, HD);
    if (!st) st = make_map(&tk, Ka, M, heads, HD);
    if (!st) st = make_map(&tv, Va, M, heads, HD);
    if (st) return st;
    Args a;
    a.amap = amap;
    a.hhat = hhat;
    a.N = N;
    a.M = M;
    a.MT = (M + 127) / 128;
    a.heads = heads;
    a.hhat_f32 = hhat_f32;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
    a.err = err;
    const int smem = (int)sizeof(Smem<HD>) + 1024;
    if (cudaFuncSetAttribute(k_av_norm<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PRISM_ERR_CUDA;
    const int64_t tiles = (N + 127) / 128;
    k_av_norm<HD><<<dim3((unsigned)tiles), 320, smem, s>>>(tq, tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace av
}  // namespace prism

extern "C" int prism_av_norm(int64_t N, int32_t M, int32_t heads, int32_t head_dim, const void* Qv,
                             const void* Ka, const void* Va, float* a_map, void* h_hat, int32_t hhat_dtype,
                             int32_t* dev_status, void* stream) {
    using namespace prism::av;
    if (N < 1 || N > 0x7fffffffLL - 127 || M < 1 || M > (1 << 20) || heads < 1 || heads > 4096 ||
        (head_dim != 64 && head_dim != 128) || (hhat_dtype != PRISM_BF16 && hhat_dtype != PRISM_F32))
        return PRISM_ERR_INVALID_ARG;
    if (!Qv || !Ka || !Va || !a_map || !dev_status) return PRISM_ERR_INVALID_ARG;
    if (!aligned16(Qv) || !aligned16(Ka) || !aligned16(Va) || !aligned16(a_map) || !aligned16(dev_status) ||
        (h_hat && !aligned16(h_hat)))
        return PRISM_ERR_INVALID_ARG;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_UNSUPPORTED;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return PRISM_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int f32 = hhat_dtype == PRISM_F32;
    nvtxRangePushA("prism av norm");
    const int st = head_dim == 128 ? launch<128>(N, M, heads, Qv, Ka, Va, a_map, h_hat, f32, dev_status, s)
                                   : launch<64>(N, M, heads, Qv, Ka, Va, a_map, h_hat, f32, dev_status, s);
    nvtxRangePop();
    return st;
}

extern "C" int prism_status_read(int32_t* dev_status, int32_t* site, void* stream) {
    if (!dev_status) return PRISM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h[4] = {0, 0, 0, 0};
    if (cudaMemcpyAsync(h, dev_status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return PRISM_ERR_CUDA;
    if (site) *site = h[1];
    if (h[0] != 0 && cudaMemsetAsync(dev_status, 0, sizeof(h), s) != cudaSuccess) return PRISM_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
    return h[0];
}
