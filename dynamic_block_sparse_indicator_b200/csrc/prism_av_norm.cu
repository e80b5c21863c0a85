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
// 128-token tile of the audio keys; the sum of squares of the normalised
// outputs accumulates in registers over the heads, so the map is written once
// per token with no atomics and no second pass.
//   Two softmax warpgroups take alternate heads (group g: heads g, g + 2, ...),
//     each thread one video token (TMEM lane) with all 128 keys of a step, its
//     own running max and sum (O rescaled in TMEM only when the max grows by
//     more than 2^8) and its group's O accumulator: the groups never exchange
//     anything inside the walk, so one group's exponentials overlap the other
//     group's products.  The steps interleave a pair of heads tile by tile.
//   TMA (128B swizzle, 3-D maps [heads][rows][D] whose out-of-range rows read
//     as zeros): Q of each group's head, K and V tiles (two-stage rings);
//   tcgen05.mma S = Q K^T into the group's 128 TMEM columns; the softmax
//     writes P = 2^(s - m) as bf16 over the S columns it has read;
//   tcgen05.mma O_g += P V with P read from TMEM, V from shared memory.  At a
//     head's end the group reads O_g into registers, frees the accumulator
//     for its next head at once, then normalises, squares and stores.
// Warp roles: 0-7 softmax and epilogue (two groups), 8 TMA producer (and TMEM
// allocator), 9 MMA issuer.  Every barrier wait is bounded (PRISM_ERR_TIMEOUT
// with a site).
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

// Max over the first kv (0..64) of a row's 64 logits held as bits.
__device__ __forceinline__ float row_max(const uint32_t* sr, int kv) {
    if (kv >= 64) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        #pragma unroll
        for (int c = 0; c < 64; c += 2)
            m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
        return fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
    }
    float mx = -INFINITY;
    #pragma unroll
    for (int c = 0; c < 64; ++c)
        if (c < kv) mx = fmaxf(mx, __uint_as_float(sr[c]));
    return mx;
}

// P = 2^(s * scale_log2 + neg) of a row's 64 keys as 32 packed bf16 pairs (zero
// past the first kv keys); returns the sum of the values.
__device__ __forceinline__ float exp_half(const uint32_t* sr, int kv, float scale_log2, float neg, uint32_t* pk) {
    float l4[4] = {0.f, 0.f, 0.f, 0.f};      // two packed pairs of partial sums
    if (kv >= 64) {
        #pragma unroll
        for (int e = 0; e < 32; ++e) {
            float x0, x1;
            ffma2(x0, x1, __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]), scale_log2, scale_log2, neg,
                  neg);
            const float p0 = ex2(x0), p1 = ex2(x1);
            const int q = (e & 1) * 2;
            add2(l4[q], l4[q + 1], l4[q], l4[q + 1], p0, p1);
            pk[e] = pack_bf16(p0, p1);
        }
    } else {
        #pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float p0 = 2 * e < kv ? ex2(fmaf(__uint_as_float(sr[2 * e]), scale_log2, neg)) : 0.f;
            const float p1 = 2 * e + 1 < kv ? ex2(fmaf(__uint_as_float(sr[2 * e + 1]), scale_log2, neg)) : 0.f;
            l4[e & 3] += p0 + p1;
            pk[e] = pack_bf16(p0, p1);
        }
    }
    return (l4[0] + l4[1]) + (l4[2] + l4[3]);
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
    uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];   // [group]
    float pn[2][128];          // [group][row] sum of squares over the group's heads
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

// Step j of the CTA's walk -> (head, key tile).  The two softmax groups take
// alternate heads (group g: heads g, g + 2, ...); the steps interleave a pair
// of heads tile by tile (head 2p tile 0, head 2p + 1 tile 0, head 2p tile 1,
// ...), and an odd last head runs its tiles alone.
__device__ __forceinline__ void step_of(int j, int MT, int heads, int& h, int& kt) {
    const int full = (heads >> 1) * 2 * MT;
    if (j < full) {
        const int p = j / (2 * MT), rem = j - p * 2 * MT;
        kt = rem >> 1;
        h = 2 * p + (rem & 1);
    } else {
        kt = j - full;
        h = heads - 1;
    }
}

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
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.pv_done[i], 1);
            mbar_init(&sm.o_free[i], 128);
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
    // TMEM columns: group g's S (then its bf16 P over the first 64 columns) at
    // 128 g, group g's O at 256 + HD g
    constexpr uint32_t TO = 256;

    if (warp == W_PROD) {
        // ------------------------------------------------ TMA producer
        // lane 0 streams Q (at each head's first step) and the K ring, lane 1 the V ring
        if (lane == 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
            for (int j = 0; j < J; ++j) {
                int h, kt;
                step_of(j, MT, a.heads, h, kt);
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
                int h, kt;
                step_of(j, MT, a.heads, h, kt);
                const int s = j % STAGES;
                if (j >= STAGES && !mbar_wait(&sm.v_empty[s], ((j / STAGES) - 1) & 1, a.err, 2403)) break;
                mbar_expect_tx(&sm.v_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_3d(sm.v[s][c], &tm_v, &sm.v_full[s], 64 * c, 128 * kt, h);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------ MMA issuer
        // S(j) = Q K(j)^T into group g(j)'s S buffer and O_g += P(j) V(j) from the
        // bf16 P written over that buffer.  One thread's MMAs run in issue order:
        // every S(j) is issued after the PV of group g(j)'s previous step, so it
        // overwrites P only once that product has read it.  n_p[g] counts group g's
        // steps (the phases of its barriers), hc[g] its heads.
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t id_pv = idesc_bf16(128, HD, 0, 1);
            int n_p[2] = {0, 0};
            bool ok = true;
            auto issue_s = [&](int j) {
                int h, kt;
                step_of(j, MT, a.heads, h, kt);
                const int g = h & 1, s = j % STAGES;
                if (kt == 0 && !mbar_wait(&sm.q_full[g], (h >> 1) & 1, a.err, 2501)) return false;
                if (!mbar_wait(&sm.k_full[s], (j / STAGES) & 1, a.err, 2502)) return false;
                tc_fence_after();
                const uint32_t qA = desc_lo(smem_u32(sm.q[g][0]), 16);
                const uint32_t kB = desc_lo(smem_u32(sm.k[s][0]), 16);
                #pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_f16(tmem + 128 * g, desc_from_lo(qA + kmajor_step(kk, SLAB)),
                             desc_from_lo(kB + kmajor_step(kk, SLAB)), id_qk, kk > 0);
                umma_commit(&sm.s_full[g]);
                umma_commit(&sm.k_empty[s]);
                if (kt == MT - 1) umma_commit(&sm.q_empty[g]);
                return true;
            };
            auto issue_pv = [&](int j) {
                int h, kt;
                step_of(j, MT, a.heads, h, kt);
                const int g = h & 1, s = j % STAGES;
                if (!mbar_wait(&sm.p_full[g], n_p[g] & 1, a.err, 2503)) return false;
                if (!mbar_wait(&sm.v_full[s], (j / STAGES) & 1, a.err, 2504)) return false;
                // the first product of the group's next head overwrites O_g: the
                // group's epilogue must have read the previous head's O first
                if (kt == 0 && h >= 2 && !mbar_wait(&sm.o_free[g], ((h >> 1) - 1) & 1, a.err, 2505)) return false;
                tc_fence_after();
                const uint32_t vT = desc_lo(smem_u32(sm.v[s][0]), SLAB);
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ts(tmem + TO + HD * g, tmem + 128 * g + 8 * kk, desc_from_lo(vT + mnmajor_step(kk)),
                                id_pv, (kt > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.pv_done[g]);
                umma_commit(&sm.v_empty[s]);
                ++n_p[g];
                return true;
            };
            for (int j = 0; ok && j <= J; ++j) {
                // S(j) and PV(j - 1): PV first when both belong to one group (an odd
                // last head), so S(j) never overwrites a P that is still to be read
                int hj = 0, hp = 0, kt_;
                if (j < J) step_of(j, MT, a.heads, hj, kt_);
                if (j >= 1) step_of(j - 1, MT, a.heads, hp, kt_);
                const bool same = j >= 1 && j < J && (hj & 1) == (hp & 1);
                if (same) ok = issue_pv(j - 1) && issue_s(j);
                else {
                    if (j < J) ok = issue_s(j);
                    if (ok && j >= 1) ok = issue_pv(j - 1);
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax + epilogue
        // Group g (warps 4g .. 4g + 3) takes heads g, g + 2, ...: a thread is one
        // video token (TMEM lane) with all 128 keys of every step of its group,
        // its own running max and sum, and the group's O accumulator, so the
        // groups never wait for each other inside the walk.  O is rescaled only
        // when the running max grows by more than 2^8 (bf16 P keeps fp32's
        // exponent range).  tcgen05.ld/st are warp-collective: every decision
        // guarding one is warp-uniform.
        const int g = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t scol = 128 * g, ocol = TO + HD * g;
        const int64_t row = (int64_t)t * 128 + r;
        const bool row_ok = row < a.N;
        float nsq = 0.f;
        bool ok = true;
        int c = 0;                                  // the group's steps so far (barrier phases)
        for (int h = g; ok && h < a.heads; h += 2) {
            float m_ref = -INFINITY, l = 0.f;
            for (int kt = 0; kt < MT; ++kt, ++c) {
                const int kv0 = min(max(a.M - kt * 128, 0), 64);          // valid keys of half 0 (uniform)
                const int kv1 = min(max(a.M - kt * 128 - 64, 0), 64);     // and of half 1
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[g], c & 1, a.err, 2002))) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[64];
                float mx = -INFINITY;
                PRISM_TMEM_LD32(tmem + lane_off + scol, (sr + 0));
                PRISM_TMEM_LD32(tmem + lane_off + scol + 32, (sr + 32));
                tmem_wait_ld();
                mx = row_max(sr, kv0);
                PRISM_TMEM_LD32(tmem + lane_off + scol + 64, (sr + 0));  // half 1 stays in registers
                PRISM_TMEM_LD32(tmem + lane_off + scol + 96, (sr + 32));
                tmem_wait_ld();
                mx = fmaxf(mx, row_max(sr, kv1));
                mx *= a.scale_log2;
                if (kt == 0) {
                    m_ref = mx;                     // a new head: its first tile sets the reference
                } else {
                    const float m_new = fmaxf(m_ref, mx);
                    const bool need = m_new > m_ref + kRescaleLog2;
                    if (__any_sync(0xffffffffu, need)) {
                        // O_g holds the products up to this group's previous step
                        if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[g], (c - 1) & 1, a.err, 2003))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float f = need ? ex2(m_ref - m_new) : 1.f;
                        #pragma unroll
                        for (int cc = 0; cc < HD / 32; ++cc) {
                            uint32_t o[32];
                            PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * cc, o);
                            tmem_wait_ld();
                            #pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                            PRISM_TMEM_ST32(tmem + lane_off + ocol + 32 * cc, o);
                        }
                        if (need) { l *= f; m_ref = m_new; }
                    }
                }
                const float neg = -m_ref;
                uint32_t pk1[32], pk0[32];
                l += exp_half(sr, kv1, a.scale_log2, neg, pk1);
                PRISM_TMEM_LD32(tmem + lane_off + scol, (sr + 0));       // half 0 again
                PRISM_TMEM_LD32(tmem + lane_off + scol + 32, (sr + 32));
                tmem_wait_ld();
                l += exp_half(sr, kv0, a.scale_log2, neg, pk0);
                // P (bf16, two keys per column) over the S columns just read
                PRISM_TMEM_ST32(tmem + lane_off + scol, pk0);
                PRISM_TMEM_ST32(tmem + lane_off + scol + 32, pk1);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_full[g]);
            }
            if (!ok) break;
            // epilogue of head h: O_g into registers, the accumulator freed at once
            // for the group's next head, then normalised, squared and stored
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[g], (c - 1) & 1, a.err, 2001))) { ok = false; break; }
            tc_fence_after();
            uint32_t o[HD];
            #pragma unroll
            for (int cc = 0; cc < HD / 32; ++cc) PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * cc, (o + 32 * cc));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.o_free[g]);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            float acc = 0.f;
            #pragma unroll
            for (int cc = 0; cc < HD / 32; ++cc) {
                float x[32];
                #pragma unroll
                for (int e = 0; e < 32; ++e) {
                    x[e] = __uint_as_float(o[32 * cc + e]) * inv;
                    acc = fmaf(x[e], x[e], acc);
                }
                if (a.hhat && row_ok) {
                    const size_t base = ((size_t)h * a.N + (size_t)row) * HD + 32 * cc;
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
        }
        // the two groups' sums of squares of each token meet once (every warp
        // takes this barrier, on success or after a failed wait)
        sm.pn[g][r] = nsq;
        named_bar(1 + (warp & 3), 64);
        if (ok && g == 0 && row_ok) a.amap[row] = sqrtf(sm.pn[0][r] + sm.pn[1][r]);
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
