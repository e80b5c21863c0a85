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
// 64-token query half attends to which 64-token key half).  The key tiles
// alternate between two softmax warpgroups: group g takes steps j = g, g + 2,
// ..., each thread one full query row of the step's 128 keys, with its own
// running max and sum and its own O accumulator in TMEM.  The groups never wait
// for each other inside the loop (no per-step exchange of row maxima), so one
// group's exponentials overlap the other's products; the two partial outputs
// are merged once at the end, O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / L.
//   TMA (128B swizzle): Q once, K and V two-stage rings (fp16 block-ordered copies)
//   tcgen05.mma S = Q K^T into TMEM (one 128-column buffer per group), issued by
//     warp 9 as soon as the group has read its previous S (s_free)
//   softmax: row max (exact rescale of the group's O when it grows), P = 2^15
//     2^(s - m) as fp16 into the group's shared-memory buffer
//   tcgen05.mma O_g += P V, issued by warp 10 (a second issuer, so a wait for P
//     never holds back the next S)
// Warp roles: 0-7 softmax (two warpgroups) and epilogue, 8 TMA producer (and
// TMEM allocator), 9 QK issuer, 10 PV issuer.  Every barrier wait is bounded
// (PRISM_ERR_TIMEOUT).  Heads with more than 1,024 key tiles run in passes over
// key-tile ranges (see kFwdKeyChunk) that carry (O, max, sum) per query row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "prism_dev.cuh"
#include "prism_internal.h"

namespace prism {

constexpr int FWD_KST = 2;          // K ring depth
constexpr int FWD_VST = 2;          // V ring depth
#ifndef PRISM_RESCALE_LOG2
#define PRISM_RESCALE_LOG2 0.0f
#endif
// O is rescaled whenever a row max grows by more than this (log2 units).
// A lazy threshold (P up to 2^8 between rescales) measured ~3x the output
// error of exact rescaling on these kernels, so the default is exact.
constexpr float kRescaleLog2 = PRISM_RESCALE_LOG2;
constexpr float kPScaleLog2 = 15.f;   // P operand scale 2^15 (<= 32768 < fp16 max)
constexpr int SLAB = 128 * 64 * 2;   // bytes of a 128-row x 64-column fp16 slab
constexpr int FWD_THREADS = 352;
// Key tiles per pass.  Every query tile's list is walked in ascending key order;
// over a whole 1M-token head (7,920 key tiles, 518 MB of fp16 K and V) the CTAs in
// flight drift apart along their lists and a third of the K/V tile loads missed
// L2.  A pass visits only 1,024 key tiles (64 MB of K and V, half of L2) for
// every query tile, and merges its (O, max, sum) into a running state that the
// next pass continues; the last pass writes O and LSE.
#ifndef PRISM_FWD_KEY_CHUNK
#define PRISM_FWD_KEY_CHUNK 1024
#endif
constexpr int kFwdKeyChunk = PRISM_FWD_KEY_CHUNK;

template <int HD>
struct FwdSmem {
    static constexpr int NSL = HD / 64;
    alignas(1024) uint8_t q[NSL][SLAB];
    alignas(1024) uint8_t k[FWD_KST][NSL][SLAB];
    alignas(1024) uint8_t v[FWD_VST][NSL][SLAB];
    alignas(1024) uint8_t p[2][2][SLAB];          // [group][64-key slab]; the epilogue's exchange reuses it
    uint64_t bar_q;
    uint64_t k_full[FWD_KST], k_empty[FWD_KST];
    uint64_t v_full[FWD_VST], v_empty[FWD_VST];
    uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
    uint32_t tmem_base;
    int e0, n;                                    // this pass's entries of the tile's list
};

struct FwdArgs {
    const int* qt_ptr;     // [heads][NT + 1]
    const int* lbase;      // index lists; head h's tile list starts at lbase + qt_off[h]
    const int64_t* qt_off; // [heads]
    int h0;                // first head of this launch (grid y = heads h0, h0 + 1, ...)
    const int* src;        // [heads][N]
    TokenRows O;           // row (h, raster token) of the output, a plain tensor or token shards
    float* lse;            // [heads][N]
    int64_t N;
    int NT;
    int out_f32;
    float scale_log2;      // log2(e) / sqrt(HD)
    const uint32_t* qkv_max;  // [heads][3]: the copies' per-head scales (qkv_shift)
    int key_lo, key_hi;    // this pass's key tiles [key_lo, key_hi)
    int first, last;       // first pass (no state to merge), last pass (write O and LSE)
    float* st_o;           // [group heads][N][HD] running O (unnormalised, relative to 2^m), block order
    float* st_m;           // [heads][N] running max (log2 units, P scale included)
    float* st_l;           // [heads][N] running sum
    int* err;
};

// First index in the ascending list e[0, n) whose tile (entry >> 4) is >= key.
__device__ __forceinline__ int fwd_lower_bound(const int* e, int n, int key) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((e[mid] >> 4) < key) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max over 64 fp32 values held as bits
__device__ __forceinline__ float max64(const uint32_t* sr) {
    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll
    for (int c = 0; c < 64; c += 2)
        m4[(c >> 1) & 3] = fmax3f(m4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
    return fmax3f(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
}

__device__ __forceinline__ void add2f(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// P' = 2^(s * scale_log2 + neg) for one row's 64 keys as 32 packed fp16 pairs
// (zeros when the key half is masked); returns the sum of the values.
__device__ __forceinline__ float exp_p64(const uint32_t* sr, bool valid, float scale_log2, float neg,
                                         uint32_t* pk) {
    float l2[2] = {0.f, 0.f};
    #pragma unroll
    for (int e = 0; e < 32; ++e) {
        float p0 = 0.f, p1 = 0.f;
        if (valid) {
            float x0, x1;
            ffma2(x0, x1, __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]), scale_log2, scale_log2, neg,
                  neg);
            p0 = ex2(x0);
            p1 = ex2(x1);
        }
        add2f(l2[0], l2[1], l2[0], l2[1], p0, p1);
        pk[e] = pack_f16(p0, p1);
    }
    return l2[0] + l2[1];
}

// 32 packed pairs (64 keys) of row r into a 128B-swizzled shared-memory slab.
__device__ __forceinline__ void store_p64(const uint32_t* pk, uint32_t slab_s, int r) {
    #pragma unroll
    for (int ch = 0; ch < 8; ++ch)
        st_shared_v4(slab_s + swz128(r, ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
}

template <int HD>
__global__ void __launch_bounds__(FWD_THREADS, 1)
k_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, FwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<HD>& sm = *reinterpret_cast<FwdSmem<HD>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSL = HD / 64;
    const int t = blockIdx.x, h = a.h0 + blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        // this pass visits the key tiles of [key_lo, key_hi) of the tile's ascending list
        const int p0 = a.qt_ptr[(size_t)h * (a.NT + 1) + t];
        const int n0 = a.qt_ptr[(size_t)h * (a.NT + 1) + t + 1] - p0;
        const int* all = a.lbase + a.qt_off[h] + p0;
        const int lo = fwd_lower_bound(all, n0, a.key_lo);
        sm.e0 = p0 + lo;
        sm.n = fwd_lower_bound(all, n0, a.key_hi) - lo;
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < FWD_KST; ++s) { mbar_init(&sm.k_full[s], 1); mbar_init(&sm.k_empty[s], 1); }
        for (int s = 0; s < FWD_VST; ++s) { mbar_init(&sm.v_full[s], 1); mbar_init(&sm.v_empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.s_free[b], 128);
            mbar_init(&sm.p_full[b], 128);
            mbar_init(&sm.pv_done[b], 1);
        }
        mbar_fence_init();
    }
    constexpr int W_PROD = 8, W_QK = 9, W_PV = 10;
    if (warp == W_PROD) {
        __syncwarp();
        tmem_alloc(&sm.tmem_base, 512);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int n = sm.n;
    // the copies carry Q 2^sq, K 2^sk, V 2^sv: the logits' scale and O undo them
    const int sq = qkv_shift(a.qkv_max[h * 3]), sk = qkv_shift(a.qkv_max[h * 3 + 1]);
    const float scale_log2 = ldexpf(a.scale_log2, -(sq + sk));
    const float o_unscale = ldexpf(1.f, -qkv_shift(a.qkv_max[h * 3 + 2]));
    const int* ents = a.lbase + a.qt_off[h] + sm.e0;
    // TMEM columns: S of group g at 128 g; O of group g at 256 + HD g
    constexpr uint32_t TO = 256;
    const int64_t qrow0 = (int64_t)h * a.N + (int64_t)t * 128;

    if (warp == W_PROD) {
        // ------------------------------------------------ TMA producer
        // lane 0 streams Q and the K ring, lane 1 the V ring
        if (lane == 0 && n > 0) {
            tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&sm.bar_q, NSL * SLAB);
            for (int c = 0; c < NSL; ++c) tma_load_2d(sm.q[c], &tm_q, &sm.bar_q, 64 * c, (int)qrow0);
            for (int j = 0; j < n; ++j) {
                const int s = j % FWD_KST;
                if (j >= FWD_KST &&
                    !mbar_wait(&sm.k_empty[s], ((j / FWD_KST) - 1) & 1, a.err, 401)) break;
                int kt = ents[j] >> 4;
                if (prism_bad_index(a.err, kt >= 0 && kt < a.NT)) kt = 0;           // checking build
                const int krow = (int)((int64_t)h * a.N + (int64_t)kt * 128);
                mbar_expect_tx(&sm.k_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_2d(sm.k[s][c], &tm_k, &sm.k_full[s], 64 * c, krow);
            }
        } else if (lane == 1 && n > 0) {
            for (int j = 0; j < n; ++j) {
                const int s = j % FWD_VST;
                if (j >= FWD_VST &&
                    !mbar_wait(&sm.v_empty[s], ((j / FWD_VST) - 1) & 1, a.err, 402)) break;
                int kt = ents[j] >> 4;
                if (prism_bad_index(a.err, kt >= 0 && kt < a.NT)) kt = 0;           // checking build
                const int krow = (int)((int64_t)h * a.N + (int64_t)kt * 128);
                mbar_expect_tx(&sm.v_full[s], NSL * SLAB);
                for (int c = 0; c < NSL; ++c) tma_load_2d(sm.v[s][c], &tm_v, &sm.v_full[s], 64 * c, krow);
            }
        }
    } else if (warp == W_QK) {
        // ------------------------------------------------ S = Q K^T issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_qk = idesc_f16(128, 128, 0, 0);
            const uint32_t qA = desc_lo(smem_u32(sm.q[0]), 16);
            if (mbar_wait(&sm.bar_q, 0, a.err, 501)) {
                for (int j = 0; j < n; ++j) {
                    const int s = j % FWD_KST, b = j & 1;
                    // group b has read S of its previous step out of TMEM
                    if (j >= 2 && !mbar_wait(&sm.s_free[b], ((j - 2) >> 1) & 1, a.err, 505)) break;
                    if (!mbar_wait(&sm.k_full[s], (j / FWD_KST) & 1, a.err, 502)) break;
                    tc_fence_after();
                    const uint32_t kB = desc_lo(smem_u32(sm.k[s][0]), 16);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + 128 * b, desc_from_lo(qA + kmajor_step(kk, SLAB)),
                                 desc_from_lo(kB + kmajor_step(kk, SLAB)), idesc_qk, kk > 0);
                    umma_commit(&sm.s_full[b]);
                    umma_commit(&sm.k_empty[s]);
                }
            }
        }
    } else if (warp == W_PV) {
        // ------------------------------------------------ O_g += P V issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t idesc_pv = idesc_f16(128, HD, 0, 1);
            for (int j = 0; j < n; ++j) {
                const int s = j % FWD_VST, b = j & 1;
                if (!mbar_wait(&sm.p_full[b], (j >> 1) & 1, a.err, 503)) break;
                if (!mbar_wait(&sm.v_full[s], (j / FWD_VST) & 1, a.err, 504)) break;
                tc_fence_after();
                const uint32_t pA = desc_lo(smem_u32(sm.p[b][0]), 16);
                const uint32_t vT = desc_lo(smem_u32(sm.v[s][0]), SLAB);
                #pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + TO + HD * b, desc_from_lo(pA + kmajor_step(kk, SLAB)),
                             desc_from_lo(vT + mnmajor_step(kk)), idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.pv_done[b]);
                umma_commit(&sm.v_empty[s]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------ softmax + epilogue
        // tcgen05.ld/st are warp-collective: every decision that guards one is
        // warp-uniform (__all_sync / __any_sync).
        const int g = warp >> 2;                   // group: steps j = g, g + 2, ...
        const int r = (warp & 3) * 32 + lane;      // query row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int qh = r >> 6;                     // query half (uniform per warp: 32 | 64)
        const uint32_t scol = 128 * g;             // this group's S columns
        const uint32_t ocol = TO + HD * g;         // this group's O columns
        const uint32_t p_s = smem_u32(sm.p[g][0]);
        float m_ref = -INFINITY, l = 0.f;          // running max (log2 units) and scaled sum
        bool ok = true;
        int cnt = 0;
        for (int j = g; j < n; j += 2, ++cnt) {
            const int msk = ents[j] & 15;
            const bool v0 = (msk >> (qh * 2)) & 1, v1 = (msk >> (qh * 2 + 1)) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[g], (j >> 1) & 1, a.err, 1))) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            float mx = -INFINITY;
            if (v0) {
                PRISM_TMEM_LD32(tmem + lane_off + scol, (sr + 0));
                PRISM_TMEM_LD32(tmem + lane_off + scol + 32, (sr + 32));
                tmem_wait_ld();
                mx = max64(sr);
            }
            if (v1) {                              // key half 1 stays in registers
                PRISM_TMEM_LD32(tmem + lane_off + scol + 64, (sr + 0));
                PRISM_TMEM_LD32(tmem + lane_off + scol + 96, (sr + 32));
                tmem_wait_ld();
                mx = fmaxf(mx, max64(sr));
            }
            mx *= scale_log2;
            const bool first = (cnt == 0) || (m_ref == -INFINITY);
            const float m_new = fmaxf(m_ref, mx);
            if (first) m_ref = m_new;
            const bool need = !first && (m_new > m_ref + kRescaleLog2);
            const float f = need ? ex2(m_ref - m_new) : 1.f;
            if (need) m_ref = m_new;
            // P is formed as 2^15 * 2^(s - m): the fp16 operand of the PV product then
            // holds probabilities down to 2^-29 as normal numbers (the near-uniform rows
            // of a 1M-token head sit near 1e-6, fp16's subnormal range), and the
            // 2^15 cancels in O = acc / l because l sums the same scaled values.
            // The exponentials go to registers first: only the stores into this
            // group's P buffer (and the rescale of O_g) wait for the previous product.
            const float neg = kPScaleLog2 - m_ref;
            uint32_t pk1[32], pk0[32];
            float lsum = exp_p64(sr, v1, scale_log2, neg, pk1);
            if (v0) {                              // key half 0 again from TMEM
                PRISM_TMEM_LD32(tmem + lane_off + scol, (sr + 0));
                PRISM_TMEM_LD32(tmem + lane_off + scol + 32, (sr + 32));
                tmem_wait_ld();
            }
            // S has been read: the next S of this group may overwrite it
            tc_fence_before();
            mbar_arrive(&sm.s_free[g]);
            lsum += exp_p64(sr, v0, scale_log2, neg, pk0);
            // O_g and this group's P buffer were last used by the product of step j - 2
            if (cnt > 0 && !__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[g], ((j - 2) >> 1) & 1, a.err, 2))) {
                ok = false;
                break;
            }
            store_p64(pk1, p_s + SLAB, r);
            store_p64(pk0, p_s, r);
            const bool rescale = __any_sync(0xffffffffu, need);
            if (rescale) {
                tc_fence_after();
                #pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    PRISM_TMEM_LD32(tmem + lane_off + ocol + 32 * c, o);
                    tmem_wait_ld();
                    #pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float y0, y1;
                        fmul2(y0, y1, __uint_as_float(o[e]), __uint_as_float(o[e + 1]), f, f);
                        o[e] = __float_as_uint(y0);
                        o[e + 1] = __float_as_uint(y1);
                    }
                    PRISM_TMEM_ST32(tmem + lane_off + ocol + 32 * c, o);
                }
            }
            l = fmaf(l, f, lsum);
            fence_proxy_async_smem();
            if (rescale) tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[g]);
        }
        // epilogue: merge the groups' partial outputs.  Each group waits for its own
        // last product first (the PV issuer completes products in step order, so the
        // other group's barrier is then at most one phase behind), then the other's.
        const bool has0 = n > 0, has1 = n > 1;
        bool fin = ok;
        for (int k = 0; k < 2 && fin; ++k) {
            const int gg = k == 0 ? g : (g ^ 1);
            if (n <= gg) continue;
            const int jl = gg + 2 * ((n - 1 - gg) / 2);
            fin = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done[gg], (jl >> 1) & 1, a.err, 4));
        }
        // the P buffers are idle once every product has completed: exchange there
        float* xm = reinterpret_cast<float*>(&sm.p[0][0][0]);    // [group][row] max
        float* xl = xm + 256;                                     // [group][row] sum
        if (fin) {
            xm[g * 128 + r] = m_ref;
            xl[g * 128 + r] = l;
        }
        named_bar(1 + (warp & 3), 64);
        const int row_perm = t * 128 + r;
        const size_t prow = (size_t)h * a.N + (size_t)row_perm;   // block order (running max, sum)
        const size_t grow = (size_t)(h - a.h0) * a.N + (size_t)row_perm;   // the group's running O
        if (fin) {
            // this pass: (O_0 2^(m_0 - m_c) + O_1 2^(m_1 - m_c), l_c) relative to 2^m_c
            const float m0 = has0 ? xm[r] : -INFINITY, m1 = has1 ? xm[128 + r] : -INFINITY;
            const float l0 = has0 ? xl[r] : 0.f, l1 = has1 ? xl[128 + r] : 0.f;
            const float mc = fmaxf(m0, m1);
            const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - mc);
            const float f1 = m1 == -INFINITY ? 0.f : ex2(m1 - mc);
            const float lc = l0 * f0 + l1 * f1;
            // merged with the state of the previous passes over the other key tiles
            const float ms = a.first ? -INFINITY : a.st_m[prow];
            const float ls = a.first ? 0.f : a.st_l[prow];
            const float m = fmaxf(mc, ms);
            const float fc = mc == -INFINITY ? 0.f : ex2(mc - m);
            const float fs = ms == -INFINITY ? 0.f : ex2(ms - m);
            const float lt = lc * fc + ls * fs;
            const float inv = a.last ? (lt > 0.f ? o_unscale / lt : 0.f) : 1.f;
            const float w0 = f0 * fc * inv, w1 = f1 * fc * inv, ws = fs * inv;
            const bool use_s = !a.first && ms != -INFINITY;
            int srow = a.last ? a.src[prow] : 0;
            if (prism_bad_index(a.err, srow >= 0 && srow < a.N)) srow = 0;         // checking build
            const size_t orow = a.last ? (size_t)h * a.N + (size_t)srow : 0;
            tc_fence_after();
            constexpr int OC = HD / 2;             // output columns written by each group
            #pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
                const int c0 = OC * g + 32 * c;
                uint32_t o0[32], o1[32];
                if (has0) PRISM_TMEM_LD32(tmem + lane_off + TO + c0, o0);
                if (has1) PRISM_TMEM_LD32(tmem + lane_off + TO + HD + c0, o1);
                tmem_wait_ld();
                float x[32];
                #pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float v = 0.f;
                    if (has0) v = __uint_as_float(o0[e]) * w0;
                    if (has1) v = fmaf(__uint_as_float(o1[e]), w1, v);
                    x[e] = v;
                }
                if (use_s) {
                    const float4* sp = reinterpret_cast<const float4*>(a.st_o + grow * HD + c0);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 y = sp[e];
                        x[4 * e] = fmaf(y.x, ws, x[4 * e]);
                        x[4 * e + 1] = fmaf(y.y, ws, x[4 * e + 1]);
                        x[4 * e + 2] = fmaf(y.z, ws, x[4 * e + 2]);
                        x[4 * e + 3] = fmaf(y.w, ws, x[4 * e + 3]);
                    }
                }
                if (!a.last) {
                    float4* sp = reinterpret_cast<float4*>(a.st_o + grow * HD + c0);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) sp[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                } else if (a.out_f32) {
                    float4* op = reinterpret_cast<float4*>(a.O.row<float>(h, srow, HD) + c0);
                    #pragma unroll
                    for (int e = 0; e < 8; ++e) op[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                } else {
                    uint4* op = reinterpret_cast<uint4*>(a.O.row<__nv_bfloat16>(h, srow, HD) + c0);
                    #pragma unroll
                    for (int e = 0; e < 4; ++e)
                        op[e] = make_uint4(pack_bf16(x[8 * e], x[8 * e + 1]), pack_bf16(x[8 * e + 2], x[8 * e + 3]),
                                           pack_bf16(x[8 * e + 4], x[8 * e + 5]), pack_bf16(x[8 * e + 6], x[8 * e + 7]));
                }
            }
            if (g == 0) {
                if (a.last) {
                    a.lse[orow] = lt > 0.f ? (m - kPScaleLog2) * 0.69314718055994531f + logf(lt) : -INFINITY;
                } else {
                    a.st_m[prow] = m;
                    a.st_l[prow] = lt;
                }
            }
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
static int launch_fwd(prism_plan_s* P, const TokenRows& O, float* lse, cudaStream_t s) {
    const Geom& g = P->g;
    FwdArgs a;
    char* b = P->ws;
    a.qt_ptr = (const int*)(b + P->L.qt_ptr);
    a.lbase = (const int*)P->lists;
    a.qt_off = (const int64_t*)(b + P->L.loff) + LIST_FWD * (size_t)g.heads;
    a.src = (const int*)(b + P->L.src);
    a.O = O;
    a.lse = lse;
    a.N = g.N;
    a.NT = g.NT;
    a.out_f32 = P->p.out_dtype == PRISM_F32;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
    a.qkv_max = (const uint32_t*)(b + P->L.qkv_max);
    a.err = (int*)(b + P->L.err);
    // The running state between passes lives in buffers the backward fills only
    // later: the fp32 dQ accumulator (O) and the per-row terms (max, sum).
    a.st_o = (float*)(b + P->L.dq_acc);
    a.st_m = (float*)(b + P->L.lse_p);
    a.st_l = (float*)(b + P->L.di_p);
    const int smem = (int)sizeof(FwdSmem<HD>) + 1024;
    if (cudaFuncSetAttribute(k_attn_fwd<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PRISM_ERR_CUDA;
    const int passes = (g.NT + kFwdKeyChunk - 1) / kFwdKeyChunk;
    // one pass: every head in one launch (no running state); several passes: the
    // running O lives in a head group's scratch, so the groups run one after another
    const int gh = passes == 1 ? g.heads : g.GH;
    {
        PrismProf prof(P, PRISM_STAGE_FWD, s);
        for (int h0 = 0; h0 < g.heads; h0 += gh) {
            const int nh = std::min(gh, g.heads - h0);
            a.h0 = h0;
            for (int c = 0; c < passes; ++c) {
                a.key_lo = c * kFwdKeyChunk;
                a.key_hi = c + 1 == passes ? g.NT : (c + 1) * kFwdKeyChunk;
                a.first = c == 0;
                a.last = c + 1 == passes;
                k_attn_fwd<HD><<<dim3(g.NT, nh), FWD_THREADS, smem, s>>>(P->tm_q, P->tm_k, P->tm_v, a);
                P->launches += 1;
            }
        }
    }
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

}  // namespace prism

int prism_launch_selftest_wait(prism_plan_s* P, void* stream) {
    prism::k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((int*)(P->ws + P->L.err));
    P->launches += 1;
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

int prism_launch_attn_fwd(prism_plan_s* P, const prism::TokenRows& O, float* lse, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return P->g.D == 128 ? prism::launch_fwd<128>(P, O, lse, s) : prism::launch_fwd<64>(P, O, lse, s);
}
