// prism_attn_bwd.cu -- gradients of the block-sparse attention on sm_100a.
//
// "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio Generation
// Model Training" detaches the plan (statistics, shapes, selection): gradients
// flow only through the attention over the selected key blocks (page
// xyznot.com/th, section on training).  The pages give no backward kernel; the
// kernels below compute the exact gradients of the forward with the selection
// fixed, FlashAttention-style, restricted to the selected (query, key) pairs:
//   D_i = rowsum(dO o O);  P = exp(S/sqrt(d) - LSE);  dV = P^T dO;
//   dP = dO V^T;  dS = P o (dP - D);  dK = dS^T Q / sqrt(d);  dQ = dS K / sqrt(d).
//
// Kernels:
//   k_bwd_absmax / k_bwd_pre   per row: D_i, dO in fp16 block order (scaled
//               by an exact per-head power of two so that max |dO| lies in
//               [0.5, 1): gradients of any magnitude keep fp16's precision and
//               dS cannot overflow), LSE in block order.
//   k_bwd_dkdv  one CTA per (128-key tile, chunk of 512 query tiles); iterates
//               the 64-row query halves of that range of the key tile's
//               transposed list; S^T = K Q^T and dP^T = V dO^T into TMEM
//               (double-buffered), softmax warps form P^T (into TMEM, over
//               dP^T) and dS^T (into TMEM, over S^T), dV += P^T dO and
//               dK += dS^T Q accumulate in TMEM with their A operands read
//               from TMEM, and are TMA reduce-added into fp32 accumulators at
//               the end of the chunk.  For head_dim 128 the same CTA also
//               forms dQ^T = K^T dS^T per unit (dS^T also in shared memory, as
//               its B operand) and adds it into an fp32 accumulator with
//               coalesced L2 reductions.  The grid runs chunk by chunk, so the
//               dQ rows being accumulated stay in L2.
//   k_acc_finalize  scales the accumulators and scatters them to raster order.
//   k_bwd_dq    (head_dim 64) one CTA per 128-row query tile; iterates the
//               64-key halves of the forward list; S = Q K^T, dP = dO V^T,
//               dS -> shared memory, dQ += dS K in TMEM.
// Warp roles as in the forward: 0-3 softmax/epilogue (thread = TMEM lane),
// 4 TMA producer + TMEM allocator, 5 MMA issuer.  All waits are bounded and
// every TMEM access is warp-uniform.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "prism_dev.cuh"
#include "prism_internal.h"

namespace prism {

constexpr int BWD_STAGES = 2;
constexpr int DKDV_STAGES = 3;   // Q/dO prefetch depth of the dK/dV kernel
constexpr int kChunkTiles = 512; // query tiles per chunk of the dK/dV grid
constexpr int SLAB128 = 128 * 128;   // bytes: 128 rows x 64 fp16
constexpr int SLAB64 = 64 * 128;     // bytes:  64 rows x 64 fp16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kPScale = 32768.f;          // 2^15: scale of the P operand of dV += P^T dO
constexpr float kPScaleLog2 = 15.f;
constexpr float kPScaleInv = 1.f / 32768.f;
constexpr int kDsShift = 7;                 // dS' = dS 2^(kDsShift - E - ev): see k_bwd_pre

// --------------------------------------------------------------- preprocess
// max |dO| per head (fp32 bits, see fold_abs): one pass over 16-byte chunks of
// each shard's rows of the head (dO is 16-byte aligned and a shard holds
// S x head_dim values of a head).
template <typename OT>
__global__ void __launch_bounds__(256) k_bwd_absmax(const TokenRows dO, uint32_t* dmax, int HD) {
    const int h = blockIdx.y;
    const int64_t n16 = dO.S * HD * (int64_t)sizeof(OT) / 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m = 0u;
    for (int sh = 0; sh < dO.n; ++sh) {
        const uint4* x = reinterpret_cast<const uint4*>(static_cast<const OT*>(dO.p[sh]) +
                                                        (int64_t)(dO.head0 + h) * dO.S * HD);
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + stride < n16; i += 2 * stride) {         // two chunks in flight
            const uint4 a = __ldg(x + i), b = __ldg(x + i + stride);
            m = fold_abs<OT>(fold_abs<OT>(m, a), b);
        }
        if (i < n16) m = fold_abs<OT>(m, __ldg(x + i));
    }
    uint32_t b = abs_bits<OT>(m);
    for (int o = 16; o > 0; o >>= 1) b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    if ((threadIdx.x & 31) == 0) atomicMax(dmax + h, b);
}

// Exponent E with max |dO| in [2^(E-1), 2^E); dO is multiplied by 2^-E.
__device__ __forceinline__ int dscale_exp(uint32_t bits, int* err) {
    const float mx = __uint_as_float(bits);
    if (!(mx <= 3.0e38f)) { atomicCAS(err, 0, PRISM_ERR_DEVICE_CHECK); return 0; }
    if (mx == 0.f) return 0;
    int e;
    frexpf(mx, &e);
    return e;
}

template <typename OT>
__global__ void __launch_bounds__(256) k_bwd_pre(const TokenRows dO, const TokenRows O,
                                                 const float* __restrict__ lse,
                                                 const int* __restrict__ src, const uint32_t* dmax,
                                                 __half* __restrict__ dOp, float* __restrict__ lse_p,
                                                 float* __restrict__ di_p, int64_t N, int HD, int h0,
                                                 const uint32_t* __restrict__ qkv_max, int* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t p = (int64_t)blockIdx.x * 8 + warp;
    const int h = h0 + blockIdx.y;                   // dOp holds the head group [h0, h0 + gridDim.y)
    if (p >= N) return;
    const float sc = ldexpf(1.f, -dscale_exp(dmax[h], err));
    const int64_t n = src[(size_t)h * N + p];
    if (prism_bad_index(err, n >= 0 && n < N)) return;
    const OT* dr = dO.row<const OT>(h, n, HD);
    const OT* orow = O.row<const OT>(h, n, HD);
    __half* out = dOp + ((size_t)(h - h0) * N + p) * HD;
    float acc = 0.f;
    for (int c = lane; c < HD; c += 32) {
        const float g = (float)dr[c];
        acc = fmaf(g, (float)orow[c], acc);
        out[c] = __float2half_rn(g * sc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    // stored for the softmax of the backward kernels, which form P' = 2^15 P as
    // ex2(s * log2(e)/sqrt(d) + lse_p) and dS' = P' (dP_copy 2^-23 + di_p) with one
    // fused multiply-add each: lse_p = 15 - LSE log2(e), di_p = -D 2^-15 2^(sv - 8)
    // with D in the dO scale 2^-E and 2^sv the V copy's scale (2^ev = 2^(15 - sv)
    // is V's magnitude), so that dS' = dS 2^(7 - E - ev).  |dP - D| is at most
    // 2 D max|dO| max|V| < 2 D 2^E 2^ev, so |dS'| < 2 D 2^7 P <= 32768 for any
    // input magnitude (head_dim 128), and a small dS sits 2^7 above its
    // normalised value, clear of fp16's subnormal range
    if (lane == 0) {
        di_p[(size_t)h * N + p] = -acc * sc * ldexpf(kPScaleInv, qkv_shift(qkv_max[h * 3 + 2]) - 15 + kDsShift);
        lse_p[(size_t)h * N + p] = kPScaleLog2 - lse[(size_t)h * N + n] * kLog2e;
    }
}

// Iterator over the 64-token halves of a tile list.  Each entry is
// (other tile << 4) | mask, mask bit (qhalf * 2 + khalf).  `own_is_key`
// selects which side of the bit pair belongs to the CTA's own tile: the
// iterated half is the other side, and the returned 2-bit mask says which of
// the own tile's halves take part.
struct HalfIter {
    const int* ents;
    int n, e, half;
    int own_is_key;
    __device__ bool next(int& row64, int& mask2) {
        while (e < n) {
            const int ent = ents[e];
            const int other = ent >> 4, mk = ent & 15;
            const int hf = half;
            if (++half == 2) { half = 0; ++e; }
            int m2;
            if (own_is_key)   // iterated = query half hf; own halves = key halves
                m2 = (mk >> (hf * 2)) & 3;
            else              // iterated = key half hf; own halves = query halves
                m2 = ((mk >> hf) & 1) | (((mk >> (2 + hf)) & 1) << 1);
            if (m2) { row64 = other * 2 + hf; mask2 = m2; return true; }
        }
        return false;
    }
};

__device__ __forceinline__ int count_units(const int* ents, int n, int own_is_key) {
    HalfIter it{ents, n, 0, 0, own_is_key};
    int r, m, c = 0;
    while (it.next(r, m)) ++c;
    return c;
}

struct BwdArgs {
    const int* ptr;        // [heads][NT + 1]
    const int* lbase;      // index lists; head h's tile list starts at lbase + ent_off[h]
    const int64_t* ent_off;
    int h0;                // first head of the launch's group: the dO copy and the
                           // accumulators hold heads h0, h0 + 1, ... (rows (h - h0) N + ...)
    const int* src;        // [heads][N]
    const float* lse_p;    // [heads][N] 15 - LSE log2(e), block order
    const float* di_p;     // [heads][N] -D 2^-15 (D scaled like dO)
    const uint32_t* dmax;  // [heads] max |dO| bits: outputs are divided by the dO scale
    TokenRows out0;        // dQ (dq): rows of the output, a plain tensor or token shards
    float* dq_acc;         // (dkdv, head_dim 128) fp32 dQ accumulator, block order, head group
    int64_t N;
    int NT;
    int out_f32;
    float scale_log2;      // log2(e) / sqrt(d)
    const uint32_t* qkv_max;  // [heads][3]: the copies' per-head scales (qkv_shift)
    float inv_sqrt_d;
    int CQ;                // query tiles per chunk of the dK/dV grid
    int* err;
};

// First index in the ascending list e[0, n) whose tile (entry >> 4) is >= key.
__device__ __forceinline__ int tiles_lower_bound(const int* e, int n, int key) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((e[mid] >> 4) < key) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

__device__ __forceinline__ void store_row(void* rowp, int c0, const uint32_t* v, float mul, int out_f32) {
    if (out_f32) {
        float4* op = reinterpret_cast<float4*>(static_cast<float*>(rowp) + c0);
        #pragma unroll
        for (int e = 0; e < 8; ++e)
            op[e] = make_float4(__uint_as_float(v[4 * e]) * mul, __uint_as_float(v[4 * e + 1]) * mul,
                                __uint_as_float(v[4 * e + 2]) * mul, __uint_as_float(v[4 * e + 3]) * mul);
    } else {
        uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(rowp) + c0);
        #pragma unroll
        for (int e = 0; e < 4; ++e)
            op[e] = make_uint4(pack_bf16(__uint_as_float(v[8 * e]) * mul, __uint_as_float(v[8 * e + 1]) * mul),
                               pack_bf16(__uint_as_float(v[8 * e + 2]) * mul, __uint_as_float(v[8 * e + 3]) * mul),
                               pack_bf16(__uint_as_float(v[8 * e + 4]) * mul, __uint_as_float(v[8 * e + 5]) * mul),
                               pack_bf16(__uint_as_float(v[8 * e + 6]) * mul, __uint_as_float(v[8 * e + 7]) * mul));
    }
}

__device__ __forceinline__ void zero_row(void* rowp, int HD, int out_f32) {
    for (int c = 0; c < HD; ++c) {
        if (out_f32) static_cast<float*>(rowp)[c] = 0.f;
        else static_cast<__nv_bfloat16*>(rowp)[c] = __float2bfloat16(0.f);
    }
}

// ------------------------------------------------------------------- dK, dV
// FUSE (head_dim 128): the same CTA also forms dQ^T = K^T dS^T for every
// 64-query unit into the TMEM columns of dP^T; a drain warpgroup (warps 10-13)
// adds it from registers into an fp32 dQ accumulator in block order with
// coalesced reductions in L2, so dQ costs one more MMA instead of a second
// kernel that recomputes S and dP.  Shared-memory bandwidth is what this
// kernel runs at (the tensor cores read every operand from it), so dS^T also
// goes to TMEM, where it is the A operand of dK, and dQ^T is not staged.
template <int HD, bool FUSE>
struct DkdvSmem {
    static constexpr int NSL = HD / 64;
    alignas(1024) uint8_t k[NSL][SLAB128];
    alignas(1024) uint8_t v[NSL][SLAB128];
    alignas(1024) uint8_t q[DKDV_STAGES][NSL][SLAB64];
    alignas(1024) uint8_t dO[DKDV_STAGES][NSL][SLAB64];
    alignas(1024) uint8_t ds[2][SLAB128];     // dS^T [128 keys][64 queries]: the B operand of dQ^T
    alignas(16) float lse[DKDV_STAGES][64];
    alignas(16) float di[DKDV_STAGES][64];
    uint64_t bar_kv;
    uint64_t st_full[DKDV_STAGES], st_empty[DKDV_STAGES];
    uint64_t s_full[2], p_full[2], pd_done[2];
    uint64_t acc_done;                        // every MMA of the CTA has completed
    uint64_t dq_full[2], dq_free[2];
    uint32_t tmem_base;
    int e0, ne, U;                            // this chunk's entries and 64-query units
};

// the dK / dV epilogue stages 8 warps x 32 rows x HD fp32 values in q, dO and ds
template <int HD, bool FUSE>
constexpr bool epilogue_fits() {
    using S = DkdvSmem<HD, FUSE>;
    return offsetof(S, lse) - offsetof(S, q) >= 8 * 32 * HD * sizeof(float);
}

template <int HD, bool FUSE>
__global__ void __launch_bounds__(FUSE ? 480 : 352, 1)
k_bwd_dkdv(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
           const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
           const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv, BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    DkdvSmem<HD, FUSE>& sm = *reinterpret_cast<DkdvSmem<HD, FUSE>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSL = HD / 64;
    // one CTA per (key tile t, chunk c of CQ query tiles): the grid runs chunk
    // after chunk, so the dQ accumulator rows and the Q / dO tiles that all CTAs
    // in flight touch are one chunk's (about 32 MB), resident in L2
    const int t = blockIdx.x, c = blockIdx.y, h = a.h0 + blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        const int p0 = a.ptr[(size_t)h * (a.NT + 1) + t];
        const int n0 = a.ptr[(size_t)h * (a.NT + 1) + t + 1] - p0;
        const int* all = a.lbase + a.ent_off[h] + p0;
        const int lo = tiles_lower_bound(all, n0, c * a.CQ);
        const int hi = tiles_lower_bound(all, n0, (c + 1) * a.CQ);
        sm.e0 = p0 + lo;
        sm.ne = hi - lo;
        sm.U = count_units(all + lo, hi - lo, 1);
    }
    __syncthreads();
    const int e0 = sm.e0, ne = sm.ne, U = sm.U;
    if (U == 0) return;                            // nothing selected in this chunk
    const int* ents = a.lbase + a.ent_off[h] + e0;
    // TMEM columns: buffer b = [128b, 128b + 128): S^T at 128b, dP^T at 128b + 64.
    // The softmax writes dS^T (fp16 pairs) over the first half of S^T and P^T
    // over the first half of dP^T; dQ^T of the unit then overwrites all 64 dP^T
    // columns after dV has read P^T (the MMAs of one issuer run in order), so
    // the next S^T into the buffer waits for dK (which reads dS^T there), not
    // for the dQ drain -- only the next dP^T does.  dV at 256, dK at 256 + HD.
    constexpr uint32_t TDV = 256, TDK = 256 + HD;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_kv, 1);
        mbar_init(&sm.acc_done, 1);
        for (int s = 0; s < DKDV_STAGES; ++s) { mbar_init(&sm.st_full[s], 1); mbar_init(&sm.st_empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], 256);
            mbar_init(&sm.pd_done[b], 1);
            mbar_init(&sm.dq_full[b], 1);
            mbar_init(&sm.dq_free[b], 128);
        }
        mbar_fence_init();
    }
    // warps 0-7: two softmax warpgroups (same 128 key rows, one 32-query half of
    // the unit each); warp 8: TMA producer + TMEM allocator; warp 9: issuer of
    // S^T and dP^T; warps 10-13 (FUSE): dQ drain; warp 14 (10 without FUSE):
    // issuer of dV, dQ^T and dK.  Two issuers on different SM sub-partitions:
    // an issuing thread that waits on a barrier stalls until its queued MMAs
    // have been handed to the tensor core, so with one issuer every wait left
    // the tensor pipe idle; each issuer now waits while the other one feeds it.
    constexpr int W_PROD = 8, W_MMA = 9, W_MMB = FUSE ? 14 : 10;
    if (warp == W_PROD) { __syncwarp(); tmem_alloc(&sm.tmem_base, 512); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int64_t hrow = (int64_t)h * a.N;               // Q, K, V copies and per-row terms
    const int64_t grow = (int64_t)(h - a.h0) * a.N;      // dO copy and accumulators (head group)
    // the copies carry Q 2^sq, K 2^sk, V 2^sv: the logit scale and dP undo them
    // (dK and dQ are unscaled when the accumulators are finalised)
    const float scale_log2 = ldexpf(a.scale_log2, -(qkv_shift(a.qkv_max[h * 3]) + qkv_shift(a.qkv_max[h * 3 + 1])));
    constexpr float pinv = 1.f / (1 << 23);               // 2^-23: dS' = dS 2^(7 - E - ev) (see k_bwd_pre)

    if (warp == W_PROD) {
        if (lane == 0 && U > 0) {
            const int krow = (int)(hrow + (int64_t)t * 128);
            mbar_expect_tx(&sm.bar_kv, 2 * NSL * SLAB128);
            for (int c = 0; c < NSL; ++c) {
                tma_load_2d(sm.k[c], &tm_k, &sm.bar_kv, 64 * c, krow);
                tma_load_2d(sm.v[c], &tm_v, &sm.bar_kv, 64 * c, krow);
            }
            HalfIter it{ents, ne, 0, 0, 1};
            int r64, m2;
            for (int u = 0; it.next(r64, m2); ++u) {
                const int s = u % DKDV_STAGES;
                if (prism_bad_index(a.err, r64 >= 0 && r64 < 2 * a.NT)) r64 = 0;   // checking build
                if (u >= DKDV_STAGES &&
                    !mbar_wait(&sm.st_empty[s], ((u / DKDV_STAGES) - 1) & 1, a.err, 1401)) break;
                const int64_t qrow = hrow + (int64_t)r64 * 64;
                const int64_t grow_q = grow + (int64_t)r64 * 64;
                mbar_expect_tx(&sm.st_full[s], 2 * NSL * SLAB64 + 2 * 256);
                for (int c = 0; c < NSL; ++c) {
                    tma_load_2d(sm.q[s][c], &tm_q64, &sm.st_full[s], 64 * c, (int)qrow);
                    tma_load_2d(sm.dO[s][c], &tm_do64, &sm.st_full[s], 64 * c, (int)grow_q);
                }
                bulk_load(sm.lse[s], a.lse_p + qrow, 256, &sm.st_full[s]);
                bulk_load(sm.di[s], a.di_p + qrow, 256, &sm.st_full[s]);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------ S^T and dP^T issuer
        if (lane == 0 && U > 0) {
            constexpr uint32_t id_s = idesc_f16(128, 64, 0, 0);
            // descriptor low words; every K step below adds an immediate
            const uint32_t kA = desc_lo(smem_u32(sm.k[0]), 16), vA = desc_lo(smem_u32(sm.v[0]), 16);
            bool ok = mbar_wait(&sm.bar_kv, 0, a.err, 1501);
            for (int u = 0; ok && u < U; ++u) {
                const int s = u % DKDV_STAGES, b = u & 1;
                if (!mbar_wait(&sm.st_full[s], (u / DKDV_STAGES) & 1, a.err, 1502)) break;
                // S^T(u) overwrites dS^T(u - 2): wait until dK(u - 2) has read it
                // (pd_done follows p_full: the softmax has also read S^T(u - 2))
                if (u >= 2 && !mbar_wait(&sm.pd_done[b], ((u - 2) >> 1) & 1, a.err, 1503)) break;
                tc_fence_after();
                const uint32_t qB = desc_lo(smem_u32(sm.q[s][0]), 16), doB = desc_lo(smem_u32(sm.dO[s][0]), 16);
                #pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_f16(tmem + 128 * b, desc_from_lo(kA + kmajor_step(kk, SLAB128)),
                             desc_from_lo(qB + kmajor_step(kk, SLAB64)), id_s, kk > 0);
                // dP^T overwrites P^T(u - 2) and (FUSE) dQ^T(u - 2): wait until dV(u - 2)
                // has read P^T (pd_done) and the drain has read dQ^T (dq_free)
                if (u >= 2) {
                    if (FUSE ? !mbar_wait(&sm.dq_free[b], ((u - 2) >> 1) & 1, a.err, 1505)
                             : !mbar_wait(&sm.pd_done[b], ((u - 2) >> 1) & 1, a.err, 1506))
                        break;
                }
                tc_fence_after();
                #pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    umma_f16(tmem + 128 * b + 64, desc_from_lo(vA + kmajor_step(kk, SLAB128)),
                             desc_from_lo(doB + kmajor_step(kk, SLAB64)), id_s, kk > 0);
                umma_commit(&sm.s_full[b]);
            }
        }
    } else if (warp == W_MMB) {
        // ------------------------------------------------ dV, dK and dQ^T issuer
        if (lane == 0 && U > 0) {
            constexpr uint32_t id_acc = idesc_f16(128, HD, 0, 1);
            constexpr uint32_t id_dq = idesc_f16(128, 64, 1, 1);
            const uint32_t kT = desc_lo(smem_u32(sm.k[0]), SLAB128);       // K^T (MN-major) for dQ^T
            int u = 0;
            for (; u < U; ++u) {
                const int b = u & 1, s = u % DKDV_STAGES;
                // P^T and dS^T of unit u are in TMEM (and dS^T in shared memory)
                if (!mbar_wait(&sm.p_full[b], (u >> 1) & 1, a.err, 1504)) break;
                tc_fence_after();
                const uint32_t qT = desc_lo(smem_u32(sm.q[s][0]), SLAB64);
                const uint32_t doT = desc_lo(smem_u32(sm.dO[s][0]), SLAB64);
                // dV += P^T dO with P^T (fp16) read from TMEM over the dP^T columns,
                // dK += dS^T Q with dS^T (fp16) read from TMEM over the S^T columns
                #pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ts(tmem + TDV, tmem + 128 * b + 64 + 8 * kk, desc_from_lo(doT + mnmajor_step(kk)),
                                id_acc, (u > 0 || kk > 0) ? 1u : 0u);
                #pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ts(tmem + TDK, tmem + 128 * b + 8 * kk, desc_from_lo(qT + mnmajor_step(kk)),
                                id_acc, (u > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sm.pd_done[b]);
                umma_commit(&sm.st_empty[s]);     // Q / dO of stage s are read
                if (FUSE) {
                    // dQ^T [HD x 64 queries] = K^T [HD x 128 keys] . dS^T [128 keys x 64 queries],
                    // over the dP^T columns (after dV above has read P^T there)
                    const uint32_t dsT = desc_lo(smem_u32(sm.ds[b]), SLAB128);     // dS^T as MN-major B
                    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + 128 * b + 64, desc_from_lo(kT + mnmajor_step(kk)),
                                 desc_from_lo(dsT + mnmajor_step(kk)), id_dq, kk > 0);
                    umma_commit(&sm.dq_full[b]);
                }
            }
            if (u == U) umma_commit(&sm.acc_done);   // dV and dK are final
        }
    } else if (warp < 8) {
        const int wg = warp >> 2;                   // which 32 queries of the unit
        const int r = (warp & 3) * 32 + lane;       // key row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int kh = r >> 6;                      // warp-uniform
        const int c0 = 32 * wg;
        bool ok = true;
        int nbar = 0;                               // quarter barriers taken in the loop
        HalfIter it{ents, ne, 0, 0, 1};
        int r64, m2;
        for (int u = 0; it.next(r64, m2); ++u) {
            const int b = u & 1, s = u % DKDV_STAGES;
            const bool valid = (m2 >> kh) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (u >> 1) & 1, a.err, 1001))) { ok = false; break; }
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.st_full[s], (u / DKDV_STAGES) & 1, a.err, 1002))) { ok = false; break; }
            // dQ^T(u - 2) has read dS^T(u - 2) in shared memory before dS^T(u) overwrites
            // it (the TMEM copies are safe: S^T(u) was written there after dK(u - 2))
            if (FUSE && u >= 2 &&
                !__all_sync(0xffffffffu, mbar_wait(&sm.dq_full[b], ((u - 2) >> 1) & 1, a.err, 1003))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sv[32], dp[32];
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + c0, sv);
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 64 + c0, dp);
            tmem_wait_ld();
            // both warpgroups of this lane quarter have read dP^T before P^T overwrites it
            named_bar(2 + (warp & 3), 64);
            ++nbar;
            const float4* lq4 = reinterpret_cast<const float4*>(sm.lse[s] + c0);
            const float4* dq4 = reinterpret_cast<const float4*>(sm.di[s] + c0);
            const uint32_t ds_s = smem_u32(sm.ds[b]);
            uint32_t pt[16], dst[16];
            #pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                // lse_p = 15 - LSE log2(e) and di_p = -D 2^-15 of the chunk's 8 queries
                const float4 x0 = lq4[2 * ch], x1 = lq4[2 * ch + 1];
                const float4 y0 = dq4[2 * ch], y1 = dq4[2 * ch + 1];
                const float lq[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                const float dq[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                uint32_t* wd = dst + 4 * ch;
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = ch * 8 + 2 * e;
                    float p0 = 0.f, p1 = 0.f, d0 = 0.f, d1 = 0.f;
                    if (valid) {
                        // P' = 2^15 P: the dV operand, normal in fp16 down to P = 2^-29
                        // (dV is unscaled at the end); dS = P (dP - D) = P' (dP 2^-15 - D 2^-15)
                        float x0_, x1_;
                        ffma2(x0_, x1_, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), scale_log2,
                              scale_log2, lq[2 * e], lq[2 * e + 1]);
                        p0 = ex2(x0_);
                        p1 = ex2(x1_);
                        float t0, t1;
                        ffma2(t0, t1, __uint_as_float(dp[c]), __uint_as_float(dp[c + 1]), pinv, pinv,
                              dq[2 * e], dq[2 * e + 1]);
                        fmul2(d0, d1, p0, p1, t0, t1);
                    }
                    pt[ch * 4 + e] = pack_f16(p0, p1);
                    wd[e] = pack_f16(d0, d1);
                }
                if (FUSE) st_shared_v4(ds_s + swz128(r, 4 * wg + ch), wd[0], wd[1], wd[2], wd[3]);
            }
            PRISM_TMEM_ST16(tmem + lane_off + 128 * b + 64 + 16 * wg, pt);
            PRISM_TMEM_ST16(tmem + lane_off + 128 * b + 16 * wg, dst);
            if (FUSE) fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
        }
        // a warp that left the loop on a failed wait still takes the barriers
        // the other warpgroup will take, so that one is never left at a barrier
        for (; nbar < U; ++nbar) named_bar(2 + (warp & 3), 64);
        // epilogue: this chunk's share of dV (warpgroup 0) and dK (warpgroup 1)
        // is TMA reduce-added into the fp32 accumulators (block order, unscaled).
        // Each warp stages its 32 rows in the Q / dO / dS^T buffers, idle once
        // every MMA of the CTA has completed (8 x 32 x HD floats fit there).
        bool fin = false;
        if (ok)
            fin = __all_sync(0xffffffffu, mbar_wait(&sm.acc_done, 0, a.err, 1004));
        if (fin) {
            tc_fence_after();
            float* stage = reinterpret_cast<float*>(&sm.q[0][0][0]) + (size_t)warp * 32 * HD;
            const uint32_t col = wg ? TDK : TDV;
            #pragma unroll
            for (int c4 = 0; c4 < HD / 32; ++c4) {
                uint32_t o[32];
                PRISM_TMEM_LD32(tmem + lane_off + col + 32 * c4, o);
                tmem_wait_ld();
                float4* dst = reinterpret_cast<float4*>(stage + (size_t)lane * HD + 32 * c4);
                #pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                         __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_reduce_add_2d(wg ? &tm_dk : &tm_dv, stage, 0, (int)(grow + (int64_t)t * 128 + 32 * (warp & 3)));
                bulk_commit();
                bulk_wait0();
            }
            __syncwarp();
        }
    } else if (FUSE && warp >= 10) {
        // ---------------------------------------------- dQ drain (warps 10-13)
        // thread = head-dim row d of dQ^T (TMEM lane); each of the 64 columns is
        // one query: a warp's reduction covers 32 adjacent floats of that query's
        // accumulator row (one 128-byte line)
        const int d = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        HalfIter it{ents, ne, 0, 0, 1};
        int r64, m2;
        for (int u = 0; it.next(r64, m2); ++u) {
            const int b = u & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.dq_full[b], (u >> 1) & 1, a.err, 3001))) break;
            tc_fence_after();
            uint32_t v[64];
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 64, v);
            PRISM_TMEM_LD32(tmem + lane_off + 128 * b + 96, (v + 32));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.dq_free[b]);
            if (prism_bad_index(a.err, r64 >= 0 && r64 < 2 * a.NT)) continue;   // checking build
            float* dst = a.dq_acc + (grow + (int64_t)r64 * 64) * HD + d;
            #pragma unroll
            for (int qq = 0; qq < 64; ++qq) red_add_f32(dst + (size_t)qq * HD, __uint_as_float(v[qq]));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == W_PROD) { __syncwarp(); tmem_dealloc(tmem, 512); }
}

// fp32 accumulators (block order, unscaled) -> outputs (raster order): one
// warp per row p, out[src[p]] = acc[p] * scale * 2^-e (the per-head dO scale).
// Two accumulators (dK, dV) or one (dQ, acc1 == nullptr) per launch.
template <typename OT>
__global__ void __launch_bounds__(256) k_acc_finalize(const float* __restrict__ acc0, float scale0, const TokenRows out0,
                                                      const float* __restrict__ acc1, float scale1,
                                                      const TokenRows out1, const int* __restrict__ src,
                                                      const uint32_t* dmax, int64_t N, int HD, int h0,
                                                      const uint32_t* __restrict__ qkv_max, int which0, int* err) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t p = (int64_t)blockIdx.x * 8 + warp;
    const int h = h0 + blockIdx.y;                   // accumulators hold the head group from h0
    if (p >= N) return;
    const float unscale = ldexpf(1.f, dscale_exp(dmax[h], err));
    // acc0 came from dS' (dS 2^(7 - E - ev), see k_bwd_pre) and the Q copy (dK) or
    // the K copy (dQ): undo both (the 2^-E with `unscale`)
    if (which0 >= 0)
        scale0 = ldexpf(scale0, 15 - qkv_shift(qkv_max[h * 3 + 2]) - kDsShift - qkv_shift(qkv_max[h * 3 + which0]));
    const int64_t n = src[(size_t)h * N + p];
    if (prism_bad_index(err, n >= 0 && n < N)) return;
    const size_t ir = ((size_t)(h - h0) * N + p) * HD;
    OT* o0 = out0.row<OT>(h, n, HD);
    for (int c = lane; c < HD; c += 32) o0[c] = (OT)(acc0[ir + c] * (scale0 * unscale));
    if (acc1) {
        OT* o1 = out1.row<OT>(h, n, HD);
        for (int c = lane; c < HD; c += 32) o1[c] = (OT)(acc1[ir + c] * (scale1 * unscale));
    }
}

// ------------------------------------------------------------------------ dQ
template <int HD>
struct DqSmem {
    static constexpr int NSL = HD / 64;
    alignas(1024) uint8_t q[NSL][SLAB128];
    alignas(1024) uint8_t dO[NSL][SLAB128];
    alignas(1024) uint8_t k[BWD_STAGES][NSL][SLAB64];
    alignas(1024) uint8_t v[BWD_STAGES][NSL][SLAB64];
    alignas(1024) uint8_t ds[2][SLAB128];     // dS [128 queries][64 keys]
    uint64_t bar_q;
    uint64_t st_full[BWD_STAGES], st_empty[BWD_STAGES];
    uint64_t s_full[2], s_free[2], ds_full[2], dq_done[2];
    uint32_t tmem_base;
};

template <int HD>
__global__ void __launch_bounds__(192, 1)
k_bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
         const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
         BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    DqSmem<HD>& sm = *reinterpret_cast<DqSmem<HD>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NSL = HD / 64;
    const int t = blockIdx.x, h = a.h0 + blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = a.ptr[(size_t)h * (a.NT + 1) + t];
    const int ne = a.ptr[(size_t)h * (a.NT + 1) + t + 1] - e0;
    const int* ents = a.lbase + a.ent_off[h] + e0;
    const int U = count_units(ents, ne, 0);
    constexpr uint32_t TS = 0, TDP = 128, TDQ = 256;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < BWD_STAGES; ++s) { mbar_init(&sm.st_full[s], 1); mbar_init(&sm.st_empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.s_free[b], 128);
            mbar_init(&sm.ds_full[b], 128);
            mbar_init(&sm.dq_done[b], 1);
        }
        mbar_fence_init();
    }
    if (warp == 4) { __syncwarp(); tmem_alloc(&sm.tmem_base, 512); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int64_t hrow = (int64_t)h * a.N;                  // Q, K, V copies, per-row terms
    const int64_t grow = (int64_t)(h - a.h0) * a.N;         // the head group's dO copy
    // the copies' scales: logits, dP and dQ (= dS K_copy 2^-sk) undo them
    const int sk = qkv_shift(a.qkv_max[h * 3 + 1]), ev = 15 - qkv_shift(a.qkv_max[h * 3 + 2]);
    const float scale_log2 = ldexpf(a.scale_log2, -(qkv_shift(a.qkv_max[h * 3]) + sk));
    constexpr float pinv = 1.f / (1 << 23);               // 2^-23: dS' = dS 2^(7 - E - ev) (see k_bwd_pre)

    if (warp == 4) {
        if (lane == 0 && U > 0) {
            const int qrow = (int)(hrow + (int64_t)t * 128);
            const int dorow = (int)(grow + (int64_t)t * 128);
            mbar_expect_tx(&sm.bar_q, 2 * NSL * SLAB128);
            for (int c = 0; c < NSL; ++c) {
                tma_load_2d(sm.q[c], &tm_q, &sm.bar_q, 64 * c, qrow);
                tma_load_2d(sm.dO[c], &tm_do, &sm.bar_q, 64 * c, dorow);
            }
            HalfIter it{ents, ne, 0, 0, 0};
            int r64, m2;
            for (int u = 0; it.next(r64, m2); ++u) {
                const int s = u % BWD_STAGES;
                if (u >= BWD_STAGES &&
                    !mbar_wait(&sm.st_empty[s], ((u / BWD_STAGES) - 1) & 1, a.err, 2401)) break;
                if (prism_bad_index(a.err, r64 >= 0 && r64 < 2 * a.NT)) r64 = 0;   // checking build
                const int krow = (int)(hrow + (int64_t)r64 * 64);
                mbar_expect_tx(&sm.st_full[s], 2 * NSL * SLAB64);
                for (int c = 0; c < NSL; ++c) {
                    tma_load_2d(sm.k[s][c], &tm_k64, &sm.st_full[s], 64 * c, krow);
                    tma_load_2d(sm.v[s][c], &tm_v64, &sm.st_full[s], 64 * c, krow);
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0 && U > 0) {
            constexpr uint32_t id_s = idesc_f16(128, 64, 0, 0);
            constexpr uint32_t id_acc = idesc_f16(128, HD, 0, 1);
            const uint32_t q_s = smem_u32(sm.q[0]), do_s = smem_u32(sm.dO[0]);
            bool ok = mbar_wait(&sm.bar_q, 0, a.err, 2501);
            for (int u = 0; ok && u <= U; ++u) {
                if (u < U) {
                    const int s = u % BWD_STAGES, b = u & 1;
                    if (!mbar_wait(&sm.st_full[s], (u / BWD_STAGES) & 1, a.err, 2502)) break;
                    if (u >= 2 && !mbar_wait(&sm.s_free[b], ((u - 2) >> 1) & 1, a.err, 2503)) break;
                    tc_fence_after();
                    const uint32_t k_s = smem_u32(sm.k[s][0]), v_s = smem_u32(sm.v[s][0]);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + TS + 64 * b, desc_kmajor(q_s, kk, SLAB128),
                                  desc_kmajor(k_s, kk, SLAB64), id_s, kk > 0);
                    #pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk)
                        umma_f16(tmem + TDP + 64 * b, desc_kmajor(do_s, kk, SLAB128),
                                  desc_kmajor(v_s, kk, SLAB64), id_s, kk > 0);
                    umma_commit(&sm.s_full[b]);
                }
                if (u >= 1) {
                    const int uu = u - 1, b = uu & 1, s = uu % BWD_STAGES;
                    if (!mbar_wait(&sm.ds_full[b], (uu >> 1) & 1, a.err, 2504)) break;
                    tc_fence_after();
                    const uint32_t ds_s = smem_u32(sm.ds[b]), k_s = smem_u32(sm.k[s][0]);
                    #pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + TDQ, desc_kmajor(ds_s, kk, SLAB128), desc_mnmajor(k_s, kk, SLAB64),
                                  id_acc, (uu > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.dq_done[b]);
                    umma_commit(&sm.st_empty[s]);
                }
            }
        }
    } else {
        const int r = threadIdx.x;                  // query row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int qh = r >> 6;
        const size_t prow = (size_t)hrow + (size_t)t * 128 + r;
        const float lse2 = a.lse_p[prow];
        const float di = a.di_p[prow];
        bool ok = true;
        HalfIter it{ents, ne, 0, 0, 0};
        int r64, m2;
        for (int u = 0; it.next(r64, m2); ++u) {
            const int b = u & 1;
            const bool valid = (m2 >> qh) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (u >> 1) & 1, a.err, 2001))) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[64], dp[64];
            PRISM_TMEM_LD32(tmem + lane_off + TS + 64 * b, sv);
            PRISM_TMEM_LD32(tmem + lane_off + TS + 64 * b + 32, (sv + 32));
            PRISM_TMEM_LD32(tmem + lane_off + TDP + 64 * b, dp);
            PRISM_TMEM_LD32(tmem + lane_off + TDP + 64 * b + 32, (dp + 32));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.s_free[b]);
            if (u >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.dq_done[b], ((u - 2) >> 1) & 1, a.err, 2003))) {
                ok = false;
                break;
            }
            const uint32_t ds_s = smem_u32(sm.ds[b]);
            #pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t wd[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = ch * 8 + 2 * e;
                    float d0 = 0.f, d1 = 0.f;
                    if (valid) {
                        // P' = 2^15 P and dS = P' (dP 2^-15 - D 2^-15), as in the dK/dV kernel
                        const float p0 = ex2(fmaf(__uint_as_float(sv[c]), scale_log2, lse2));
                        const float p1 = ex2(fmaf(__uint_as_float(sv[c + 1]), scale_log2, lse2));
                        d0 = p0 * fmaf(__uint_as_float(dp[c]), pinv, di);
                        d1 = p1 * fmaf(__uint_as_float(dp[c + 1]), pinv, di);
                    }
                    wd[e] = pack_f16(d0, d1);
                }
                st_shared_v4(ds_s + swz128(r, ch), wd[0], wd[1], wd[2], wd[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.ds_full[b]);
        }
        int srow = a.src[prow];
        if (prism_bad_index(a.err, srow >= 0 && srow < a.N)) srow = 0;               // checking build
        void* orow = a.out_f32 ? static_cast<void*>(a.out0.row<float>(h, srow, HD))
                               : static_cast<void*>(a.out0.row<__nv_bfloat16>(h, srow, HD));
        bool fin = false;
        if (ok && U > 0)
            fin = __all_sync(0xffffffffu, mbar_wait(&sm.dq_done[(U - 1) & 1], ((U - 1) >> 1) & 1, a.err, 2004));
        if (fin) {
            tc_fence_after();
            const float unscale = ldexpf(1.f, dscale_exp(a.dmax[h], a.err));
            #pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                PRISM_TMEM_LD32(tmem + lane_off + TDQ + 32 * c, o);
                tmem_wait_ld();
                store_row(orow, 32 * c, o, ldexpf(a.inv_sqrt_d * unscale, ev - kDsShift - sk), a.out_f32);
            }
        } else if (U == 0) {
            zero_row(orow, HD, a.out_f32);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 4) { __syncwarp(); tmem_dealloc(tmem, 512); }
}

template <int HD>
static int launch_bwd(prism_plan_s* P, const TokenRows& dO, const TokenRows& O, const float* lse,
                      const TokenRows& dQ, const TokenRows& dK, const TokenRows& dV, cudaStream_t s) {
    const Geom& g = P->g;
    char* b = P->ws;
    const int* src = (const int*)(b + P->L.src);
    __half* dOp = (__half*)(b + P->L.dop);
    float* lse_p = (float*)(b + P->L.lse_p);
    float* di_p = (float*)(b + P->L.di_p);
    uint32_t* dmax = (uint32_t*)(b + P->L.dmax);
    int* err = (int*)(b + P->L.err);
    const bool f32 = P->p.out_dtype == PRISM_F32;
    cudaMemsetAsync(dmax, 0, sizeof(uint32_t) * g.heads, s);
    {
        PrismProf prof(P, PRISM_STAGE_BWD_PRE, s);
        const dim3 gmax(296, g.heads);
        if (f32) k_bwd_absmax<float><<<gmax, 256, 0, s>>>(dO, dmax, HD);
        else k_bwd_absmax<__nv_bfloat16><<<gmax, 256, 0, s>>>(dO, dmax, HD);
        P->launches += 1;
    }
    BwdArgs a{};
    a.src = src;
    a.lse_p = lse_p;
    a.di_p = di_p;
    a.dmax = dmax;
    a.N = g.N;
    a.NT = g.NT;
    a.out_f32 = f32;
    a.scale_log2 = kLog2e / sqrtf((float)HD);
    a.inv_sqrt_d = 1.f / sqrtf((float)HD);
    a.qkv_max = (const uint32_t*)(b + P->L.qkv_max);
    a.err = err;
    a.lbase = (const int*)P->lists;
    const int64_t* loff = (const int64_t*)(b + P->L.loff);
    constexpr bool FUSE = HD == 128;
    static_assert(epilogue_fits<HD, FUSE>(), "dK/dV staging does not fit in the Q/dO/dS buffers");
    float* dq_acc = (float*)(b + P->L.dq_acc);
    a.dq_acc = dq_acc;
    float* dk_acc = (float*)(b + P->L.dk_acc);
    float* dv_acc = (float*)(b + P->L.dv_acc);
    const int sm1 = (int)sizeof(DkdvSmem<HD, FUSE>) + 1024;
    const int sm2 = (int)sizeof(DqSmem<HD>) + 1024;
    if (cudaFuncSetAttribute(k_bwd_dkdv<HD, FUSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm1) != cudaSuccess)
        return PRISM_ERR_CUDA;
    if (!FUSE &&
        cudaFuncSetAttribute(k_bwd_dq<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm2) != cudaSuccess)
        return PRISM_ERR_CUDA;
    // chunks of kChunkTiles query tiles (65536 tokens): about 32 MB of dQ
    // accumulator per chunk, so the reduce-adds of the CTAs in flight stay in L2
    a.CQ = kChunkTiles;
    const unsigned chunks = (unsigned)((g.NT + kChunkTiles - 1) / kChunkTiles);
    // the dO copy and the accumulators hold one group of heads: the groups run in turn
    for (int h0 = 0; h0 < g.heads; h0 += g.GH) {
        const int nh = std::min(g.GH, g.heads - h0);
        const size_t acc_bytes = sizeof(float) * (size_t)nh * g.N * HD;
        const dim3 grows((unsigned)((g.N + 7) / 8), nh);
        a.h0 = h0;
        {
            PrismProf prof(P, PRISM_STAGE_BWD_PRE, s);
            if (f32)
                k_bwd_pre<float><<<grows, 256, 0, s>>>(dO, O, lse, src, dmax, dOp, lse_p, di_p, g.N, HD, h0,
                                                       a.qkv_max, err);
            else
                k_bwd_pre<__nv_bfloat16><<<grows, 256, 0, s>>>(dO, O, lse, src, dmax, dOp, lse_p, di_p, g.N, HD,
                                                               h0, a.qkv_max, err);
        }
        // dK, dV (and for head_dim 128 dQ) per key tile over the transposed lists
        a.ptr = (const int*)(b + P->L.kt_ptr);
        a.ent_off = loff + LIST_BWD * (size_t)g.heads;
        {
            PrismProf prof(P, PRISM_STAGE_BWD_DKDV, s);
            if (FUSE) cudaMemsetAsync(dq_acc, 0, acc_bytes, s);
            cudaMemsetAsync(dk_acc, 0, acc_bytes, s);
            cudaMemsetAsync(dv_acc, 0, acc_bytes, s);
            k_bwd_dkdv<HD, FUSE><<<dim3(g.NT, chunks, nh), FUSE ? 480 : 352, sm1, s>>>(
                P->tm_k, P->tm_v, P->tm_q64, P->tm_do64, P->tm_dk, P->tm_dv, a);
            if (f32)
                k_acc_finalize<float><<<grows, 256, 0, s>>>(dk_acc, a.inv_sqrt_d, dK, dv_acc, 1.f / kPScale, dV, src,
                                                            dmax, g.N, HD, h0, a.qkv_max, 0, err);
            else
                k_acc_finalize<__nv_bfloat16><<<grows, 256, 0, s>>>(dk_acc, a.inv_sqrt_d, dK, dv_acc, 1.f / kPScale,
                                                                    dV, src, dmax, g.N, HD, h0, a.qkv_max, 0, err);
        }
        {
            PrismProf prof(P, PRISM_STAGE_BWD_DQ, s);
            if (FUSE) {
                if (f32)
                    k_acc_finalize<float><<<grows, 256, 0, s>>>(dq_acc, a.inv_sqrt_d, dQ, nullptr, 0.f, TokenRows{},
                                                                src, dmax, g.N, HD, h0, a.qkv_max, 1, err);
                else
                    k_acc_finalize<__nv_bfloat16><<<grows, 256, 0, s>>>(dq_acc, a.inv_sqrt_d, dQ, nullptr, 0.f,
                                                                        TokenRows{}, src, dmax, g.N, HD, h0,
                                                                        a.qkv_max, 1, err);
            } else {
                // dQ per query tile over the forward lists (head_dim 64)
                a.ptr = (const int*)(b + P->L.qt_ptr);
                a.ent_off = loff + LIST_FWD * (size_t)g.heads;
                a.out0 = dQ;
                k_bwd_dq<HD><<<dim3(g.NT, nh), 192, sm2, s>>>(P->tm_q, P->tm_do, P->tm_k64, P->tm_v64, a);
            }
        }
        P->launches += 4;
    }
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

}  // namespace prism

int prism_launch_attn_bwd(prism_plan_s* P, const prism::TokenRows& dO, const prism::TokenRows& O, const float* lse,
                          const prism::TokenRows& dQ, const prism::TokenRows& dK, const prism::TokenRows& dV,
                          void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return P->g.D == 128 ? prism::launch_bwd<128>(P, dO, O, lse, dQ, dK, dV, s)
                         : prism::launch_bwd<64>(P, dO, O, lse, dQ, dK, dV, s);
}
