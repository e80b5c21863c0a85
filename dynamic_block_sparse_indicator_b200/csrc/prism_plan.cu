// prism_plan.cu -- Prism's plan (Algorithm 1, stages 1-3) on sm_100a, and the
// host side of the C ABI (validation, workspace layout, plan handle, export).
//
// Method: "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
// Generation Model Training" (arXiv 2610.05416).  Stage 1 follows the
// equations of section "Metode" 1-2 (page xyznot.com/id/paper/2610.05416) and
// the stage list of section "方法步骤详情" (page paper.rainbus.top); stage 3
// follows section "Metode" 3.  Where the pages leave a step open, the kernels
// take the same plain readings as the CPU oracle:
//   - directional profiles are means over the plane orthogonal to the axis;
//   - r = 1/3 each when the three variances sum to zero;
//   - a_bar = zone mean of the audio norm map / its max over zones,
//     v_hat_d = directional variance of the map's slice means / their sum;
//   - rho = channel mean of (mean per-frame spatial variance + variance of the
//     frame differences), divided by its max over the head's zones;
//   - the 16 candidates are ordered by volume then lexicographically, snapping
//     ties go to the lower index; blocks tile a zone in raster order;
//   - Top-p keeps the shortest prefix of (P desc, j asc) whose mass reaches p,
//     the union with Top-k is the first max(k, L) blocks of that order.
// Every decision (B, shape, selection) is taken in fp32; the audio statistics
// are accumulated in fp64 (the map is tiny and its constant regions must give
// exactly zero variance).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <new>

#include "prism_dev.cuh"
#include "prism_internal.h"

namespace prism {

// ------------------------------------------------------------------ geometry
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The selection kernel stages one query block's row of block probabilities in
// shared memory up to kSelSmemRow blocks (192 KB); longer rows (grids above
// 3.1M tokens, e.g. a native 4K layer) go to a global-memory row per CTA of a
// grid-stride launch of kSelGlobalCtas CTAs.
constexpr int kSelSmemRow = 48 * 1024;
constexpr int kSelGlobalCtas = 296;
constexpr int kMaxBlocks = 1 << 18;          // N / 64 limit: 16.7M tokens per head

Geom make_geom(const prism_params* p) {
    Geom g{};
    g.T = p->T; g.H = p->H; g.W = p->W; g.heads = p->heads; g.D = p->head_dim; g.dtype = p->dtype;
    g.Zt = p->T / 8; g.Zh = p->H / 8; g.Zw = p->W / 8;
    g.Nz = g.Zt * g.Zh * g.Zw;
    g.N = (int64_t)p->T * p->H * p->W;
    g.NB = (int)(g.N / 64);
    g.NT = (int)(g.N / 128);
    g.WORDS = (g.NB + 31) / 32;
    // The forward's pass state and the backward's fp32 accumulators and fp16 dO
    // are sized for a group of heads walked in sequence: at least 2M tokens per
    // group (about 16K query tiles per launch, many waves on 148 SMs), one head
    // at a time above that (the 1M-token layer: two heads, 3.6 GB instead of
    // 72 GB for 40 heads).
    g.GH = (int)std::min<int64_t>(p->heads, std::max<int64_t>(1, ((int64_t)1 << 21) / g.N));
    g.SEL_ROWS = g.NB > kSelSmemRow ? kSelGlobalCtas : 0;
    return g;
}

Layout make_layout(const Geom& g) {
    Layout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    const size_t H = (size_t)g.heads, NB = (size_t)g.NB, NT = (size_t)g.NT, N = (size_t)g.N;
    const size_t GH = (size_t)g.GH;
    L.err = take(16);
    L.araw = take(sizeof(double) * g.Nz);
    L.abar = take(sizeof(float) * g.Nz);
    L.vhat = take(sizeof(float) * g.Nz * 3);
    L.zstat = take(sizeof(float) * H * g.Nz * 4);
    L.shape_id = take(H * g.Nz);
    L.zdiff = take(sizeof(float) * H * g.Nz * 7);
    L.zcut = take(H * g.Nz);
    L.shape_id2 = take(H * g.Nz);
    L.rstat = take(sizeof(float) * H * g.Nz * 8);
    L.araw_seg = take(sizeof(double) * g.Nz * 6);
    L.vhat_seg = take(sizeof(float) * g.Nz * 18);
    L.zone_off = take(sizeof(int) * H * (g.Nz + 1));
    L.nblocks = take(sizeof(int) * H);
    L.blk_start = take(sizeof(int) * H * (NB + 1));
    L.t64_blk = take(sizeof(int) * H * NB);
    L.src = take(sizeof(int) * H * N);
    L.qbar = take(sizeof(float) * H * NB * g.D);
    L.kbar = take(sizeof(float) * H * NB * g.D);
    L.sel = take(sizeof(uint32_t) * H * NB * g.WORDS);
    L.selT = take(sizeof(uint32_t) * H * NB * g.WORDS);
    L.row_ptr = take(sizeof(int) * H * (NB + 1));
    L.col_ptr = take(sizeof(int) * H * (NB + 1));
    L.qt_ptr = take(sizeof(int) * H * (NT + 1));
    L.kt_ptr = take(sizeof(int) * H * (NT + 1));
    L.loff = take(sizeof(int64_t) * LIST_KINDS * H);
    L.selrow = take(sizeof(float) * (size_t)g.SEL_ROWS * (NB + NB / 32 + 1));
    L.qkv_max = take(sizeof(uint32_t) * H * 3);
    L.qp = take(2 * H * N * g.D);
    L.kp = take(2 * H * N * g.D);
    L.vp = take(2 * H * N * g.D);
    L.dop = take(2 * GH * N * g.D);
    L.lse_p = take(sizeof(float) * H * N);
    L.di_p = take(sizeof(float) * H * N);
    L.dmax = take(sizeof(uint32_t) * H);
    L.dq_acc = take(sizeof(float) * GH * N * g.D);
    L.dk_acc = take(sizeof(float) * GH * N * g.D);
    L.dv_acc = take(sizeof(float) * GH * N * g.D);
    L.core = off;
    L.col_idx = take(sizeof(int) * H * NB * NB);
    L.row_idx = take(sizeof(int) * H * NB * NB);
    L.qt_ent = take(sizeof(int) * H * NT * NT);
    L.kt_ent = take(sizeof(int) * H * NT * NT);
    L.total = off;
    return L;
}

int validate_params(const prism_params* p) {
    if (!p) return PRISM_ERR_INVALID_ARG;
    if (p->T <= 0 || p->H <= 0 || p->W <= 0) return PRISM_ERR_INVALID_ARG;
    if (p->T % 8 || p->H % 8 || p->W % 8) return PRISM_ERR_INVALID_ARG;
    if (p->heads < 1) return PRISM_ERR_INVALID_ARG;
    if (p->head_dim != 64 && p->head_dim != 128) return PRISM_ERR_INVALID_ARG;
    if (p->dtype != PRISM_BF16 && p->dtype != PRISM_F32) return PRISM_ERR_INVALID_ARG;
    if (p->out_dtype != PRISM_BF16 && p->out_dtype != PRISM_F32) return PRISM_ERR_INVALID_ARG;
    if (p->top_k < 0) return PRISM_ERR_INVALID_ARG;
    if (!(p->top_p >= 0.f && p->top_p <= 1.f)) return PRISM_ERR_INVALID_ARG;
    if (!(p->top_k_frac >= 0.f && p->top_k_frac <= 1.f)) return PRISM_ERR_INVALID_ARG;
    if (p->top_k < 1 && !(p->top_k_frac > 0.f) && p->top_p <= 0.f) return PRISM_ERR_INVALID_ARG;
    if (!(p->alpha >= 0.f) || !std::isfinite(p->alpha)) return PRISM_ERR_INVALID_ARG;
    if (p->shape_mode < PRISM_SHAPE_DYNAMIC || p->shape_mode > PRISM_SHAPE_FIXED) return PRISM_ERR_INVALID_ARG;
    if (p->shape_mode == PRISM_SHAPE_FIXED && (p->fixed_shape < 0 || p->fixed_shape >= 16))
        return PRISM_ERR_INVALID_ARG;
    if (!(p->eps > 0.f) || !std::isfinite(p->eps)) return PRISM_ERR_INVALID_ARG;
    if (!(p->cut_ratio >= 0.f) || !std::isfinite(p->cut_ratio)) return PRISM_ERR_INVALID_ARG;
    if (p->cut_ratio > 0.f && p->shape_mode == PRISM_SHAPE_FIXED) return PRISM_ERR_INVALID_ARG;
    if (!(p->tau256 >= 0.f && p->tau128 >= p->tau256 && p->tau128 <= 1e30f))
        return PRISM_ERR_INVALID_ARG;
    const int64_t N = (int64_t)p->T * p->H * p->W;
    if (N / 64 > kMaxBlocks) return PRISM_ERR_INVALID_ARG;
    if ((int64_t)p->heads * N >= (int64_t)1 << 31) return PRISM_ERR_INVALID_ARG;
    return PRISM_OK;
}

// ---------------------------------------------------------- shape table
// The 16 candidates (b_T, b_H, b_W): volume 64, 128, 256; lexicographic.
__constant__ int8_t c_shape[16][3] = {
    {2, 4, 8}, {2, 8, 4}, {4, 2, 8}, {4, 4, 4}, {4, 8, 2}, {8, 2, 4}, {8, 4, 2},
    {2, 8, 8}, {4, 4, 8}, {4, 8, 4}, {8, 2, 8}, {8, 4, 4}, {8, 8, 2},
    {4, 8, 8}, {8, 4, 8}, {8, 8, 4}};
__constant__ int8_t c_log2shape[16][3] = {
    {1, 2, 3}, {1, 3, 2}, {2, 1, 3}, {2, 2, 2}, {2, 3, 1}, {3, 1, 2}, {3, 2, 1},
    {1, 3, 3}, {2, 2, 3}, {2, 3, 2}, {3, 1, 3}, {3, 2, 2}, {3, 3, 1},
    {2, 3, 3}, {3, 2, 3}, {3, 3, 2}};

struct DevPlan {
    int T, H, W, heads, D, Zh, Zw, Nz, NB, NT, WORDS;
    int64_t N;
    int* err;
    double* araw;
    float* abar;
    float* vhat;
    float* zstat;
    uint8_t* shape_id;
    float* zdiff;          // adaptive temporal boundaries (null when cut_ratio = 0)
    uint8_t* zcut;
    uint8_t* shape_id2;
    float* rstat;
    double* araw_seg;
    float* vhat_seg;
    int* zone_off;
    int* nblocks;
    int* blk_start;
    int* t64_blk;
    int* src;
    float* qbar;
    float* kbar;
    uint32_t* sel;
    uint32_t* selT;
    int* row_ptr;
    int* col_ptr;
    int* qt_ptr;
    int* kt_ptr;
    int* lbase;            // index lists: kind k of head h starts at lbase + loff[k * heads + h]
    int64_t* loff;
    float* selrow;         // staged block rows of the selection (SEL_ROWS > 0)
    int SEL_ROWS;
    uint32_t* qkv_max;     // [heads][3] max |Q|, |K|, |V| bits
    __half* qp;
    __half* kp;
    __half* vp;
};

static DevPlan dev_plan(const prism_plan_s* P) {
    DevPlan d{};
    const Geom& g = P->g;
    const Layout& L = P->L;
    d.T = g.T; d.H = g.H; d.W = g.W; d.heads = g.heads; d.D = g.D; d.Zh = g.Zh; d.Zw = g.Zw;
    d.Nz = g.Nz; d.NB = g.NB; d.NT = g.NT; d.WORDS = g.WORDS; d.N = g.N;
    char* b = P->ws;
    d.err = (int*)(b + L.err);
    d.araw = (double*)(b + L.araw);
    d.abar = (float*)(b + L.abar);
    d.vhat = (float*)(b + L.vhat);
    d.zstat = (float*)(b + L.zstat);
    d.shape_id = (uint8_t*)(b + L.shape_id);
    if (P->has_cuts) {
        d.zdiff = (float*)(b + L.zdiff);
        d.zcut = (uint8_t*)(b + L.zcut);
        d.shape_id2 = (uint8_t*)(b + L.shape_id2);
        d.rstat = (float*)(b + L.rstat);
        d.araw_seg = (double*)(b + L.araw_seg);
        d.vhat_seg = (float*)(b + L.vhat_seg);
    }
    d.zone_off = (int*)(b + L.zone_off);
    d.nblocks = (int*)(b + L.nblocks);
    d.blk_start = (int*)(b + L.blk_start);
    d.t64_blk = (int*)(b + L.t64_blk);
    d.src = (int*)(b + L.src);
    d.qbar = (float*)(b + L.qbar);
    d.kbar = (float*)(b + L.kbar);
    d.sel = (uint32_t*)(b + L.sel);
    d.selT = (uint32_t*)(b + L.selT);
    d.row_ptr = (int*)(b + L.row_ptr);
    d.col_ptr = (int*)(b + L.col_ptr);
    d.qt_ptr = (int*)(b + L.qt_ptr);
    d.kt_ptr = (int*)(b + L.kt_ptr);
    d.lbase = (int*)P->lists;
    d.loff = (int64_t*)(b + L.loff);
    d.selrow = (float*)(b + L.selrow);
    d.qkv_max = (uint32_t*)(b + L.qkv_max);
    d.SEL_ROWS = g.SEL_ROWS;
    d.qp = (__half*)(b + L.qp);
    d.kp = (__half*)(b + L.kp);
    d.vp = (__half*)(b + L.vp);
    return d;
}

__device__ __forceinline__ void dev_fail(int* err, int code) { atomicCAS(err, 0, code); }

// ---------------------------------------------------- block-wide reductions
template <int NT_>
__device__ __forceinline__ float block_sum(float v, float* red) {
    // deterministic: warp xor tree, then warp partials summed in warp order
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
    #pragma unroll
    for (int i = 0; i < NT_ / 32; ++i) s += red[i];
    return s;
}
template <int NT_>
__device__ __forceinline__ int block_sum_int(int v, int* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    int s = 0;
    #pragma unroll
    for (int i = 0; i < NT_ / 32; ++i) s += red[i];
    return s;
}
template <int NT_>
__device__ __forceinline__ float block_max(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
    #pragma unroll
    for (int i = 1; i < NT_ / 32; ++i) s = fmaxf(s, red[i]);
    return s;
}

// Block-wide exclusive scan of `n` ints in place (single CTA of 1024 threads);
// a[n] receives the total.  Deterministic (integer).
__device__ void block_exclusive_scan_inplace(int* a, int n, int* red) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
    int s = 0;
    for (int i = b0; i < b1; ++i) s += a[i];
    // scan of per-thread sums over the block
    __syncthreads();
    red[tid] = s;
    __syncthreads();
    for (int o = 1; o < nt; o <<= 1) {
        int v = tid >= o ? red[tid - o] : 0;
        __syncthreads();
        red[tid] += v;
        __syncthreads();
    }
    int run = red[tid] - s;
    for (int i = b0; i < b1; ++i) { int c = a[i]; a[i] = run; run += c; }
    if (tid == nt - 1) a[n] = red[nt - 1];
    __syncthreads();
}

// ================================================================ stage 1
// Audio terms, head independent.  One CTA per zone; fp64 accumulation.
__global__ void __launch_bounds__(256) k_audio_zone(DevPlan d, const float* __restrict__ amap) {
    const int m = blockIdx.x;
    const int zt = m / (d.Zh * d.Zw), zh = (m / d.Zw) % d.Zh, zw = m % d.Zw;
    __shared__ double v[512];
    __shared__ double sl[3][8];
    for (int i = threadIdx.x; i < 512; i += 256) {
        const int lt = i >> 6, lh = (i >> 3) & 7, lw = i & 7;
        const int64_t n = ((int64_t)(8 * zt + lt) * d.H + 8 * zh + lh) * d.W + 8 * zw + lw;
        v[i] = (double)amap[n];
    }
    __syncthreads();
    if (threadIdx.x < 24) {
        const int ax = threadIdx.x / 8, s = threadIdx.x % 8;
        double acc = 0.0;
        for (int a = 0; a < 8; ++a)
            for (int b = 0; b < 8; ++b) {
                int lt, lh, lw;
                if (ax == 0) { lt = s; lh = a; lw = b; }
                else if (ax == 1) { lt = a; lh = s; lw = b; }
                else { lt = a; lh = b; lw = s; }
                acc += v[(lt << 6) | (lh << 3) | lw];
            }
        sl[ax][s] = acc / 64.0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double mean = 0.0;
        for (int s = 0; s < 8; ++s) mean += sl[0][s];
        mean /= 8.0;
        double sig[3], tot = 0.0;
        for (int ax = 0; ax < 3; ++ax) {
            double a = 0.0;
            for (int s = 0; s < 8; ++s) { double e = sl[ax][s] - mean; a += e * e; }
            sig[ax] = a / 8.0;
            tot += sig[ax];
        }
        d.araw[m] = mean;
        for (int ax = 0; ax < 3; ++ax) d.vhat[m * 3 + ax] = tot > 0.0 ? (float)(sig[ax] / tot) : 0.f;
    }
}

// Audio terms of the six parts a split can make (frames [0, c) and [c, 8) for
// c = 2, 4, 6), head independent: the zone reading applied to each part (mean
// of the map over the part; slice means along T (c or 8 - c slices), H and W
// (8 each); their variances around the part's mean; v_hat = variance / sum).
__global__ void __launch_bounds__(256) k_audio_seg(DevPlan d, const float* __restrict__ amap) {
    const int m = blockIdx.x;
    const int zt = m / (d.Zh * d.Zw), zh = (m / d.Zw) % d.Zh, zw = m % d.Zw;
    __shared__ double v[512];
    for (int i = threadIdx.x; i < 512; i += 256) {
        const int lt = i >> 6, lh = (i >> 3) & 7, lw = i & 7;
        const int64_t n = ((int64_t)(8 * zt + lt) * d.H + 8 * zh + lh) * d.W + 8 * zw + lw;
        v[i] = (double)amap[n];
    }
    __syncthreads();
    if (threadIdx.x < 6) {
        const int ci = threadIdx.x >> 1, part = threadIdx.x & 1, c = 2 * (ci + 1);
        const int t0 = part ? c : 0, t1 = part ? 8 : c, L = t1 - t0;
        double st[8], sh[8], sw[8], tot = 0.0;
        for (int i = 0; i < 8; ++i) st[i] = sh[i] = sw[i] = 0.0;
        for (int lt = t0; lt < t1; ++lt)
            for (int lh = 0; lh < 8; ++lh)
                for (int lw = 0; lw < 8; ++lw) {
                    const double x = v[(lt << 6) | (lh << 3) | lw];
                    st[lt - t0] += x; sh[lh] += x; sw[lw] += x; tot += x;
                }
        const double mean = tot / (64.0 * L);
        double sig[3] = {0.0, 0.0, 0.0};
        for (int i = 0; i < L; ++i) { const double e = st[i] / 64.0 - mean; sig[0] += e * e; }
        for (int i = 0; i < 8; ++i) {
            const double eh = sh[i] / (8.0 * L) - mean, ew = sw[i] / (8.0 * L) - mean;
            sig[1] += eh * eh; sig[2] += ew * ew;
        }
        sig[0] /= L; sig[1] /= 8.0; sig[2] /= 8.0;
        const double s3 = sig[0] + sig[1] + sig[2];
        const int k = m * 6 + threadIdx.x;
        d.araw_seg[k] = mean;
        for (int ax = 0; ax < 3; ++ax) d.vhat_seg[k * 3 + ax] = s3 > 0.0 ? (float)(sig[ax] / s3) : 0.f;
    }
}

__global__ void __launch_bounds__(1024) k_audio_norm(DevPlan d) {
    __shared__ double red[32];
    double mx = 0.0;
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) mx = fmax(mx, d.araw[m]);
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
    for (int i = 1; i < 32; ++i) mx = fmax(mx, red[i]);
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x)
        d.abar[m] = mx > 0.0 ? (float)(d.araw[m] / mx) : 0.f;
}

__global__ void k_audio_none(DevPlan d) {
    for (int m = blockIdx.x * blockDim.x + threadIdx.x; m < d.Nz; m += gridDim.x * blockDim.x) {
        d.abar[m] = 0.f;
        d.vhat[3 * m] = d.vhat[3 * m + 1] = d.vhat[3 * m + 2] = 0.f;
    }
}

// Value statistics per (zone, head): sigma^2_{v,T/H/W} and the raw density.
// Thread = (channel pair, group of h-rows of the zone); one pass over the zone
// with the values shifted by the zone's first token (per channel).
template <typename T>
struct Pair { };
template <>
struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 load(const __nv_bfloat16* p) {
        __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
        return __bfloat1622float2(v);
    }
};
template <>
struct Pair<float> {
    static __device__ __forceinline__ float2 load(const float* p) {
        return *reinterpret_cast<const float2*>(p);
    }
};

// MODE 0: statistics of whole zones.  MODE 1: the same, plus the zone's
// frame-difference energies e_t = mean over its 64 tokens and D channels of
// (V[t+1] - V[t])^2 and its split decision (adaptive temporal boundaries).
// MODE 2: statistics of the two parts of every split zone (grid z = part),
// over the part's frames [t0, t1) only.
template <typename T, int D, int MODE>
__global__ void __launch_bounds__(256) k_zone_stats(DevPlan d, const TokenRows V, float cut_ratio) {
    constexpr int CP = D / 2;            // channel pairs
    constexpr int G = 256 / CP;          // groups
    constexpr int RPG = 8 / G;           // h-rows per group
    constexpr int NE = MODE == 1 ? 7 : 0;
    constexpr int NV = 26 + NE;          // ST[8] SQ[8] SW[8] Dsum Dsq (+ E[7])
    extern __shared__ float zs_dyn[];    // [G][D][NV]
    float (*red)[D][NV] = reinterpret_cast<float (*)[D][NV]>(zs_dyn);
    __shared__ float shs[D][8];
    __shared__ float cst[D][4];
    __shared__ float cse[MODE == 1 ? D : 1][8];
    __shared__ float ez[8];
    const int m = blockIdx.x, h = blockIdx.y;
    int t0 = 0, t1 = 8;
    if (MODE == 2) {
        const int c = d.zcut[(size_t)h * d.Nz + m];
        if (c == 0) return;
        t0 = blockIdx.z ? c : 0;
        t1 = blockIdx.z ? 8 : c;
    }
    const int L = t1 - t0;
    const int zt = m / (d.Zh * d.Zw), zh = (m / d.Zw) % d.Zh, zw = m % d.Zw;
    const int cp = threadIdx.x % CP, grp = threadIdx.x / CP;
    auto tok = [&](int lt, int lh, int lw) -> int64_t {
        return ((int64_t)(8 * zt + lt) * d.H + 8 * zh + lh) * d.W + 8 * zw + lw;
    };
    const float2 ref = Pair<T>::load(V.row_t<const T>(h, 8 * zt + t0, tok(t0, 0, 0), D) + 2 * cp);
    float ST[2][8], SQ[2][8], SW[2][8], SH[2][RPG], Ds[2], Dq[2], Et[2][NE > 0 ? NE : 1];
    #pragma unroll
    for (int c = 0; c < 2; ++c) {
        #pragma unroll
        for (int i = 0; i < 8; ++i) ST[c][i] = SQ[c][i] = SW[c][i] = 0.f;
        #pragma unroll
        for (int i = 0; i < RPG; ++i) SH[c][i] = 0.f;
        #pragma unroll
        for (int i = 0; i < (NE > 0 ? NE : 1); ++i) Et[c][i] = 0.f;
        Ds[c] = Dq[c] = 0.f;
    }
    #pragma unroll
    for (int rr = 0; rr < RPG; ++rr) {
        const int lh = grp * RPG + rr;
        float prev[2][8];
        #pragma unroll
        for (int i = 0; i < 8; ++i) prev[0][i] = prev[1][i] = 0.f;
        #pragma unroll
        for (int lt = 0; lt < 8; ++lt) {
            if (MODE == 2 && (lt < t0 || lt >= t1)) continue;
            float2 x[8];
            const T* vr = V.row_t<const T>(h, 8 * zt + lt, tok(lt, lh, 0), D) + 2 * cp;   // 8 adjacent tokens
            #pragma unroll
            for (int lw = 0; lw < 8; ++lw) x[lw] = Pair<T>::load(vr + lw * D);
            #pragma unroll
            for (int lw = 0; lw < 8; ++lw) {
                const float v0 = x[lw].x - ref.x, v1 = x[lw].y - ref.y;
                ST[0][lt] += v0; ST[1][lt] += v1;
                SQ[0][lt] += v0 * v0; SQ[1][lt] += v1 * v1;
                SW[0][lw] += v0; SW[1][lw] += v1;
                SH[0][rr] += v0; SH[1][rr] += v1;
                if (lt > t0) {
                    const float d0 = v0 - prev[0][lw], d1 = v1 - prev[1][lw];
                    Ds[0] += d0; Ds[1] += d1;
                    Dq[0] += d0 * d0; Dq[1] += d1 * d1;
                    if (MODE == 1) { Et[0][(lt - 1) % 7] += d0 * d0; Et[1][(lt - 1) % 7] += d1 * d1; }
                }
                prev[0][lw] = v0; prev[1][lw] = v1;
            }
        }
    }
    #pragma unroll
    for (int c = 0; c < 2; ++c) {
        float* r = red[grp][2 * cp + c];
        #pragma unroll
        for (int i = 0; i < 8; ++i) { r[i] = ST[c][i]; r[8 + i] = SQ[c][i]; r[16 + i] = SW[c][i]; }
        r[24] = Ds[c]; r[25] = Dq[c];
        #pragma unroll
        for (int i = 0; i < NE; ++i) r[26 + i] = Et[c][i];
        #pragma unroll
        for (int rr = 0; rr < RPG; ++rr) shs[2 * cp + c][grp * RPG + rr] = SH[c][rr];
    }
    __syncthreads();
    // per-part divisors: a whole zone (L = 8) divides by the same constants 64, 8, 448
    const float n_plane = 8.f * (float)L, n_len = (float)L, n_diff = 64.f * (float)(L - 1);
    if (threadIdx.x < D) {
        const int c = threadIdx.x;
        float st[8], sq[8], sw[8], ds = 0.f, dq = 0.f, et[NE > 0 ? NE : 1];
        #pragma unroll
        for (int i = 0; i < 8; ++i) st[i] = sq[i] = sw[i] = 0.f;
        #pragma unroll
        for (int i = 0; i < (NE > 0 ? NE : 1); ++i) et[i] = 0.f;
        for (int g = 0; g < G; ++g) {
            const float* r = red[g][c];
            #pragma unroll
            for (int i = 0; i < 8; ++i) { st[i] += r[i]; sq[i] += r[8 + i]; sw[i] += r[16 + i]; }
            ds += r[24]; dq += r[25];
            #pragma unroll
            for (int i = 0; i < NE; ++i) et[i] += r[26 + i];
        }
        float zsum = 0.f;
        #pragma unroll
        for (int i = 0; i < 8; ++i) zsum += st[i];
        const float mu = zsum / (64.f * n_len);
        float vt = 0.f, vh = 0.f, vw = 0.f, sp = 0.f;
        #pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float eh = shs[c][i] / n_plane - mu, ew = sw[i] / n_plane - mu;
            vh += eh * eh; vw += ew * ew;
            if (i >= t0 && i < t1) {
                const float et_ = st[i] / 64.f - mu;
                vt += et_ * et_;
                const float fm = st[i] / 64.f;
                sp += sq[i] / 64.f - fm * fm;
            }
        }
        const float dm = ds / n_diff;
        const float temporal = dq / n_diff - dm * dm;
        cst[c][0] = vt / n_len; cst[c][1] = vh / 8.f; cst[c][2] = vw / 8.f;
        cst[c][3] = sp / n_len + temporal;
        #pragma unroll
        for (int i = 0; i < NE; ++i) cse[c][i] = et[i];
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        float s = 0.f;
        for (int c = 0; c < D; ++c) s += cst[c][threadIdx.x];
        if (MODE == 2)
            d.rstat[(((size_t)h * d.Nz + m) * 2 + blockIdx.z) * 4 + threadIdx.x] = s / (float)D;
        else
            d.zstat[((size_t)h * d.Nz + m) * 4 + threadIdx.x] = s / (float)D;
    }
    if (MODE == 1) {
        if (threadIdx.x >= 32 && threadIdx.x < 32 + 7) {
            const int t = threadIdx.x - 32;
            float s = 0.f;
            for (int c = 0; c < D; ++c) s += cse[c][t];
            const float e = s / (64.f * (float)D);
            ez[t] = e;
            d.zdiff[((size_t)h * d.Nz + m) * 7 + t] = e;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            // largest energy (lowest t on ties) against cut_ratio x the median of the seven
            int tm = 0;
            float srt[7];
            for (int t = 0; t < 7; ++t) {
                srt[t] = ez[t];
                if (ez[t] > ez[tm]) tm = t;
            }
            for (int i = 1; i < 7; ++i)
                for (int j = i; j > 0 && srt[j - 1] > srt[j]; --j) { const float x = srt[j]; srt[j] = srt[j - 1]; srt[j - 1] = x; }
            int cut = 0;
            if (ez[tm] > __fmul_rn(cut_ratio, srt[3])) {
                const int bnd = tm + 1;                           // boundary frame 1..7
                cut = bnd <= 2 ? 2 : (bnd <= 5 ? 4 : 6);         // nearest of 2, 4, 6; 3 and 5 to 4
            }
            d.zcut[(size_t)h * d.Nz + m] = (uint8_t)cut;
        }
    }
}

// Per head: rho normalisation, volume, closed form, snapping, block offsets.
// Closed form with the mapping exponent alpha (the pages' method: 1/2):
// l*_d = -alpha log2 g_d + 1/3 (S + alpha sum_d' log2 g_d'), so that
// b_d ~ g_d^-alpha and prod b_d = B.
__device__ int snap_shape(const float g[3], int vol, float alpha, int L = 8) {
    const float lg0 = log2f(g[0]), lg1 = log2f(g[1]), lg2 = log2f(g[2]);
    const float S = vol == 64 ? 6.f : (vol == 128 ? 7.f : 8.f);
    float inner = __fadd_rn(S, __fmul_rn(alpha, lg0));
    inner = __fadd_rn(inner, __fmul_rn(alpha, lg1));
    inner = __fadd_rn(inner, __fmul_rn(alpha, lg2));
    const float third = __fdiv_rn(inner, 3.f);
    const float e0 = __fadd_rn(__fmul_rn(-alpha, lg0), third);
    const float e1 = __fadd_rn(__fmul_rn(-alpha, lg1), third);
    const float e2 = __fadd_rn(__fmul_rn(-alpha, lg2), third);
    const int lo = vol == 64 ? 0 : (vol == 128 ? 7 : 13);
    const int hi = vol == 64 ? 7 : (vol == 128 ? 13 : 16);
    // candidates whose time edge divides the region's L frames (all for a whole zone)
    int best = -1;
    float bd = 0.f;
    for (int s = lo; s < hi; ++s) {
        if (L % c_shape[s][0]) continue;
        const float d0 = __fsub_rn((float)c_log2shape[s][0], e0);
        const float d1 = __fsub_rn((float)c_log2shape[s][1], e1);
        const float d2 = __fsub_rn((float)c_log2shape[s][2], e2);
        float dist = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
        dist = __fadd_rn(dist, __fmul_rn(d2, d2));
        if (best < 0 || dist < bd) { best = s; bd = dist; }
    }
    return best;
}

// Shape id of zone m of head h from its statistics (zs: the head's zone
// stats, mx: the head's maximum raw density).
struct ShapeRule {
    float eps, tau128, tau256, alpha;
    int mode, fixed;
};
__device__ int zone_shape(const DevPlan& d, const float* zs, float mx, int m, const ShapeRule& rule) {
    if (rule.mode == PRISM_SHAPE_FIXED) return rule.fixed;
    const float rho = mx > 0.f ? __fdiv_rn(zs[m * 4 + 3], mx) : 0.f;
    const int vol = rho < rule.tau256 ? 256 : (rho < rule.tau128 ? 128 : 64);
    float g[3];
    if (rule.mode == PRISM_SHAPE_ISOTROPIC) {
        g[0] = g[1] = g[2] = 1.f;
    } else {
        const float s0 = zs[m * 4], s1 = zs[m * 4 + 1], s2 = zs[m * 4 + 2];
        const float tot = __fadd_rn(__fadd_rn(s0, s1), s2);
        float r[3];
        if (tot > 0.f) { r[0] = __fdiv_rn(s0, tot); r[1] = __fdiv_rn(s1, tot); r[2] = __fdiv_rn(s2, tot); }
        else { r[0] = r[1] = r[2] = 1.f / 3.f; }
        const float ab = d.abar[m];
        #pragma unroll
        for (int ax = 0; ax < 3; ++ax)
            g[ax] = __fadd_rn(__fadd_rn(r[ax], __fmul_rn(ab, d.vhat[3 * m + ax])), rule.eps);
    }
    return snap_shape(g, vol, rule.alpha);
}

__global__ void __launch_bounds__(1024) k_zone_finalize(DevPlan d, ShapeRule rule, int use_given_shapes) {
    __shared__ float redf[32];
    __shared__ int red[1024];
    extern __shared__ int nbz[];   // [Nz + 1]
    const int h = blockIdx.x;
    const float* zs = d.zstat + (size_t)h * d.Nz * 4;
    uint8_t* sid = d.shape_id + (size_t)h * d.Nz;
    if (!use_given_shapes) {
        float mx = 0.f;
        for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) mx = fmaxf(mx, zs[m * 4 + 3]);
        mx = block_max<1024>(mx, redf);
        for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) sid[m] = (uint8_t)zone_shape(d, zs, mx, m, rule);
        __syncthreads();
    }
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
        const int s = sid[m] < 16 ? sid[m] : 0;
        if (sid[m] >= 16) dev_fail(d.err, PRISM_ERR_DEVICE_CHECK);
        nbz[m] = 512 / (c_shape[s][0] * c_shape[s][1] * c_shape[s][2]);
    }
    __syncthreads();
    block_exclusive_scan_inplace(nbz, d.Nz, red);
    int* zoff = d.zone_off + (size_t)h * (d.Nz + 1);
    int* bs = d.blk_start + (size_t)h * (d.NB + 1);
    int* t64 = d.t64_blk + (size_t)h * d.NB;
    for (int m = threadIdx.x; m <= d.Nz; m += blockDim.x) zoff[m] = nbz[m];
    const int nb = nbz[d.Nz];
    if (threadIdx.x == 0) d.nblocks[h] = nb;
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
        const int s = sid[m] < 16 ? sid[m] : 0;
        const int vol = c_shape[s][0] * c_shape[s][1] * c_shape[s][2];
        const int j0 = nbz[m], cnt = nbz[m + 1] - nbz[m];
        for (int k = 0; k < cnt; ++k) {
            const int st = 512 * m + k * vol;
            bs[j0 + k] = st;
            for (int u = 0; u < vol / 64; ++u) t64[st / 64 + u] = j0 + k;
        }
    }
    for (int j = nb + threadIdx.x; j <= d.NB; j += blockDim.x) bs[j] = (int)d.N;
}

// Shape of one part of a split zone (or a whole zone, L = 8) from its
// statistics st = (sigma2_T, sigma2_H, sigma2_W, rho_raw), the head's maximum
// density mx, its audio coupling ab and v_hat vh.  The volume is capped at the
// largest that tiles L frames (b_T in {2, 4, 8} must divide L: 128 for 2 or 6).
__device__ int region_shape(const float* st, float mx, float ab, const float* vh, int L, const ShapeRule& rule) {
    const float rho = mx > 0.f ? __fdiv_rn(st[3], mx) : 0.f;
    int vol = rho < rule.tau256 ? 256 : (rho < rule.tau128 ? 128 : 64);
    if ((L == 2 || L == 6) && vol == 256) vol = 128;
    float g[3];
    if (rule.mode == PRISM_SHAPE_ISOTROPIC) {
        g[0] = g[1] = g[2] = 1.f;
    } else {
        const float tot = __fadd_rn(__fadd_rn(st[0], st[1]), st[2]);
        float r[3];
        if (tot > 0.f) { r[0] = __fdiv_rn(st[0], tot); r[1] = __fdiv_rn(st[1], tot); r[2] = __fdiv_rn(st[2], tot); }
        else { r[0] = r[1] = r[2] = 1.f / 3.f; }
        #pragma unroll
        for (int ax = 0; ax < 3; ++ax) g[ax] = __fadd_rn(__fadd_rn(r[ax], __fmul_rn(ab, vh[ax])), rule.eps);
    }
    return snap_shape(g, vol, rule.alpha, L);
}

// A split frame outside {0, 2, 4, 6} (an imported plan's mistake) is read as 4
// everywhere, so every index stays inside its zone; finalize reports it.
__device__ __forceinline__ int sane_cut(int c) { return (c == 0 || c == 2 || c == 4 || c == 6) ? c : 4; }

// Parts of zone m (at most two): first frame, length, shape.
__device__ __forceinline__ int zone_parts(const DevPlan& d, int h, int m, int* t0, int* len, int* sh) {
    const size_t k = (size_t)h * d.Nz + m;
    const int c = sane_cut(d.zcut[k]);
    if (c == 0) { t0[0] = 0; len[0] = 8; sh[0] = d.shape_id[k]; return 1; }
    t0[0] = 0; len[0] = c; sh[0] = d.shape_id[k];
    t0[1] = c; len[1] = 8 - c; sh[1] = d.shape_id2[k];
    return 2;
}

// Volume of a part's blocks; a shape id out of range, a split frame other than
// 0, 2, 4, 6, a b_T that does not divide the part's length or a volume that
// does not tile it sets *bad, and the part is tiled with 128-token blocks so
// that every later index stays inside the zone (64 L is a multiple of 128).
__device__ __forceinline__ int part_vol(int sh, int len, int c, bool* bad) {
    *bad = sh >= 16 || (c != 0 && c != 2 && c != 4 && c != 6);
    if (*bad) return 128;
    const int vol = c_shape[sh][0] * c_shape[sh][1] * c_shape[sh][2];
    *bad = (len % c_shape[sh][0]) != 0 || ((64 * len) % vol) != 0;
    return *bad ? 128 : vol;
}

// Finalize with adaptive temporal boundaries: rho and a_bar normalised over
// the head's zones and parts, one shape per part, block offsets and the
// 64-token tile -> block map with each split zone's first part first.
__global__ void __launch_bounds__(1024) k_zone_finalize_cut(DevPlan d, ShapeRule rule, int use_given_shapes,
                                                            int has_audio) {
    __shared__ float redf[32];
    __shared__ double redd[32];
    __shared__ int red[1024];
    extern __shared__ int nbz[];   // [Nz + 1]
    const int h = blockIdx.x;
    const float* zs = d.zstat + (size_t)h * d.Nz * 4;
    const float* rs = d.rstat + (size_t)h * d.Nz * 8;
    const uint8_t* cut = d.zcut + (size_t)h * d.Nz;
    uint8_t* sid = d.shape_id + (size_t)h * d.Nz;
    uint8_t* sid2 = d.shape_id2 + (size_t)h * d.Nz;
    if (!use_given_shapes) {
        float mx = 0.f;
        double ma = 0.0;
        for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
            const int c = cut[m];
            if (c == 0) {
                mx = fmaxf(mx, zs[m * 4 + 3]);
                if (has_audio) ma = fmax(ma, d.araw[m]);
            } else {
                for (int p = 0; p < 2; ++p) {
                    mx = fmaxf(mx, rs[(m * 2 + p) * 4 + 3]);
                    if (has_audio) ma = fmax(ma, d.araw_seg[m * 6 + (c / 2 - 1) * 2 + p]);
                }
            }
        }
        mx = block_max<1024>(mx, redf);
        for (int o = 16; o > 0; o >>= 1) ma = fmax(ma, __shfl_xor_sync(0xffffffffu, ma, o));
        if ((threadIdx.x & 31) == 0) redd[threadIdx.x >> 5] = ma;
        __syncthreads();
        ma = redd[0];
        for (int i = 1; i < 32; ++i) ma = fmax(ma, redd[i]);
        const float zero3[3] = {0.f, 0.f, 0.f};
        for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
            const int c = cut[m];
            if (c == 0) {
                const float ab = has_audio && ma > 0.0 ? (float)(d.araw[m] / ma) : 0.f;
                sid[m] = (uint8_t)region_shape(zs + m * 4, mx, ab, has_audio ? d.vhat + 3 * m : zero3, 8, rule);
                sid2[m] = 255;
            } else {
                for (int p = 0; p < 2; ++p) {
                    const int k = m * 6 + (c / 2 - 1) * 2 + p;
                    const float ab = has_audio && ma > 0.0 ? (float)(d.araw_seg[k] / ma) : 0.f;
                    const int s = region_shape(rs + (m * 2 + p) * 4, mx, ab, has_audio ? d.vhat_seg + 3 * k : zero3,
                                               p ? 8 - c : c, rule);
                    (p ? sid2 : sid)[m] = (uint8_t)s;
                }
            }
        }
        __syncthreads();
    }
    // blocks per zone; a part whose shape cannot tile it is a device-check error
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
        int t0[2], len[2], sh[2];
        const int np = zone_parts(d, h, m, t0, len, sh);
        int nb = 0;
        if (sane_cut(cut[m]) != cut[m]) dev_fail(d.err, PRISM_ERR_DEVICE_CHECK);
        for (int p = 0; p < np; ++p) {
            bool bad;
            const int vol = part_vol(sh[p], len[p], sane_cut(cut[m]), &bad);
            if (bad) dev_fail(d.err, PRISM_ERR_DEVICE_CHECK);
            nb += 64 * len[p] / vol;
        }
        nbz[m] = nb;
    }
    __syncthreads();
    block_exclusive_scan_inplace(nbz, d.Nz, red);
    int* zoff = d.zone_off + (size_t)h * (d.Nz + 1);
    int* bs = d.blk_start + (size_t)h * (d.NB + 1);
    int* t64 = d.t64_blk + (size_t)h * d.NB;
    for (int m = threadIdx.x; m <= d.Nz; m += blockDim.x) zoff[m] = nbz[m];
    const int nbt = nbz[d.Nz];
    if (threadIdx.x == 0) d.nblocks[h] = nbt;
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
        int t0[2], len[2], sh[2];
        const int np = zone_parts(d, h, m, t0, len, sh);
        int j = nbz[m];
        for (int p = 0; p < np; ++p) {
            bool bad;
            const int v = part_vol(sh[p], len[p], sane_cut(cut[m]), &bad);
            const int pos0 = 512 * m + 64 * t0[p];
            const int cnt = 64 * len[p] / v;
            for (int k = 0; k < cnt; ++k, ++j) {
                const int st = pos0 + k * v;
                bs[j] = st;
                for (int u = 0; u < v / 64; ++u) t64[st / 64 + u] = j;
            }
        }
    }
    for (int j = nbt + threadIdx.x; j <= d.NB; j += blockDim.x) bs[j] = (int)d.N;
}

// ================================================================ stage 2
// The block-ordered copies are fp16 (their products' rounding error is 8x below
// bf16's), each head's Q, K and V scaled by an exact power of two that puts the
// head's largest magnitude in [2^14, 2^15) (qkv_shift): any finite input keeps
// fp16's relative precision down to 2^-28 of its head's maximum, and a bf16
// value converts exactly unless it is that small.  A non-finite input is a
// device-check error.

// Largest magnitude of each head's Q, K and V (float bits, atomicMax: the bits
// of non-negative floats order like the values; a NaN's bits exceed infinity's).
// One pass over 16-byte chunks (the inputs are 16-byte aligned and a head holds
// N x D elements, a multiple of 16 bytes); see fold_abs.
template <typename T>
__global__ void __launch_bounds__(256) k_qkv_absmax(const TokenRows Q, const TokenRows K, const TokenRows V,
                                                    uint32_t* __restrict__ mx, int D, int* err) {
    const int h = blockIdx.y;
    const int64_t n16 = Q.S * D * (int64_t)sizeof(T) / 16;      // 16-byte chunks of one shard's head
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m[3] = {0u, 0u, 0u};
    for (int sh = 0; sh < Q.n; ++sh) {
        const int64_t off = ((int64_t)(Q.head0 + h) * Q.S) * D;   // the same layout for Q, K, V
        const uint4* q = reinterpret_cast<const uint4*>(static_cast<const T*>(Q.p[sh]) + off);
        const uint4* k = reinterpret_cast<const uint4*>(static_cast<const T*>(K.p[sh]) + off);
        const uint4* v = reinterpret_cast<const uint4*>(static_cast<const T*>(V.p[sh]) + off);
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + stride < n16; i += 2 * stride) {     // two chunks of each tensor in flight
            const uint4 q0 = __ldg(q + i), q1 = __ldg(q + i + stride);
            const uint4 k0 = __ldg(k + i), k1 = __ldg(k + i + stride);
            const uint4 v0 = __ldg(v + i), v1 = __ldg(v + i + stride);
            m[0] = fold_abs<T>(fold_abs<T>(m[0], q0), q1);
            m[1] = fold_abs<T>(fold_abs<T>(m[1], k0), k1);
            m[2] = fold_abs<T>(fold_abs<T>(m[2], v0), v1);
        }
        if (i < n16) {
            m[0] = fold_abs<T>(m[0], __ldg(q + i));
            m[1] = fold_abs<T>(m[1], __ldg(k + i));
            m[2] = fold_abs<T>(m[2], __ldg(v + i));
        }
    }
    #pragma unroll
    for (int t = 0; t < 3; ++t) {
        uint32_t b = abs_bits<T>(m[t]);
        for (int o = 16; o > 0; o >>= 1) b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
        if ((threadIdx.x & 31) == 0) {
            if (!(b <= 0x7f7fffffu)) atomicCAS(err, 0, PRISM_ERR_DEVICE_CHECK);      // inf or NaN
            atomicMax(mx + h * 3 + t, b);
        }
    }
}

__device__ __forceinline__ uint32_t ph2(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Gather one block: rows in block order into the fp16 copies, raster index of
// each slot into src, and fp32 block means of Q and K (from the input values).
template <typename T, int D>
__global__ void __launch_bounds__(256) k_gather_pool(DevPlan d, const TokenRows Q, const TokenRows K,
                                                     const TokenRows V) {
    constexpr int EPC = 16 / sizeof(T);      // input elements per 16-byte chunk
    constexpr int CPR = D / EPC;             // chunks per row
    constexpr int RP = 256 / CPR;            // rows in flight
    __shared__ float pq[RP][D], pk[RP][D];
    const int j = blockIdx.x, h = blockIdx.y;
    if (j >= d.nblocks[h]) return;
    const int* bs = d.blk_start + (size_t)h * (d.NB + 1);
    const int start = bs[j], vol = bs[j + 1] - start;
    const int m = start >> 9;
    // the block's part of the zone: frames [toff, toff + L), first slot 512 m + 64 toff
    int s, toff = 0, rlo = start - 512 * m;
    if (d.zcut) {
        int t0[2], len[2], sh[2];
        const int np = zone_parts(d, h, m, t0, len, sh);
        const int p = (np == 2 && rlo >= 64 * t0[1]) ? 1 : 0;
        bool bad;
        part_vol(sh[p], len[p], sane_cut(d.zcut[(size_t)h * d.Nz + m]), &bad);
        s = bad ? 7 : sh[p];                     // 2 x 8 x 8 tiles any part (device-check error set)
        toff = t0[p];
        rlo -= 64 * t0[p];
    } else {
        s = d.shape_id[(size_t)h * d.Nz + m];
        s = s < 16 ? s : 0;
    }
    const int bt = c_shape[s][0], bh = c_shape[s][1], bw = c_shape[s][2];
    const int kin = rlo / vol;
    const int nkw = 8 / bw, nkh = 8 / bh;
    const int kw = kin % nkw, kh = (kin / nkw) % nkh, kt = kin / (nkw * nkh);
    const int zt = m / (d.Zh * d.Zw), zh = (m / d.Zw) % d.Zh, zw = m % d.Zw;
    const int c = threadIdx.x % CPR, rl = threadIdx.x / CPR;
    // the copies' exact power-of-two scales (the pooled means use the inputs as they are)
    const float sq = ldexpf(1.f, qkv_shift(d.qkv_max[h * 3])), sk = ldexpf(1.f, qkv_shift(d.qkv_max[h * 3 + 1])),
                sv = ldexpf(1.f, qkv_shift(d.qkv_max[h * 3 + 2]));
    float aq[EPC], ak[EPC];
    #pragma unroll
    for (int e = 0; e < EPC; ++e) aq[e] = ak[e] = 0.f;
    const size_t hoff = (size_t)h * d.N * D;
    for (int r = rl; r < vol; r += RP) {
        const int lw = r % bw, lh = (r / bw) % bh, lt = r / (bw * bh);
        const int ft = 8 * zt + toff + kt * bt + lt;
        const int64_t n = ((int64_t)ft * d.H + 8 * zh + kh * bh + lh) * d.W + 8 * zw + kw * bw + lw;
        if (prism_bad_index(d.err, n >= 0 && n < d.N && start + r < d.N)) continue;
        const size_t dst = hoff + (size_t)(start + r) * D + (size_t)c * EPC;
        if (c == 0) d.src[(size_t)h * d.N + start + r] = (int)n;
        const uint4 q4 = *reinterpret_cast<const uint4*>(Q.row_t<const T>(h, ft, n, D) + c * EPC);
        const uint4 k4 = *reinterpret_cast<const uint4*>(K.row_t<const T>(h, ft, n, D) + c * EPC);
        const uint4 v4 = *reinterpret_cast<const uint4*>(V.row_t<const T>(h, ft, n, D) + c * EPC);
        float fq[EPC], fk[EPC], fv[EPC];
        if constexpr (sizeof(T) == 2) {
            const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&q4);
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&k4);
            const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v4);
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 a0 = __bfloat1622float2(q2[e]), a1 = __bfloat1622float2(k2[e]),
                             a2 = __bfloat1622float2(v2[e]);
                fq[2 * e] = a0.x; fq[2 * e + 1] = a0.y;
                fk[2 * e] = a1.x; fk[2 * e + 1] = a1.y;
                fv[2 * e] = a2.x; fv[2 * e + 1] = a2.y;
            }
        } else {
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                fq[e] = reinterpret_cast<const float*>(&q4)[e];
                fk[e] = reinterpret_cast<const float*>(&k4)[e];
                fv[e] = reinterpret_cast<const float*>(&v4)[e];
            }
        }
        uint32_t oq[EPC / 2], ok[EPC / 2], ov[EPC / 2];
        #pragma unroll
        for (int e = 0; e < EPC / 2; ++e) {
            oq[e] = ph2(fq[2 * e] * sq, fq[2 * e + 1] * sq);
            ok[e] = ph2(fk[2 * e] * sk, fk[2 * e + 1] * sk);
            ov[e] = ph2(fv[2 * e] * sv, fv[2 * e + 1] * sv);
        }
        #pragma unroll
        for (int e = 0; e < EPC; ++e) {
            aq[e] += fq[e];
            ak[e] += fk[e];
        }
        if constexpr (EPC == 8) {
            *reinterpret_cast<uint4*>(d.qp + dst) = make_uint4(oq[0], oq[1], oq[2], oq[3]);
            *reinterpret_cast<uint4*>(d.kp + dst) = make_uint4(ok[0], ok[1], ok[2], ok[3]);
            *reinterpret_cast<uint4*>(d.vp + dst) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
        } else {
            *reinterpret_cast<uint2*>(d.qp + dst) = make_uint2(oq[0], oq[1]);
            *reinterpret_cast<uint2*>(d.kp + dst) = make_uint2(ok[0], ok[1]);
            *reinterpret_cast<uint2*>(d.vp + dst) = make_uint2(ov[0], ov[1]);
        }
    }
    #pragma unroll
    for (int e = 0; e < EPC; ++e) { pq[rl][c * EPC + e] = aq[e]; pk[rl][c * EPC + e] = ak[e]; }
    __syncthreads();
    for (int ch = threadIdx.x; ch < 2 * D; ch += 256) {
        const int cc = ch % D;
        float s2 = 0.f;
        if (ch < D) { for (int r = 0; r < RP; ++r) s2 += pq[r][cc]; }
        else { for (int r = 0; r < RP; ++r) s2 += pk[r][cc]; }
        float* out = (ch < D ? d.qbar : d.kbar) + ((size_t)h * d.NB + j) * D + cc;
        *out = s2 / (float)vol;
    }
}

// ================================================================ stage 3
// One CTA per (query block, head): fp32 logits against every key block,
// softmax, Top-k U Top-p count, and the selected set as a bitmap row.
constexpr int SEL_THREADS = 512;

__device__ __forceinline__ uint32_t fkey(float x) { return __float_as_uint(x); }

// One query block's row: prow holds the row's logits then probabilities (NB
// floats), tiecnt the per-word tie counts (NB / 32 + 1 ints); both in shared or
// global memory.  Called by every thread of the CTA.
template <int D>
__device__ void select_row(const DevPlan& d, int i, int h, float* prow, int* tiecnt, float* redf, int* redi,
                           int top_k, float top_k_frac, float top_p) {
    const int nb = d.nblocks[h];
    int* rowcnt = d.row_ptr + (size_t)h * (d.NB + 1);
    if (i >= nb) {                                  // rows past the head's blocks: empty
        if (threadIdx.x == 0) rowcnt[i] = 0;
        uint32_t* row = d.sel + ((size_t)h * d.NB + i) * d.WORDS;
        for (int w = threadIdx.x; w < d.WORDS; w += SEL_THREADS) row[w] = 0u;
        return;                                     // uniform: i and h are the CTA's
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PL = D / 32;
    float q[PL];
    const float* qb = d.qbar + ((size_t)h * d.NB + i) * D;
    #pragma unroll
    for (int e = 0; e < PL; ++e) q[e] = qb[lane + 32 * e];
    const float* kb = d.kbar + (size_t)h * d.NB * D;
    const float sq = sqrtf((float)D);
    for (int j = warp; j < nb; j += SEL_THREADS / 32) {
        const float* kr = kb + (size_t)j * D;
        float a = 0.f;
        #pragma unroll
        for (int e = 0; e < PL; ++e) a = fmaf(q[e], kr[lane + 32 * e], a);
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) prow[j] = __fdiv_rn(a, sq);
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int j = threadIdx.x; j < nb; j += SEL_THREADS) mx = fmaxf(mx, prow[j]);
    mx = block_max<SEL_THREADS>(mx, redf);
    float z = 0.f;
    for (int j = threadIdx.x; j < nb; j += SEL_THREADS) {
        const float e = expf(prow[j] - mx);
        prow[j] = e;
        z += e;
    }
    z = block_sum<SEL_THREADS>(z, redf);
    for (int j = threadIdx.x; j < nb; j += SEL_THREADS) prow[j] = __fdiv_rn(prow[j], z);
    __syncthreads();

    // L = shortest prefix of (P desc, j asc) with mass >= p
    // k as a fraction of the head's block count: ceil(frac * N_b) in fp32
    const int K = min(top_k_frac > 0.f ? (int)ceilf(__fmul_rn(top_k_frac, (float)nb)) : top_k, nb);
    int L;
    if (top_p >= 1.f) L = nb;
    else if (top_p <= 0.f) L = 0;
    else {
        float tot = 0.f;
        for (int j = threadIdx.x; j < nb; j += SEL_THREADS) tot += prow[j];
        tot = block_sum<SEL_THREADS>(tot, redf);
        if (tot < top_p) L = nb;
        else {
            uint32_t lo = 0u, hi = 0x3F800001u;      // mass(P >= lo) >= p > mass(P >= hi)
            while (hi - lo > 1u) {
                const uint32_t mid = lo + ((hi - lo) >> 1);
                float ms = 0.f;
                for (int j = threadIdx.x; j < nb; j += SEL_THREADS)
                    if (fkey(prow[j]) >= mid) ms += prow[j];
                ms = block_sum<SEL_THREADS>(ms, redf);
                if (ms >= top_p) lo = mid; else hi = mid;
            }
            float mg = 0.f;
            int cg = 0, ct = 0;
            for (int j = threadIdx.x; j < nb; j += SEL_THREADS) {
                const uint32_t k = fkey(prow[j]);
                if (k > lo) { mg += prow[j]; ++cg; }
                else if (k == lo) ++ct;
            }
            mg = block_sum<SEL_THREADS>(mg, redf);
            cg = block_sum_int<SEL_THREADS>(cg, redi);
            ct = block_sum_int<SEL_THREADS>(ct, redi);
            const float v = __uint_as_float(lo);
            int c = 0;
            float acc = mg;
            while (c < ct && acc < top_p) { acc += v; ++c; }
            if (c == 0) c = ct > 0 ? 1 : 0;    // the threshold element itself reached p
            L = cg + c;
        }
    }
    const int cnt = max(K, L);
    // threshold of the first cnt elements of the order
    uint32_t lo = 0u;
    int cgt = 0;
    if (cnt < nb) {
        uint32_t hi = 0x3F800001u;                  // count(P >= lo) >= cnt > count(P >= hi)
        while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            int cc = 0;
            for (int j = threadIdx.x; j < nb; j += SEL_THREADS) cc += fkey(prow[j]) >= mid;
            cc = block_sum_int<SEL_THREADS>(cc, redi);
            if (cc >= cnt) lo = mid; else hi = mid;
        }
        int cc = 0;
        for (int j = threadIdx.x; j < nb; j += SEL_THREADS) cc += fkey(prow[j]) > lo;
        cgt = block_sum_int<SEL_THREADS>(cc, redi);
    }
    const int need = cnt - cgt;                     // ties at the threshold, lowest j first
    uint32_t* row = d.sel + ((size_t)h * d.NB + i) * d.WORDS;
    const int nw = (nb + 31) / 32;
    for (int w = threadIdx.x; w < nw; w += SEL_THREADS) {
        uint32_t tb = 0u;
        if (cnt < nb)
            for (int b = 0; b < 32; ++b) {
                const int j = 32 * w + b;
                if (j < nb && fkey(prow[j]) == lo) tb |= 1u << b;
            }
        tiecnt[w] = __popc(tb);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < nw; ++w) { const int t = tiecnt[w]; tiecnt[w] = run; run += t; }
    }
    __syncthreads();
    for (int w = threadIdx.x; w < d.WORDS; w += SEL_THREADS) {
        uint32_t bits = 0u;
        if (w < nw) {
            if (cnt >= nb) {
                const int left = nb - 32 * w;
                bits = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
            } else {
                int rank = tiecnt[w];
                for (int b = 0; b < 32; ++b) {
                    const int j = 32 * w + b;
                    if (j >= nb) break;
                    const uint32_t k = fkey(prow[j]);
                    if (k > lo) bits |= 1u << b;
                    else if (k == lo) { if (rank < need) bits |= 1u << b; ++rank; }
                }
            }
        }
        row[w] = bits;
    }
    if (threadIdx.x == 0) rowcnt[i] = cnt;
}

// One CTA per (query block, head), the row staged in shared memory.
template <int D>
__global__ void __launch_bounds__(SEL_THREADS) k_select(DevPlan d, int top_k, float top_k_frac, float top_p) {
    extern __shared__ float prow[];                 // [NB] row, then [NB / 32 + 1] tie counts
    __shared__ float redf[SEL_THREADS / 32];
    __shared__ int redi[SEL_THREADS / 32];
    select_row<D>(d, blockIdx.x, blockIdx.y, prow, reinterpret_cast<int*>(prow + d.NB), redf, redi, top_k,
                  top_k_frac, top_p);
}

// Rows longer than shared memory holds: a grid-stride loop over (query block,
// head), each CTA staging its rows in its own slice of global scratch (read
// back from L2 by the bisections).
template <int D>
__global__ void __launch_bounds__(SEL_THREADS) k_select_global(DevPlan d, int top_k, float top_k_frac, float top_p) {
    __shared__ float redf[SEL_THREADS / 32];
    __shared__ int redi[SEL_THREADS / 32];
    float* prow = d.selrow + (size_t)blockIdx.x * (d.NB + d.NB / 32 + 1);
    int* tiecnt = reinterpret_cast<int*>(prow + d.NB);
    const int64_t rows = (int64_t)d.NB * d.heads;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        select_row<D>(d, (int)(r % d.NB), (int)(r / d.NB), prow, tiecnt, redf, redi, top_k, top_k_frac, top_p);
        __syncthreads();                            // the row's scratch is reused by the next row
    }
}

// Bitmap popcount per row (used for imported selections and for the transpose).
__global__ void k_row_popc(const uint32_t* __restrict__ bits, int* __restrict__ cnt, const int* nblocks,
                           int NB, int WORDS) {
    const int h = blockIdx.y;
    const int nb = nblocks[h];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= NB) return;
    int c = 0;
    if (i < nb) {
        const uint32_t* r = bits + ((size_t)h * NB + i) * WORDS;
        const int nw = (nb + 31) / 32;
        for (int w = 0; w < nw; ++w) {
            uint32_t x = r[w];
            if (w == nw - 1 && (nb & 31)) x &= (1u << (nb & 31)) - 1u;
            c += __popc(x);
        }
    }
    cnt[(size_t)h * (NB + 1) + i] = c;
}

// Clear bits beyond nblocks in an imported bitmap (rows and columns).
__global__ void k_mask_bits(uint32_t* bits, const int* nblocks, int NB, int WORDS) {
    const int h = blockIdx.y;
    const int nb = nblocks[h];
    const size_t n = (size_t)NB * WORDS;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / WORDS), w = (int)(e % WORDS);
        uint32_t x = bits[(size_t)h * n + e];
        if (i >= nb || 32 * w >= nb) x = 0u;
        else if (32 * w + 32 > nb) x &= (1u << (nb - 32 * w)) - 1u;
        bits[(size_t)h * n + e] = x;
    }
}

// 32x32 bit-tile transpose: selT[j][i] = sel[i][j].
__global__ void k_transpose_bits(DevPlan d) {
    const int tr = blockIdx.x, w = blockIdx.y, h = blockIdx.z;
    const int lane = threadIdx.x;
    const int i = 32 * tr + lane;
    uint32_t x = 0u;
    if (i < d.nblocks[h]) x = d.sel[((size_t)h * d.NB + i) * d.WORDS + w];
    uint32_t mine = 0u;
    #pragma unroll
    for (int b = 0; b < 32; ++b) {
        const uint32_t col = __ballot_sync(0xffffffffu, (x >> b) & 1u);
        if (lane == b) mine = col;
    }
    const int j = 32 * w + lane;
    if (j < d.NB && tr < d.WORDS) d.selT[((size_t)h * d.NB + j) * d.WORDS + tr] = mine;
}

// Exclusive scan of per-head count arrays [heads][n + 1] in place.
__global__ void __launch_bounds__(1024) k_scan_heads(int* a, int n) {
    __shared__ int red[1024];
    block_exclusive_scan_inplace(a + (size_t)blockIdx.x * (n + 1), n, red);
}

// Bitmap rows -> ascending index lists (CSR from sel, CSC from selT).
__global__ void k_fill_lists(const uint32_t* __restrict__ bits, const int* __restrict__ ptr,
                             int* __restrict__ lbase, const int64_t* __restrict__ loff, const int* nblocks,
                             int NB, int WORDS, int* err) {
    const int i = blockIdx.x, h = blockIdx.y;
    const int nb = nblocks[h];
    if (i >= nb) return;
    const int lane = threadIdx.x;
    const uint32_t* r = bits + ((size_t)h * NB + i) * WORDS;
    const int* p = ptr + (size_t)h * (NB + 1);
    int* out = lbase + loff[h];
    int base = p[i];
    const int end = p[i + 1];
    const int nw = (nb + 31) / 32;
    for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        uint32_t x = w < nw ? r[w] : 0u;
        if (w == nw - 1 && (nb & 31)) x &= (1u << (nb & 31)) - 1u;
        const int pc = __popc(x);
        int incl = pc;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int pos = base + incl - pc;
        while (x) {
            const int b = __ffs(x) - 1;
            x &= x - 1u;
            if (pos < end) out[pos] = 32 * w + b;
            else dev_fail(err, PRISM_ERR_DEVICE_CHECK);
            ++pos;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// Tile lists for the attention kernels.  A 128-token tile holds one block
// part (volume 128/256) or two 64-token blocks; entry = (other tile << 4) | mask
// with mask bit (qhalf * 2 + khalf) set when query half qhalf of the pair
// attends to key half khalf.  Forward: per query tile, over key tiles (from
// sel); backward: per key tile, over query tiles (from selT, same bit order).
__device__ __forceinline__ int bit_of(const uint32_t* rowbits, int j) {
    return (rowbits[j >> 5] >> (j & 31)) & 1u;
}

template <bool FILL>
__global__ void __launch_bounds__(256) k_tile_lists(const uint32_t* __restrict__ bits,
                                                    const int* __restrict__ t64, int* ptr,
                                                    int* lbase, const int64_t* __restrict__ loff, int NB, int NT,
                                                    int WORDS, int transposed, int* err) {
    __shared__ int red[256];
    const int t = blockIdx.x, h = blockIdx.y;
    const int* tb = t64 + (size_t)h * NB;
    const uint32_t* b = bits + (size_t)h * NB * WORDS;
    // own halves: blocks of the two 64-token halves of tile t
    const int a0 = tb[2 * t], a1 = tb[2 * t + 1];
    const uint32_t* r0 = b + (size_t)a0 * WORDS;
    const uint32_t* r1 = b + (size_t)a1 * WORDS;
    const int per = (NT + 255) / 256;
    const int c0 = min(NT, (int)threadIdx.x * per), c1 = min(NT, c0 + per);
    auto mask_of = [&](int o) -> int {
        const int o0 = tb[2 * o], o1 = tb[2 * o + 1];
        // own half x (row bits rx) against other half y (block oy)
        const int m00 = bit_of(r0, o0), m01 = bit_of(r0, o1);
        const int m10 = bit_of(r1, o0), m11 = bit_of(r1, o1);
        // forward: own = query halves, other = key halves: bit (q*2 + k)
        // backward: own = key halves, other = query halves: bit (q*2 + k) = (other*2 + own)
        if (!transposed) return m00 | (m01 << 1) | (m10 << 2) | (m11 << 3);
        return m00 | (m10 << 1) | (m01 << 2) | (m11 << 3);
    };
    int cnt = 0;
    for (int o = c0; o < c1; ++o) cnt += mask_of(o) != 0;
    int* p = ptr + (size_t)h * (NT + 1);
    if (!FILL) {
        const int tot = block_sum_int<256>(cnt, red);
        if (threadIdx.x == 0) p[t] = tot;
        return;
    }
    __syncthreads();
    red[threadIdx.x] = cnt;
    __syncthreads();
    for (int o = 1; o < 256; o <<= 1) {
        const int v = threadIdx.x >= o ? red[threadIdx.x - o] : 0;
        __syncthreads();
        red[threadIdx.x] += v;
        __syncthreads();
    }
    int pos = p[t] + red[threadIdx.x] - cnt;
    const int end = p[t + 1];
    int* e = lbase + loff[h];
    for (int o = c0; o < c1; ++o) {
        const int mk = mask_of(o);
        if (mk) {
            if (pos < end) e[pos] = (o << 4) | mk;
            else dev_fail(err, PRISM_ERR_DEVICE_CHECK);
            ++pos;
        }
    }
}

// ------------------------------------------------------------- host helpers
static int cuda_status(cudaError_t e) { return e == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA; }

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

static int make_tmap(CUtensorMap* m, void* base, int64_t rows, int D, int box_rows) {
    auto enc = get_encode();
    if (!enc) return PRISM_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

static int make_tmap_f32(CUtensorMap* m, void* base, int64_t rows, int D, int box_rows) {
    auto enc = get_encode();
    if (!enc) return PRISM_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 4};
    cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

static int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return PRISM_ERR_UNSUPPORTED;
    return PRISM_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int g_profile_plans = 0;   // prism_profile_plans: timing state of new plans

static ShapeRule shape_rule(const prism_params& p) {
    // alpha 0 stands for the pages' 1/2
    return ShapeRule{p.eps, p.tau128, p.tau256, p.alpha > 0.f ? p.alpha : 0.5f, p.shape_mode, p.fixed_shape};
}

static int plan_common(const prism_params* p, const void* Q, const void* K, const void* V,
                       void* workspace, size_t ws_bytes, prism_plan_s** outP) {
    int st = validate_params(p);
    if (st) return st;
    if (!Q || !K || !V || !workspace) return PRISM_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V)) return PRISM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PRISM_ERR_INVALID_ARG;
    st = check_device();
    if (st) return st;
    Geom g = make_geom(p);
    Layout L = make_layout(g);
    // a workspace with room for the lists at their dense bound plans in one call;
    // one with room for the core alone leaves the lists to prism_plan_attach_lists
    if (ws_bytes < L.core) return PRISM_ERR_WORKSPACE;
    prism_plan_s* P = new (std::nothrow) prism_plan_s();
    if (!P) return PRISM_ERR_CUDA;
    P->p = *p;
    P->g = g;
    P->L = L;
    P->ws = static_cast<char*>(workspace);
    P->ws_bytes = ws_bytes;
    P->profile = g_profile_plans;
    P->lists = ws_bytes >= L.total ? P->ws + L.col_idx : nullptr;
    P->lists_ready = 0;
    cudaGetDevice(&P->device);
    const int64_t rows = (int64_t)g.heads * g.N;      // Q, K, V copies: every head
    const int64_t grows = (int64_t)g.GH * g.N;        // dO copy and accumulators: one head group
    st = make_tmap(&P->tm_q, P->ws + L.qp, rows, g.D, 128);
    if (!st) st = make_tmap(&P->tm_k, P->ws + L.kp, rows, g.D, 128);
    if (!st) st = make_tmap(&P->tm_v, P->ws + L.vp, rows, g.D, 128);
    if (!st) st = make_tmap(&P->tm_do, P->ws + L.dop, grows, g.D, 128);
    if (!st) st = make_tmap(&P->tm_q64, P->ws + L.qp, rows, g.D, 64);
    if (!st) st = make_tmap(&P->tm_k64, P->ws + L.kp, rows, g.D, 64);
    if (!st) st = make_tmap(&P->tm_v64, P->ws + L.vp, rows, g.D, 64);
    if (!st) st = make_tmap(&P->tm_do64, P->ws + L.dop, grows, g.D, 64);
    if (!st) st = make_tmap_f32(&P->tm_dk, P->ws + L.dk_acc, grows, g.D, 32);
    if (!st) st = make_tmap_f32(&P->tm_dv, P->ws + L.dv_acc, grows, g.D, 32);
    if (st) { delete P; return st; }
    *outP = P;
    return PRISM_OK;
}

template <typename T, int D>
static void launch_stats(prism_plan_s* P, const DevPlan& d, const TokenRows& V, cudaStream_t s) {
    const Geom& g = P->g;
    const int sm = (256 / (D / 2)) * D * 26 * (int)sizeof(float);
    if (!P->has_cuts) {
        cudaFuncSetAttribute(k_zone_stats<T, D, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        k_zone_stats<T, D, 0><<<dim3(g.Nz, g.heads), 256, sm, s>>>(d, V, 0.f);
        return;
    }
    // whole zones with their energies and split decisions, then the parts of the split zones
    const int sm1 = (256 / (D / 2)) * D * 33 * (int)sizeof(float);
    cudaFuncSetAttribute(k_zone_stats<T, D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm1);
    k_zone_stats<T, D, 1><<<dim3(g.Nz, g.heads), 256, sm1, s>>>(d, V, P->p.cut_ratio);
    cudaFuncSetAttribute(k_zone_stats<T, D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    k_zone_stats<T, D, 2><<<dim3(g.Nz, g.heads, 2), 256, sm, s>>>(d, V, 0.f);
}

template <typename T, int D>
static void launch_gather(prism_plan_s* P, const DevPlan& d, const TokenRows& Q, const TokenRows& K,
                          const TokenRows& V, cudaStream_t s) {
    const Geom& g = P->g;
    cudaMemsetAsync(d.qkv_max, 0, sizeof(uint32_t) * 3 * g.heads, s);
    k_qkv_absmax<T><<<dim3(296, g.heads), 256, 0, s>>>(Q, K, V, d.qkv_max, D, d.err);
    k_gather_pool<T, D><<<dim3(g.NB, g.heads), 256, 0, s>>>(d, Q, K, V);
}

// Counts and pointers of the index lists (CSR rows already counted by the
// selection or the imported bitmap's popcount; the CSC from the transpose; the
// forward and backward tile lists per 128-token tile), each scanned per head:
// ptr[h][n] then holds the head's list length.
static void launch_list_counts(prism_plan_s* P, const DevPlan& d, cudaStream_t s) {
    const Geom& g = P->g;
    k_scan_heads<<<g.heads, 1024, 0, s>>>(d.row_ptr, g.NB);
    k_transpose_bits<<<dim3(g.WORDS, g.WORDS, g.heads), 32, 0, s>>>(d);
    k_row_popc<<<dim3((g.NB + 255) / 256, g.heads), 256, 0, s>>>(d.selT, d.col_ptr, d.nblocks, g.NB, g.WORDS);
    k_scan_heads<<<g.heads, 1024, 0, s>>>(d.col_ptr, g.NB);
    k_tile_lists<false><<<dim3(g.NT, g.heads), 256, 0, s>>>(d.sel, d.t64_blk, d.qt_ptr, nullptr, nullptr, g.NB, g.NT,
                                                             g.WORDS, 0, d.err);
    k_scan_heads<<<g.heads, 1024, 0, s>>>(d.qt_ptr, g.NT);
    k_tile_lists<false><<<dim3(g.NT, g.heads), 256, 0, s>>>(d.selT, d.t64_blk, d.kt_ptr, nullptr, nullptr, g.NB, g.NT,
                                                             g.WORDS, 1, d.err);
    k_scan_heads<<<g.heads, 1024, 0, s>>>(d.kt_ptr, g.NT);
}

// The lists themselves, at the offsets in d.loff.
static void launch_list_fill(prism_plan_s* P, const DevPlan& d, cudaStream_t s) {
    const Geom& g = P->g;
    const int64_t H = g.heads;
    k_fill_lists<<<dim3(g.NB, g.heads), 32, 0, s>>>(d.sel, d.row_ptr, d.lbase, d.loff + LIST_CSR * H, d.nblocks,
                                                    g.NB, g.WORDS, d.err);
    k_fill_lists<<<dim3(g.NB, g.heads), 32, 0, s>>>(d.selT, d.col_ptr, d.lbase, d.loff + LIST_CSC * H, d.nblocks,
                                                    g.NB, g.WORDS, d.err);
    k_tile_lists<true><<<dim3(g.NT, g.heads), 256, 0, s>>>(d.sel, d.t64_blk, d.qt_ptr, d.lbase, d.loff + LIST_FWD * H,
                                                            g.NB, g.NT, g.WORDS, 0, d.err);
    k_tile_lists<true><<<dim3(g.NT, g.heads), 256, 0, s>>>(d.selT, d.t64_blk, d.kt_ptr, d.lbase, d.loff + LIST_BWD * H,
                                                            g.NB, g.NT, g.WORDS, 1, d.err);
}

static int run_plan(prism_plan_s* P, const TokenRows& Q, const TokenRows& K, const TokenRows& V, const float* amap,
                    const uint8_t* given_shapes, const uint32_t* given_sel, cudaStream_t s,
                    const uint8_t* given_cut = nullptr, const uint8_t* given_sid2 = nullptr) {
    // kernels launched below: audio 1-3, stats 1-2, finalize 1, max + gather 2, select
    // (or mask + popcount) 1-2, list counts 8, list fill 4 (here in one-call plans)
    const int cut_extra = P->has_cuts && !given_shapes ? 1 + (amap ? 1 : 0) : 0;
    P->launches += (given_shapes ? 0 : (amap ? 3 : 2)) + cut_extra + 3 + (given_sel ? 2 : 1) + 8 + (P->lists ? 4 : 0);
    const Geom& g = P->g;
    const prism_params& p = P->p;
    DevPlan d = dev_plan(P);
    cudaMemsetAsync(P->ws + P->L.err, 0, 16, s);
    const bool bf = p.dtype == PRISM_BF16;
    if (!given_shapes) {
        PrismProf prof(P, PRISM_STAGE_PLAN_STATS, s);
        if (amap) {
            k_audio_zone<<<g.Nz, 256, 0, s>>>(d, amap);
            k_audio_norm<<<1, 1024, 0, s>>>(d);
            if (P->has_cuts) k_audio_seg<<<g.Nz, 256, 0, s>>>(d, amap);
        } else {
            k_audio_none<<<(g.Nz + 255) / 256, 256, 0, s>>>(d);
        }
        if (bf && g.D == 128) launch_stats<__nv_bfloat16, 128>(P, d, V, s);
        else if (bf) launch_stats<__nv_bfloat16, 64>(P, d, V, s);
        else if (g.D == 128) launch_stats<float, 128>(P, d, V, s);
        else launch_stats<float, 64>(P, d, V, s);
    } else {
        cudaMemcpyAsync(d.shape_id, given_shapes, (size_t)g.heads * g.Nz, cudaMemcpyDeviceToDevice, s);
        if (P->has_cuts) {
            cudaMemcpyAsync(d.zcut, given_cut, (size_t)g.heads * g.Nz, cudaMemcpyDeviceToDevice, s);
            cudaMemcpyAsync(d.shape_id2, given_sid2, (size_t)g.heads * g.Nz, cudaMemcpyDeviceToDevice, s);
        }
    }
    {
        PrismProf prof(P, PRISM_STAGE_PLAN_SHAPES, s);
        const size_t fin_smem = sizeof(int) * (g.Nz + 1);
        if (P->has_cuts) {
            if (fin_smem > 48 * 1024)
                cudaFuncSetAttribute(k_zone_finalize_cut, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fin_smem);
            k_zone_finalize_cut<<<g.heads, 1024, fin_smem, s>>>(d, shape_rule(p), given_shapes ? 1 : 0,
                                                               amap ? 1 : 0);
        } else {
            if (fin_smem > 48 * 1024)
                cudaFuncSetAttribute(k_zone_finalize, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fin_smem);
            k_zone_finalize<<<g.heads, 1024, fin_smem, s>>>(d, shape_rule(p), given_shapes ? 1 : 0);
        }
    }
    {
        PrismProf prof(P, PRISM_STAGE_PLAN_GATHER, s);
        if (bf && g.D == 128) launch_gather<__nv_bfloat16, 128>(P, d, Q, K, V, s);
        else if (bf) launch_gather<__nv_bfloat16, 64>(P, d, Q, K, V, s);
        else if (g.D == 128) launch_gather<float, 128>(P, d, Q, K, V, s);
        else launch_gather<float, 64>(P, d, Q, K, V, s);
    }
    PrismProf prof_sel(P, PRISM_STAGE_PLAN_SELECT, s);
    if (!given_sel) {
        const size_t sm = sizeof(float) * ((size_t)g.NB + g.NB / 32 + 1);
        if (g.SEL_ROWS > 0) {
            if (g.D == 128)
                k_select_global<128><<<g.SEL_ROWS, SEL_THREADS, 0, s>>>(d, p.top_k, p.top_k_frac, p.top_p);
            else
                k_select_global<64><<<g.SEL_ROWS, SEL_THREADS, 0, s>>>(d, p.top_k, p.top_k_frac, p.top_p);
        } else if (g.D == 128) {
            cudaFuncSetAttribute(k_select<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            k_select<128><<<dim3(g.NB, g.heads), SEL_THREADS, sm, s>>>(d, p.top_k, p.top_k_frac, p.top_p);
        } else {
            cudaFuncSetAttribute(k_select<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            k_select<64><<<dim3(g.NB, g.heads), SEL_THREADS, sm, s>>>(d, p.top_k, p.top_k_frac, p.top_p);
        }
    } else {
        cudaMemcpyAsync(d.sel, given_sel, sizeof(uint32_t) * (size_t)g.heads * g.NB * g.WORDS,
                        cudaMemcpyDeviceToDevice, s);
        k_mask_bits<<<dim3(256, g.heads), 256, 0, s>>>(d.sel, d.nblocks, g.NB, g.WORDS);
        k_row_popc<<<dim3((g.NB + 255) / 256, g.heads), 256, 0, s>>>(d.sel, d.row_ptr, d.nblocks, g.NB, g.WORDS);
    }
    prof_sel.close();
    {
        PrismProf prof(P, PRISM_STAGE_PLAN_LISTS, s);
        launch_list_counts(P, d, s);
        if (P->lists) {
            // one-call plan: every head's lists at their dense bound inside the workspace
            const Layout& L = P->L;
            const int64_t H = g.heads, nb2 = (int64_t)g.NB * g.NB, nt2 = (int64_t)g.NT * g.NT;
            const int64_t base[LIST_KINDS] = {0, (int64_t)(L.row_idx - L.col_idx) / 4,
                                              (int64_t)(L.qt_ent - L.col_idx) / 4, (int64_t)(L.kt_ent - L.col_idx) / 4};
            const int64_t stride[LIST_KINDS] = {nb2, nb2, nt2, nt2};
            P->loff_host.assign(LIST_KINDS * H, 0);
            for (int k = 0; k < LIST_KINDS; ++k) {
                for (int64_t h = 0; h < H; ++h) P->loff_host[k * H + h] = base[k] + h * stride[k];
                P->list_len[k] = H * stride[k];
            }
            cudaMemcpyAsync(P->ws + L.loff, P->loff_host.data(), sizeof(int64_t) * LIST_KINDS * H,
                            cudaMemcpyHostToDevice, s);
            launch_list_fill(P, d, s);
            P->lists_ready = 1;
        }
    }
    return cuda_status(cudaGetLastError());
}

// Lengths of the four index lists of every head (synchronises the stream):
// the totals the per-head scans left in the last pointer of each head.
static int read_list_lengths(prism_plan_s* P, cudaStream_t s, std::vector<int>* len) {
    const Geom& g = P->g;
    const Layout& L = P->L;
    const size_t H = g.heads;
    len->assign(LIST_KINDS * H, 0);
    const size_t ptr_off[LIST_KINDS] = {L.row_ptr, L.col_ptr, L.qt_ptr, L.kt_ptr};
    const size_t n[LIST_KINDS] = {(size_t)g.NB, (size_t)g.NB, (size_t)g.NT, (size_t)g.NT};
    for (int k = 0; k < LIST_KINDS; ++k) {
        const char* src = P->ws + ptr_off[k] + sizeof(int) * n[k];      // ptr[h][n] of head 0
        if (cudaMemcpy2DAsync(len->data() + k * H, sizeof(int), src, sizeof(int) * (n[k] + 1), sizeof(int), H,
                              cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return PRISM_ERR_CUDA;
    }
    return cudaStreamSynchronize(s) == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}

}  // namespace prism

using namespace prism;

// ================================================================== C ABI
extern "C" size_t prism_plan_workspace_bytes(const prism_params* p) {
    if (validate_params(p) != PRISM_OK) return 0;
    return make_layout(make_geom(p)).total;
}

extern "C" size_t prism_plan_core_bytes(const prism_params* p) {
    if (validate_params(p) != PRISM_OK) return 0;
    return make_layout(make_geom(p)).core;
}

extern "C" int prism_plan_list_bytes(prism_plan_t P, size_t* bytes, void* stream) {
    if (!P || !bytes) return PRISM_ERR_INVALID_ARG;
    *bytes = 0;
    if (P->lists_ready) return PRISM_OK;
    std::vector<int> len;
    const int st = read_list_lengths(P, static_cast<cudaStream_t>(stream), &len);
    if (st) return st;
    // packed: kind after kind, heads in order inside each kind
    const int64_t H = P->g.heads;
    P->loff_host.assign(LIST_KINDS * H, 0);
    int64_t pos = 0;
    for (int k = 0; k < LIST_KINDS; ++k) {
        const int64_t k0 = pos;
        for (int64_t h = 0; h < H; ++h) {
            P->loff_host[k * H + h] = pos;
            pos += len[k * H + h];
        }
        P->list_len[k] = pos - k0;
    }
    *bytes = sizeof(int) * (size_t)std::max<int64_t>(pos, 1);
    return PRISM_OK;
}

extern "C" int prism_plan_attach_lists(prism_plan_t P, void* lists, size_t bytes, void* stream) {
    if (!P || !lists || !aligned16(lists)) return PRISM_ERR_INVALID_ARG;
    if (P->lists_ready) return PRISM_ERR_INVALID_ARG;
    if (P->loff_host.empty()) return PRISM_ERR_INVALID_ARG;          // prism_plan_list_bytes first
    int64_t need = 0;
    for (int k = 0; k < LIST_KINDS; ++k) need += P->list_len[k];
    if (bytes < sizeof(int) * (size_t)std::max<int64_t>(need, 1)) return PRISM_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    P->lists = static_cast<char*>(lists);
    const DevPlan d = dev_plan(P);
    cudaMemcpyAsync(P->ws + P->L.loff, P->loff_host.data(), sizeof(int64_t) * P->loff_host.size(),
                    cudaMemcpyHostToDevice, s);
    {
        PrismProf prof(P, PRISM_STAGE_PLAN_LISTS, s);
        launch_list_fill(P, d, s);
    }
    P->launches += 4;
    P->lists_ready = 1;
    return cuda_status(cudaGetLastError());
}

extern "C" int prism_plan(const prism_params* p, const void* Q, const void* K, const void* V,
                          const float* a_map, void* workspace, size_t ws_bytes, void* stream,
                          prism_plan_t* out) {
    if (!out) return PRISM_ERR_INVALID_ARG;
    *out = nullptr;
    if (a_map && !aligned16(a_map)) return PRISM_ERR_INVALID_ARG;
    prism_plan_s* P = nullptr;
    int st = plan_common(p, Q, K, V, workspace, ws_bytes, &P);
    if (st) return st;
    P->has_audio = a_map != nullptr;
    P->has_cuts = p->cut_ratio > 0.f;
    const Geom& g = P->g;
    st = run_plan(P, plain_rows(Q, g.T, (int64_t)g.H * g.W, g.heads), plain_rows(K, g.T, (int64_t)g.H * g.W, g.heads),
                  plain_rows(V, g.T, (int64_t)g.H * g.W, g.heads), a_map, nullptr, nullptr, static_cast<cudaStream_t>(stream));
    if (st) { delete P; return st; }
    *out = P;
    return PRISM_OK;
}

extern "C" int prism_plan_sharded(const prism_params* p, const void* const* Q, const void* const* K,
                                  const void* const* V, int shards, int heads_total, int head0,
                                  const float* a_map, void* workspace, size_t ws_bytes, void* stream,
                                  prism_plan_t* out) {
    if (!out) return PRISM_ERR_INVALID_ARG;
    *out = nullptr;
    if (!p || !Q || !K || !V || shards < 1 || shards > kMaxShards) return PRISM_ERR_INVALID_ARG;
    if (a_map && !aligned16(a_map)) return PRISM_ERR_INVALID_ARG;
    if (p->T % shards != 0 || head0 < 0 || heads_total < 1 || p->heads < 1 || head0 + p->heads > heads_total)
        return PRISM_ERR_INVALID_ARG;
    for (int i = 0; i < shards; ++i)
        if (!Q[i] || !K[i] || !V[i] || !aligned16(Q[i]) || !aligned16(K[i]) || !aligned16(V[i]))
            return PRISM_ERR_INVALID_ARG;
    prism_plan_s* P = nullptr;
    int st = plan_common(p, Q[0], K[0], V[0], workspace, ws_bytes, &P);
    if (st) return st;
    P->has_audio = a_map != nullptr;
    P->has_cuts = p->cut_ratio > 0.f;
    const Geom& g = P->g;
    const int64_t HW = (int64_t)g.H * g.W;
    st = run_plan(P, shard_rows(Q, shards, g.T, HW, heads_total, head0), shard_rows(K, shards, g.T, HW, heads_total, head0),
                  shard_rows(V, shards, g.T, HW, heads_total, head0), a_map, nullptr, nullptr,
                  static_cast<cudaStream_t>(stream));
    if (st) { delete P; return st; }
    *out = P;
    return PRISM_OK;
}

extern "C" int prism_plan_import_cuts(const prism_params* p, const void* Q, const void* K, const void* V,
                                      const uint8_t* shape_id, const uint8_t* zone_cut, const uint8_t* shape_id2,
                                      const uint32_t* sel, void* workspace, size_t ws_bytes, void* stream,
                                      prism_plan_t* out) {
    if (!out) return PRISM_ERR_INVALID_ARG;
    *out = nullptr;
    if (!shape_id || !sel || !aligned16(sel)) return PRISM_ERR_INVALID_ARG;
    if ((zone_cut == nullptr) != (shape_id2 == nullptr)) return PRISM_ERR_INVALID_ARG;
    prism_plan_s* P = nullptr;
    int st = plan_common(p, Q, K, V, workspace, ws_bytes, &P);
    if (st) return st;
    P->has_audio = 0;
    P->has_cuts = zone_cut != nullptr;
    const Geom& g = P->g;
    st = run_plan(P, plain_rows(Q, g.T, (int64_t)g.H * g.W, g.heads), plain_rows(K, g.T, (int64_t)g.H * g.W, g.heads),
                  plain_rows(V, g.T, (int64_t)g.H * g.W, g.heads), nullptr, shape_id, sel, static_cast<cudaStream_t>(stream),
                  zone_cut, shape_id2);
    if (st) { delete P; return st; }
    *out = P;
    return PRISM_OK;
}

extern "C" int prism_plan_import_sharded(const prism_params* p, const void* const* Q, const void* const* K,
                                         const void* const* V, int shards, int heads_total, int head0,
                                         const uint8_t* shape_id, const uint8_t* zone_cut,
                                         const uint8_t* shape_id2, const uint32_t* sel, void* workspace,
                                         size_t ws_bytes, void* stream, prism_plan_t* out) {
    if (!out) return PRISM_ERR_INVALID_ARG;
    *out = nullptr;
    if (!p || !Q || !K || !V || shards < 1 || shards > kMaxShards) return PRISM_ERR_INVALID_ARG;
    if (!shape_id || !sel || !aligned16(sel)) return PRISM_ERR_INVALID_ARG;
    if ((zone_cut == nullptr) != (shape_id2 == nullptr)) return PRISM_ERR_INVALID_ARG;
    if (p->T % shards != 0 || head0 < 0 || heads_total < 1 || p->heads < 1 || head0 + p->heads > heads_total)
        return PRISM_ERR_INVALID_ARG;
    for (int i = 0; i < shards; ++i)
        if (!Q[i] || !K[i] || !V[i] || !aligned16(Q[i]) || !aligned16(K[i]) || !aligned16(V[i]))
            return PRISM_ERR_INVALID_ARG;
    prism_plan_s* P = nullptr;
    int st = plan_common(p, Q[0], K[0], V[0], workspace, ws_bytes, &P);
    if (st) return st;
    P->has_audio = 0;
    P->has_cuts = zone_cut != nullptr;
    const Geom& g = P->g;
    const int64_t HW = (int64_t)g.H * g.W;
    st = run_plan(P, shard_rows(Q, shards, g.T, HW, heads_total, head0), shard_rows(K, shards, g.T, HW, heads_total, head0),
                  shard_rows(V, shards, g.T, HW, heads_total, head0), nullptr, shape_id, sel,
                  static_cast<cudaStream_t>(stream), zone_cut, shape_id2);
    if (st) { delete P; return st; }
    *out = P;
    return PRISM_OK;
}

extern "C" int prism_plan_import(const prism_params* p, const void* Q, const void* K, const void* V,
                                 const uint8_t* shape_id, const uint32_t* sel, void* workspace,
                                 size_t ws_bytes, void* stream, prism_plan_t* out) {
    return prism_plan_import_cuts(p, Q, K, V, shape_id, nullptr, nullptr, sel, workspace, ws_bytes, stream, out);
}

extern "C" size_t prism_plan_item_bytes(prism_plan_t P, int item) {
    if (!P) return 0;
    const Geom& g = P->g;
    const size_t H = g.heads, NB = g.NB;
    switch (item) {
        case PRISM_ITEM_SHAPE_ID: return H * g.Nz;
        case PRISM_ITEM_NBLOCKS: return 4 * H;
        case PRISM_ITEM_BLK_START: return 4 * H * (NB + 1);
        case PRISM_ITEM_SEL_BITS: return 4 * H * NB * g.WORDS;
        case PRISM_ITEM_ROW_PTR: return 4 * H * (NB + 1);
        case PRISM_ITEM_COL_IDX: return P->lists_ready ? 4 * (size_t)P->list_len[LIST_CSR] : 0;
        case PRISM_ITEM_COL_PTR: return 4 * H * (NB + 1);
        case PRISM_ITEM_ROW_IDX: return P->lists_ready ? 4 * (size_t)P->list_len[LIST_CSC] : 0;
        case PRISM_ITEM_LIST_OFFSETS: return P->lists_ready ? 8 * LIST_KINDS * H : 0;
        case PRISM_ITEM_QBAR: return 4 * H * NB * g.D;
        case PRISM_ITEM_KBAR: return 4 * H * NB * g.D;
        case PRISM_ITEM_SRC: return 4 * H * (size_t)g.N;
        case PRISM_ITEM_ZONE_STATS: return 4 * H * g.Nz * 4;
        case PRISM_ITEM_ZONE_CUT: return P->has_cuts ? H * g.Nz : 0;
        case PRISM_ITEM_SHAPE_ID2: return P->has_cuts ? H * g.Nz : 0;
        case PRISM_ITEM_ZONE_ENERGY: return P->has_cuts ? 4 * H * g.Nz * 7 : 0;
        case PRISM_ITEM_REGION_STATS: return P->has_cuts ? 4 * H * g.Nz * 8 : 0;
        case PRISM_ITEM_QKV_MAX: return 4 * H * 3;
        default: return 0;
    }
}

extern "C" int prism_plan_export(prism_plan_t P, int item, void* host_dst, size_t bytes, void* stream) {
    if (!P || !host_dst) return PRISM_ERR_INVALID_ARG;
    const size_t need = prism_plan_item_bytes(P, item);
    if (need == 0 || bytes != need) return PRISM_ERR_INVALID_ARG;
    const Layout& L = P->L;
    const int64_t H = P->g.heads;
    if (item == PRISM_ITEM_LIST_OFFSETS) {       // host copy: each head's offset inside its kind's list
        int64_t* out = static_cast<int64_t*>(host_dst);
        for (int k = 0; k < LIST_KINDS; ++k)
            for (int64_t h = 0; h < H; ++h) out[k * H + h] = P->loff_host[k * H + h] - P->loff_host[k * H];
        return PRISM_OK;
    }
    if (item == PRISM_ITEM_COL_IDX || item == PRISM_ITEM_ROW_IDX) {
        const int k = item == PRISM_ITEM_COL_IDX ? LIST_CSR : LIST_CSC;
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
        const char* src = P->lists + sizeof(int) * (size_t)P->loff_host[k * H];
        return cudaMemcpy(host_dst, src, bytes, cudaMemcpyDeviceToHost) == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
    }
    size_t off;
    switch (item) {
        case PRISM_ITEM_SHAPE_ID: off = L.shape_id; break;
        case PRISM_ITEM_NBLOCKS: off = L.nblocks; break;
        case PRISM_ITEM_BLK_START: off = L.blk_start; break;
        case PRISM_ITEM_SEL_BITS: off = L.sel; break;
        case PRISM_ITEM_ROW_PTR: off = L.row_ptr; break;
        case PRISM_ITEM_COL_PTR: off = L.col_ptr; break;
        case PRISM_ITEM_QBAR: off = L.qbar; break;
        case PRISM_ITEM_KBAR: off = L.kbar; break;
        case PRISM_ITEM_SRC: off = L.src; break;
        case PRISM_ITEM_ZONE_STATS: off = L.zstat; break;
        case PRISM_ITEM_ZONE_CUT: off = L.zcut; break;
        case PRISM_ITEM_SHAPE_ID2: off = L.shape_id2; break;
        case PRISM_ITEM_ZONE_ENERGY: off = L.zdiff; break;
        case PRISM_ITEM_REGION_STATS: off = L.rstat; break;
        case PRISM_ITEM_QKV_MAX: off = L.qkv_max; break;
        default: return PRISM_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
    if (cudaMemcpy(host_dst, P->ws + off, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return PRISM_ERR_CUDA;
    return PRISM_OK;
}

extern "C" int prism_get_status(prism_plan_t P, void* stream) {
    return prism_get_status_ex(P, nullptr, stream);
}

extern "C" int prism_get_status_ex(prism_plan_t P, int32_t* site, void* stream) {
    if (!P) return PRISM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
    int e[4] = {0, 0, 0, 0};
    if (cudaMemcpy(e, P->ws + P->L.err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return PRISM_ERR_CUDA;
    if (site) *site = e[0] ? e[1] : 0;
    if (e[0]) {
        const int zero[4] = {0, 0, 0, 0};
        cudaMemcpy(P->ws + P->L.err, zero, sizeof(zero), cudaMemcpyHostToDevice);
    }
    return e[0];
}

static void drop_events(prism_plan_s* P) {
    for (auto& t : P->timed) { cudaEventDestroy(t.a); cudaEventDestroy(t.b); }
    P->timed.clear();
}

extern "C" void prism_plan_destroy(prism_plan_t P) {
    if (!P) return;
    drop_events(P);
    delete P;
}

extern "C" int prism_profile_plans(int on) {
    const int prev = g_profile_plans;
    g_profile_plans = on ? 1 : 0;
    return prev;
}

extern "C" int prism_profile_enable(prism_plan_t P, int on) {
    if (!P) return PRISM_ERR_INVALID_ARG;
    P->profile = on ? 1 : 0;
    return PRISM_OK;
}

extern "C" int prism_profile_read(prism_plan_t P, float* ms, int* launches, void* stream) {
    if (!P || !ms) return PRISM_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PRISM_ERR_CUDA;
    for (int i = 0; i < PRISM_STAGE_COUNT; ++i) { ms[i] = 0.f; if (launches) launches[i] = 0; }
    int st = PRISM_OK;
    for (auto& t : P->timed) {
        float e = 0.f;
        if (cudaEventSynchronize(t.b) != cudaSuccess || cudaEventElapsedTime(&e, t.a, t.b) != cudaSuccess)
            st = PRISM_ERR_CUDA;
        if (t.stage >= 0 && t.stage < PRISM_STAGE_COUNT) {
            ms[t.stage] += e;
            if (launches) launches[t.stage] += 1;
        }
    }
    drop_events(P);
    return st;
}

extern "C" int prism_selftest_timeout(prism_plan_t P, void* stream) {
    if (!P) return PRISM_ERR_INVALID_ARG;
    return prism_launch_selftest_wait(P, stream);
}

extern "C" int64_t prism_launch_count(prism_plan_t P) { return P ? P->launches : 0; }

extern "C" const char* prism_status_string(int st) {
    switch (st) {
        case PRISM_OK: return "ok";
        case PRISM_ERR_INVALID_ARG: return "invalid argument";
        case PRISM_ERR_WORKSPACE: return "workspace too small";
        case PRISM_ERR_CUDA: return "CUDA error";
        case PRISM_ERR_TIMEOUT: return "device wait timed out";
        case PRISM_ERR_DEVICE_CHECK: return "device-side check failed";
        case PRISM_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
        case PRISM_ERR_SCRATCH_LIMIT: return "problem larger than the no-allocation entry point's static scratch";
        default: return "unknown status";
    }
}

extern "C" const char* prism_version(void) { return "prism-b200 0.1 sm_100a"; }

extern "C" int prism_attn_fwd(prism_plan_t P, void* O, float* lse, void* stream) {
    if (!P || !O || !lse || !P->lists_ready) return PRISM_ERR_INVALID_ARG;
    if (!aligned16(O) || !aligned16(lse)) return PRISM_ERR_INVALID_ARG;
    const Geom& g = P->g;
    return prism_launch_attn_fwd(P, plain_rows(O, g.T, (int64_t)g.H * g.W, g.heads), lse, stream);
}

extern "C" int prism_attn_bwd(prism_plan_t P, const void* dO, const void* O, const float* lse,
                              void* dQ, void* dK, void* dV, void* stream) {
    if (!P || !dO || !O || !lse || !dQ || !dK || !dV || !P->lists_ready) return PRISM_ERR_INVALID_ARG;
    if (!aligned16(dO) || !aligned16(O) || !aligned16(lse) || !aligned16(dQ) || !aligned16(dK) ||
        !aligned16(dV))
        return PRISM_ERR_INVALID_ARG;
    const Geom& g = P->g;
    const int64_t HW = (int64_t)g.H * g.W;
    return prism_launch_attn_bwd(P, plain_rows(dO, g.T, HW, g.heads), plain_rows(O, g.T, HW, g.heads), lse,
                                 plain_rows(dQ, g.T, HW, g.heads), plain_rows(dK, g.T, HW, g.heads),
                                 plain_rows(dV, g.T, HW, g.heads), stream);
}

// The shard layout arguments of the *_sharded entry points: shards dividing T,
// a head range inside the shards' heads, non-null 16-byte aligned pointers.
static bool shards_ok(const prism_plan_s* P, int shards, int heads_total, int head0,
                      std::initializer_list<const void* const*> arrays) {
    if (!P || shards < 1 || shards > kMaxShards || P->g.T % shards != 0) return false;
    if (head0 < 0 || heads_total < 1 || head0 + P->g.heads > heads_total) return false;
    for (const void* const* xs : arrays) {
        if (!xs) return false;
        for (int i = 0; i < shards; ++i)
            if (!xs[i] || !aligned16(xs[i])) return false;
    }
    return true;
}

extern "C" int prism_attn_fwd_sharded(prism_plan_t P, void* const* O, int shards, int heads_total, int head0,
                                      float* lse, void* stream) {
    if (!P || !lse || !aligned16(lse) || !P->lists_ready) return PRISM_ERR_INVALID_ARG;
    if (!shards_ok(P, shards, heads_total, head0, {O})) return PRISM_ERR_INVALID_ARG;
    const Geom& g = P->g;
    return prism_launch_attn_fwd(P, shard_rows(O, shards, g.T, (int64_t)g.H * g.W, heads_total, head0), lse,
                                 stream);
}

extern "C" int prism_attn_bwd_sharded(prism_plan_t P, const void* const* dO, const void* const* O,
                                      const float* lse, void* const* dQ, void* const* dK, void* const* dV,
                                      int shards, int heads_total, int head0, void* stream) {
    if (!P || !lse || !aligned16(lse) || !P->lists_ready) return PRISM_ERR_INVALID_ARG;
    if (!shards_ok(P, shards, heads_total, head0, {dO, O, dQ, dK, dV})) return PRISM_ERR_INVALID_ARG;
    const Geom& g = P->g;
    const int64_t HW = (int64_t)g.H * g.W;
    auto rows = [&](const void* const* xs) { return shard_rows(xs, shards, g.T, HW, heads_total, head0); };
    return prism_launch_attn_bwd(P, rows(dO), rows(O), lse, rows(dQ), rows(dK), rows(dV), stream);
}

// ====================================================== no-allocation stage 1
// Some callers cannot allocate device memory at all: a plugin that lives inside
// another engine's fixed memory plan and may only use the buffers it is handed,
// code on a latency-critical path where cudaMalloc's implicit device
// synchronisation is not acceptable, or a deployment whose device memory budget
// is fixed up front.  For them stage 1 (zone statistics -> block volume ->
// shape) runs with its intermediates in this file-scope device array instead
// of a caller workspace.  Every GPU that loads the library holds the array
// until the process exits.
namespace prism {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;   // 4 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Floats of scratch used for (Nz zones, heads): audio zone means (fp64), a_bar,
// v_hat and the per-head zone statistics, each region 256-byte aligned.
static size_t noalloc_floats(int Nz, int heads, size_t* off_abar, size_t* off_vhat, size_t* off_zstat) {
    auto up = [](size_t f) { return (f + 63) & ~size_t(63); };
    size_t o = up(2 * (size_t)Nz);
    *off_abar = o;
    o = up(o + Nz);
    *off_vhat = o;
    o = up(o + 3 * (size_t)Nz);
    *off_zstat = o;
    return o + 4 * (size_t)Nz * heads;
}

// Variant of k_zone_finalize that stops at the shapes: shape id per zone and
// the head's block count, no block offsets.
__global__ void __launch_bounds__(1024) k_zone_shapes_static(DevPlan d, ShapeRule rule,
                                                             uint8_t* __restrict__ sid_out,
                                                             int* __restrict__ nblocks_out) {
    __shared__ float redf[32];
    __shared__ int redi[32];
    const int h = blockIdx.x;
    const float* zs = d.zstat + (size_t)h * d.Nz * 4;
    float mx = 0.f;
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) mx = fmaxf(mx, zs[m * 4 + 3]);
    mx = block_max<1024>(mx, redf);
    int blocks = 0;
    for (int m = threadIdx.x; m < d.Nz; m += blockDim.x) {
        const int s = zone_shape(d, zs, mx, m, rule);
        sid_out[(size_t)h * d.Nz + m] = (uint8_t)s;
        blocks += 512 / (c_shape[s][0] * c_shape[s][1] * c_shape[s][2]);
    }
    blocks = block_sum_int<1024>(blocks, redi);
    if (threadIdx.x == 0) nblocks_out[h] = blocks;
}

template <typename T, int D>
static void noalloc_stats(const Geom& g, const DevPlan& d, const void* V, cudaStream_t s) {
    const int sm = (256 / (D / 2)) * D * 26 * (int)sizeof(float);
    cudaFuncSetAttribute(k_zone_stats<T, D, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    k_zone_stats<T, D, 0><<<dim3(g.Nz, g.heads), 256, sm, s>>>(d, plain_rows(V, g.T, (int64_t)g.H * g.W, g.heads), 0.f);
}

// Device address of the scratch array, looked up once per device (with that
// device current) the first time the entry point runs on it.
// The lookup runs once per device under a std::once_flag, so host threads
// making their first calls on one device at the same time do not race on the
// cache; a failed lookup leaves nullptr and the call reports PRISM_ERR_CUDA.
static float* noalloc_scratch_ptr(int dev) {
    static std::once_flag once[64];
    static std::atomic<float*> ptrs[64];
    if (dev < 0 || dev >= 64) return nullptr;
    std::call_once(once[dev], [dev] {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) ptrs[dev].store(static_cast<float*>(p));
    });
    return ptrs[dev].load();
}

}  // namespace prism

extern "C" int prism_zone_shapes_noalloc(const prism_params* p, const void* V, const float* a_map,
                                         uint8_t* shape_id, int32_t* nblocks, void* stream) {
    using namespace prism;
    int st = validate_params(p);
    if (st) return st;
    if (p->cut_ratio != 0.f) return PRISM_ERR_INVALID_ARG;   // whole zones only
    if (!V || !shape_id || !nblocks || !aligned16(V) || (a_map && !aligned16(a_map)))
        return PRISM_ERR_INVALID_ARG;
    st = check_device();
    if (st) return st;
    const Geom g = make_geom(p);
    size_t o_abar, o_vhat, o_zstat;
    if (noalloc_floats(g.Nz, g.heads, &o_abar, &o_vhat, &o_zstat) > kNoAllocScratchFloats)
        return PRISM_ERR_SCRATCH_LIMIT;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
    float* base = noalloc_scratch_ptr(dev);
    if (!base) return PRISM_ERR_CUDA;
    DevPlan d{};
    d.T = g.T; d.H = g.H; d.W = g.W; d.heads = g.heads; d.D = g.D; d.Zh = g.Zh; d.Zw = g.Zw;
    d.Nz = g.Nz; d.N = g.N;
    d.araw = reinterpret_cast<double*>(base);
    d.abar = base + o_abar;
    d.vhat = base + o_vhat;
    d.zstat = base + o_zstat;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // every scratch value below is written before it is read: nothing to clear
    if (a_map) {
        k_audio_zone<<<g.Nz, 256, 0, s>>>(d, a_map);
        k_audio_norm<<<1, 1024, 0, s>>>(d);
    } else {
        k_audio_none<<<(g.Nz + 255) / 256, 256, 0, s>>>(d);
    }
    const bool bf = p->dtype == PRISM_BF16;
    if (bf && g.D == 128) noalloc_stats<__nv_bfloat16, 128>(g, d, V, s);
    else if (bf) noalloc_stats<__nv_bfloat16, 64>(g, d, V, s);
    else if (g.D == 128) noalloc_stats<float, 128>(g, d, V, s);
    else noalloc_stats<float, 64>(g, d, V, s);
    k_zone_shapes_static<<<g.heads, 1024, 0, s>>>(d, shape_rule(*p), shape_id, nblocks);
    return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}
