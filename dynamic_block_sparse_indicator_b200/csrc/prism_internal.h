// prism_internal.h -- host-side plan handle and the workspace layout shared by
// the plan, forward and backward translation units of libprism.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/prism.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <vector>

namespace prism {

// Bounds checks of the gather / scatter / list indices, compiled in with
// -DPRISM_CHECKS=1 (the library's checking build): a failed check records
// PRISM_ERR_DEVICE_CHECK in the plan's error word and the caller skips the
// access; no trap.  Off by default (the checks cost registers in hot loops).
#ifndef PRISM_CHECKS
#define PRISM_CHECKS 0
#endif
#if defined(__CUDACC__)
__device__ __forceinline__ bool prism_bad_index(int* err, bool in_bounds) {
    if (PRISM_CHECKS && !in_bounds) {
        atomicCAS(err, 0, PRISM_ERR_DEVICE_CHECK);
        return true;
    }
    return false;
}
#endif

// Per-head input scaling of the fp16 tensor-core copies: Q, K and V of a head
// are multiplied by exact powers of two 2^shift chosen so that the head's
// largest magnitude lies in [2^14, 2^15) (below fp16's maximum 65504), so
// inputs of any finite magnitude keep fp16's relative precision down to 2^-28
// of the head's maximum.  max_bits holds the head's max |x| as float bits; the
// kernels undo the shifts exactly (logit scale, O, dQ, dK, dP).
#if defined(__CUDACC__)
__device__ __forceinline__ int qkv_shift(uint32_t max_bits) {
    const float m = __uint_as_float(max_bits);
    if (!(m > 0.f) || !(m <= 3.402823466e38f)) return 0;    // zero, or not finite (device-checked)
    int e;
    frexpf(m, &e);                                          // m in [2^(e-1), 2^e)
    return 15 - e;
}
#endif

// Where row (h, token n) of a [heads][N][D] tensor lives.  A plain tensor is
// one shard.  A sequence-parallel caller's tensor is `n` token shards, shard s
// holding frames [s F, (s + 1) F) of every one of `stride_heads` heads as
// [stride_heads][F HW][D] (a rank's part of the sequence); a plan covers heads
// head0, head0 + 1, ... of them.  The shard pointers may be other GPUs' memory
// mapped for peer access: the kernels read and write them with plain loads and
// stores, so the exchange between sequence and head layouts happens inside the
// passes the plan and the attention make anyway.
constexpr int kMaxShards = 16;
struct TokenRows {
    void* p[kMaxShards];
    int64_t S;             // tokens per shard (F HW)
    int64_t HW;            // tokens per frame
    int F;                 // frames per shard
    int n;                 // shards
    int stride_heads;      // heads held by each shard
    int head0;             // the shard head of plan head 0
#if defined(__CUDACC__)
    // row (h, token tok of frame t)
    template <typename T>
    __device__ __forceinline__ T* row_t(int h, int t, int64_t tok, int D) const {
        const int sh = n == 1 ? 0 : t / F;
        return static_cast<T*>(p[sh]) + ((int64_t)(head0 + h) * S + (tok - (int64_t)sh * S)) * D;
    }
    template <typename T>
    __device__ __forceinline__ T* row(int h, int64_t tok, int D) const {
        return row_t<T>(h, n == 1 ? 0 : (int)(tok / HW), tok, D);
    }
#endif
};

// One plain [heads][N][D] tensor.
inline TokenRows plain_rows(const void* x, int T, int64_t HW, int heads) {
    TokenRows r{};
    r.p[0] = const_cast<void*>(x);
    r.HW = HW;
    r.F = T;
    r.S = (int64_t)T * HW;
    r.n = 1;
    r.stride_heads = heads;
    r.head0 = 0;
    return r;
}

// `shards` token shards of `heads_total` heads; the plan's head 0 is shard head head0.
inline TokenRows shard_rows(const void* const* xs, int shards, int T, int64_t HW, int heads_total, int head0) {
    TokenRows r{};
    for (int i = 0; i < shards; ++i) r.p[i] = const_cast<void*>(xs[i]);
    r.HW = HW;
    r.F = T / shards;
    r.S = (int64_t)r.F * HW;
    r.n = shards;
    r.stride_heads = heads_total;
    r.head0 = head0;
    return r;
}

// Geometry derived from prism_params.
struct Geom {
    int T, H, W, heads, D, dtype;
    int Zt, Zh, Zw, Nz;   // macro-zones per axis / total
    int64_t N;            // tokens per head
    int NB;               // max blocks per head = N / 64
    int NT;               // 128-token tiles per head = N / 128
    int WORDS;            // 32-bit words per selection-bitmap row = ceil(NB / 32)
    int GH;               // heads per group of the forward-state / gradient scratch
    int SEL_ROWS;         // CTAs of the selection kernel when a block row is staged in global memory (0: shared)
};

// Kinds of index lists (offset tables loff[kind][heads], in ints from the list base).
enum { LIST_CSR = 0, LIST_CSC = 1, LIST_FWD = 2, LIST_BWD = 3, LIST_KINDS = 4 };

// Byte offsets of the workspace regions (each 256-byte aligned).
struct Layout {
    size_t err;                         // int32[4]: error word + detail
    size_t araw;                        // double[Nz]  zone mean of the audio map
    size_t abar, vhat;                  // float[Nz], float[Nz][3]
    size_t zstat;                       // float[heads][Nz][4]
    size_t shape_id;                    // uint8[heads][Nz]   (first part's shape when split)
    size_t zdiff;                       // float[heads][Nz][7] frame-difference energies
    size_t zcut;                        // uint8[heads][Nz]   split frame: 0, 2, 4, 6
    size_t shape_id2;                   // uint8[heads][Nz]   second part's shape (255: none)
    size_t rstat;                       // float[heads][Nz][2][4] statistics of the parts
    size_t araw_seg;                    // double[Nz][3][2]   audio means of the six possible parts
    size_t vhat_seg;                    // float[Nz][3][2][3] their v_hat
    size_t zone_off;                    // int32[heads][Nz + 1]  first block of each zone
    size_t nblocks;                     // int32[heads]
    size_t blk_start;                   // int32[heads][NB + 1]
    size_t t64_blk;                     // int32[heads][NB]      block of each 64-token tile
    size_t src;                         // int32[heads][N]        raster token of each slot
    size_t qbar, kbar;                  // float[heads][NB][D]
    size_t sel, selT;                   // uint32[heads][NB][WORDS]
    size_t row_ptr, col_ptr;            // int32[heads][NB + 1]  CSR / CSC row pointers
    size_t qt_ptr, kt_ptr;              // int32[heads][NT + 1]  forward / backward tile-list pointers
    size_t loff;                        // int64[LIST_KINDS][heads] list offsets (ints from the list base)
    size_t selrow;                      // float[SEL_ROWS][NB + NB/32 + 1]: staged block rows (SEL_ROWS > 0)
    size_t qkv_max;                     // uint32[heads][3]: max |Q|, |K|, |V| bits (the copies' scaling)
    size_t qp, kp, vp;                  // fp16[heads][N][D] block-ordered copies, scaled by 2^shift
    size_t dop;                         // fp16[GH][N][D] block-ordered dO of a head group
    size_t lse_p, di_p;                 // float[heads][N] (backward, block order)
    size_t dmax;                        // uint32[heads]: max |dO| bits (backward scaling)
    size_t dq_acc;                      // float[GH][N][D]: dQ (and the forward's pass state) of a head group
    size_t dk_acc, dv_acc;              // float[GH][N][D]: dK, dV of a head group, block order
    size_t core;                        // bytes up to here: everything but the index lists
    size_t col_idx, row_idx;            // lists inside the workspace (one-call plans):
    size_t qt_ent, kt_ent;              // int32[heads][NB * NB] x 2, int32[heads][NT * NT] x 2
    size_t total;                       // core + the lists at their dense bound
};

Geom make_geom(const prism_params* p);
Layout make_layout(const Geom& g);
int validate_params(const prism_params* p);

}  // namespace prism

struct prism_plan_s {
    prism_params p;
    prism::Geom g;
    prism::Layout L;
    char* ws;                 // device workspace base
    size_t ws_bytes;
    int device;
    int has_audio;
    int has_cuts;             // adaptive temporal boundaries in force (computed or imported)
    char* lists;              // base of the index lists: inside ws (one-call) or the caller's list buffer
    int lists_ready;          // lists built (attention calls need them)
    int64_t list_len[prism::LIST_KINDS];  // ints per kind over all heads (packed lists)
    std::vector<int64_t> loff_host;       // [LIST_KINDS][heads] offsets uploaded to L.loff
    CUtensorMap tm_q, tm_k, tm_v, tm_do;       // 2D [heads*N, D] fp16, 128-row boxes, 128B swizzle
    CUtensorMap tm_q64, tm_k64, tm_v64, tm_do64;  // the same with 64-row boxes
    CUtensorMap tm_dk, tm_dv;                     // fp32 dK, dV accumulators, the same boxes
    // tm_do / tm_do64 cover the head group's dO copy: [GH*N, D]
    int64_t launches;                             // kernels launched so far
    int profile;                                  // per-stage event timing on?
    struct Timed { int stage; cudaEvent_t a, b; };
    std::vector<Timed> timed;                     // pending event pairs
};

// Names of the stages as NVTX ranges (a profiler's timeline shows each launch
// group under the stage that issued it).
inline const char* prism_stage_name(int stage) {
    static const char* names[PRISM_STAGE_COUNT] = {
        "prism fwd", "prism bwd pre", "prism bwd dK dV", "prism bwd dQ", "prism plan stats",
        "prism plan shapes", "prism plan gather", "prism plan select", "prism plan lists"};
    return stage >= 0 && stage < PRISM_STAGE_COUNT ? names[stage] : "prism";
}

// Around one stage's launches: an NVTX range always, and an event pair on the
// stream when profiling is on.
struct PrismProf {
    prism_plan_s* P;
    int stage;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    bool open = true;
    PrismProf(prism_plan_s* P_, int stage_, cudaStream_t s_) : P(P_), stage(stage_), s(s_) {
        nvtxRangePushA(prism_stage_name(stage));
        if (P->profile && cudaEventCreate(&a) == cudaSuccess && cudaEventCreate(&b) == cudaSuccess)
            cudaEventRecord(a, s);
    }
    // ends the range and records the closing event now (idempotent; the destructor calls it)
    void close() {
        if (a && b) {
            cudaEventRecord(b, s);
            P->timed.push_back({stage, a, b});
            a = b = nullptr;
        }
        if (open) {
            nvtxRangePop();
            open = false;
        }
    }
    ~PrismProf() { close(); }
};

// Internal entry points of the attention translation units (O, dO, dQ, dK, dV
// addressed through TokenRows; the LSE is the plan's [heads][N]).
int prism_launch_attn_fwd(prism_plan_s* P, const prism::TokenRows& O, float* lse, void* stream);
int prism_launch_selftest_wait(prism_plan_s* P, void* stream);
int prism_launch_attn_bwd(prism_plan_s* P, const prism::TokenRows& dO, const prism::TokenRows& O, const float* lse,
                          const prism::TokenRows& dQ, const prism::TokenRows& dK, const prism::TokenRows& dV,
                          void* stream);
