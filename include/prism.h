/*
 * prism.h -- C ABI of libprism, a B200 (sm_100a) implementation of Prism's
 * dynamic block-sparse video self-attention.
 *
 * Method: "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
 * Generation Model Training" (arXiv 2610.05416).  The equations are those of
 * the page xyznot.com/id/paper/2610.05416, section "Metode" 1-3; the five
 * stages and the hyperparameters are those of the page
 * paper.rainbus.top/paper/2610.05416, section "方法步骤详情" (Algorithm 1).
 *
 * Call sequence for one layer:
 *   prism_plan()      stage 1 (zone statistics, volume, shape), stage 2 (token
 *                     reorder), stage 3 (block pooling, scores, Top-k U Top-p)
 *   prism_attn_fwd()  stages 4-5 (sparse attention, inverse permutation)
 *   prism_attn_bwd()  gradients through stage 4 only (the plan is detached)
 *
 * Conventions
 *   - Every call is asynchronous on the caller's CUDA stream (passed as
 *     `void*`, i.e. a cudaStream_t; NULL = legacy default stream) and returns
 *     an int status (PRISM_OK or a PRISM_ERR_* code).  No call aborts the
 *     process.  Only prism_get_status() and prism_plan_export() synchronise,
 *     and only the given stream.
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library allocates no device memory.  The caller allocates the plan
 *     workspace (size from prism_plan_workspace_bytes) and keeps it, and the
 *     Q, K, V tensors, alive until prism_plan_destroy().
 *   - Token order: raster n = (t*H + h)*W + w over the latent T x H x W grid.
 *     Q, K, V, O, dO, dQ, dK, dV are [heads][N][head_dim] row-major in that
 *     order; Q, K, V of element type `dtype`, the others of `out_dtype`.
 *     LSE is [heads][N] fp32 (natural log), same order.
 *   - Pointers must be 16-byte aligned.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PRISM_API __attribute__((visibility("default")))
#else
#define PRISM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define PRISM_OK               0
#define PRISM_ERR_INVALID_ARG  1  /* bad grid / head_dim / k,p / null pointer / misaligned */
#define PRISM_ERR_WORKSPACE    2  /* workspace smaller than prism_plan_workspace_bytes() */
#define PRISM_ERR_CUDA         3  /* a CUDA runtime or driver call failed */
#define PRISM_ERR_TIMEOUT      4  /* a bounded device-side wait gave up; kernel returned */
#define PRISM_ERR_DEVICE_CHECK 5  /* a device-side bounds/consistency check failed */
#define PRISM_ERR_UNSUPPORTED  6  /* no sm_100 device, or the build lacks the kernels */
#define PRISM_ERR_SCRATCH_LIMIT 7 /* too large for prism_zone_shapes_noalloc's static scratch */

/* Element types (prism_params.dtype / out_dtype). */
#define PRISM_BF16 0
#define PRISM_F32  1

/*
 * Problem description.
 *   T, H, W   latent grid, each a positive multiple of the macro-zone edge 8
 *             (zones are 8 x 8 x 8: page xyznot.com/id, section "Ide utama").
 *   heads     number of heads in this call (>= 1).
 *   head_dim  D, 64 or 128.
 *   dtype     element type of Q, K, V: PRISM_BF16 or PRISM_F32.  fp32 inputs
 *             feed the statistics and the pooled means in fp32; attention runs
 *             on their fp16 rounding (round to nearest even).
 *   out_dtype element type of O, dO, dQ, dK, dV: PRISM_BF16 or PRISM_F32.
 *             The tensor-core products take fp16 operands with fp32
 *             accumulation either way; fp32 outputs keep the fp32 accumulators
 *             unrounded.  Each head's Q, K, V and dO are multiplied by exact
 *             powers of two before their fp16 conversion (Q, K, V: the head's
 *             largest magnitude into [2^14, 2^15); dO: into [0.5, 1)), and the
 *             kernels undo the factors exactly: any finite input magnitude is
 *             accepted, a bf16 value converts exactly unless it lies below
 *             2^-28 of its head's largest (then it rounds to fp16's subnormal
 *             grid), and a non-finite input makes the plan report
 *             PRISM_ERR_DEVICE_CHECK.
 *   top_k     k of Top-k (>= 0); k >= number of blocks keeps every block.
 *   top_p     p of Top-p in [0, 1]; p >= 1 keeps every block, p <= 0 none.
 *             Empty sets (top_k < 1, top_k_frac <= 0 and top_p <= 0) are
 *             rejected.
 *   eps       epsilon of g_d = r_{v,d} + a_bar * v_hat_{a,d} + eps.
 *   tau128, tau256   density thresholds (the pages use 0.5 and 0.25).
 * Variants of the pages' ablation (page xyznot.com/id, Table 10) and operating
 * point (page paper.rainbus.top: Top-k 95%, Top-p 0.2):
 *   alpha       exponent of the shape mapping b_d ~ g_d^-alpha:
 *               l*_d = -alpha log2 g_d + 1/3 (log2 B + alpha sum_d' log2 g_d').
 *               0 means the pages' 1/2; must be >= 0.
 *   shape_mode  PRISM_SHAPE_DYNAMIC (the method), PRISM_SHAPE_ISOTROPIC (g_d
 *               taken equal on the three axes: the volume still follows rho,
 *               the shape is the candidate nearest the cube, ties to the lower
 *               index) or PRISM_SHAPE_FIXED (every zone takes candidate
 *               fixed_shape, whatever its statistics: the fixed-block
 *               comparator).
 *   fixed_shape candidate index 0..15 for PRISM_SHAPE_FIXED, ignored otherwise.
 *               Candidates are ordered by volume (64, 128, 256), each volume
 *               lexicographically in (b_T, b_H, b_W): 3 = 4x4x4, 8 = 4x4x8,
 *               13 = 4x8x8 (the candidate nearest the cube of each volume).
 *   top_k_frac  k as a fraction of the head's block count: when > 0, each
 *               head's k is ceil(top_k_frac * N_b) in fp32 (the pages' "Top-k
 *               95%" sparsity keeps 5%: 0.05) and top_k is ignored; in [0, 1].
 * Adaptive temporal zone boundaries (page paper.rainbus.top, section
 * "独立分析的弱点" item (1) and section "未来方向": split a macro-zone where a
 * shot cut shows in the frame differences):
 *   cut_ratio   0 keeps every zone whole (the pages' method).  When > 0, per
 *               zone and head the frame-difference energies e_t (mean over the
 *               zone's 64 tokens and D channels of (V[t+1] - V[t])^2, t = 0..6,
 *               fp32) are formed; a cut follows the largest e_t (lowest t on
 *               ties) when it exceeds cut_ratio times their median; the
 *               boundary snaps to the nearest of frames 2, 4, 6 (3 and 5 to 4),
 *               and each part is planned like a zone: its own statistics,
 *               volume capped at what its length tiles (128 for 2 or 6 frames),
 *               shape among the candidates whose b_T divides its length; rho
 *               and a_bar are normalised over the head's zones and parts.  The
 *               first part's blocks come first in the zone.  Must be >= 0 and
 *               finite; not allowed with PRISM_SHAPE_FIXED.  Smooth content
 *               stays below 2 and a shot cut is typically above 3.5: 2.5 is a
 *               reasonable value.
 */
#define PRISM_SHAPE_DYNAMIC   0
#define PRISM_SHAPE_ISOTROPIC 1
#define PRISM_SHAPE_FIXED     2
typedef struct prism_params {
    int32_t T, H, W;
    int32_t heads;
    int32_t head_dim;
    int32_t dtype;
    int32_t out_dtype;
    int32_t top_k;
    float   top_p;
    float   eps;
    float   tau128;
    float   tau256;
    float   alpha;
    int32_t shape_mode;
    int32_t fixed_shape;
    float   top_k_frac;
    float   cut_ratio;
} prism_params;

/* Opaque host-side handle: a small host struct pointing into the workspace. */
typedef struct prism_plan_s* prism_plan_t;

/*
 * Workspace.  The plan's index lists (the CSR key-block lists of S_i, their
 * transpose, and the per-128-token-tile lists the attention kernels walk) are
 * data dependent.  Two ways to hold them:
 *   one call   a workspace of prism_plan_workspace_bytes(p) bytes holds the
 *              lists at their dense bound (N/64 blocks per head, every pair
 *              selected: 2 (N/64)^2 + 2 (N/128)^2 ints per head, 2.5 GB for one
 *              1M-token head); prism_plan() returns a plan ready for attention.
 *   two calls  a workspace of prism_plan_core_bytes(p) bytes (the rest: block-
 *              ordered Q, K, V copies, statistics, bitmaps, and a head group's
 *              forward-state and gradient scratch) makes prism_plan() stop after
 *              counting the lists; prism_plan_list_bytes() then gives their exact
 *              size (it synchronises the stream) and prism_plan_attach_lists()
 *              builds them in a second buffer the caller allocates and keeps
 *              alive with the workspace.  A 40-head 1M-token layer needs about
 *              62 GB this way at the 2K workload's 92% pair density.
 * Both return 0 when `p` is invalid.  Scratch that only the forward and the
 * backward use (the forward's state between key-range passes, the fp32 dQ, dK,
 * dV accumulators, the fp16 dO copy) is sized for a group of heads those calls
 * walk one group after another: heads of at least 2M tokens together, one head
 * at a time for larger heads.
 */
PRISM_API size_t prism_plan_workspace_bytes(const prism_params* p);
PRISM_API size_t prism_plan_core_bytes(const prism_params* p);

/*
 * prism_plan -- stages 1-3 of Algorithm 1 for every head.
 *   Stage 1 (page paper.rainbus.top, section "方法步骤详情"; equations of page
 *   xyznot.com/id, section "Metode" 1-2): per 8x8x8 zone and head, the
 *   directional value variances sigma^2_{v,d} of the mean-pooled V profiles,
 *   r_{v,d}, the audio coupling a_bar and v_hat_{a,d} from a_map, g_d, the
 *   density rho -> volume B in {64,128,256} (thresholds tau256, tau128), the
 *   closed form l*_d = -1/2 log2 g_d + 1/3 (log2 B + 1/2 sum log2 g) snapped to
 *   the nearest of the 16 candidate shapes (alpha and shape_mode select the
 *   ablation variants).
 *   Stage 2: reorder tokens so every block is contiguous (fp16 copies of Q,
 *   K, V in block order, kept in the workspace).
 *   Stage 3 ("Metode" 3): block means Qbar, Kbar; P_i = softmax(Qbar_i Kbar^T
 *   / sqrt(D)); S_i = Top-k(P_i, k) U Top-p(P_i, p) as per-query-block CSR
 *   key-block lists and their transpose.
 * Arguments
 *   Q, K, V    device, [heads][N][head_dim] of `dtype`, raster order.
 *   a_map      device fp32 [T][H][W], the cached audio-to-video cross-attention
 *              output norm of the previous layer, shared by all heads; NULL for
 *              the first layer (then g_d = r_{v,d} + eps).
 *   workspace  device, 256-B aligned: >= prism_plan_workspace_bytes(p) bytes for
 *              a plan ready at once, >= prism_plan_core_bytes(p) to attach the
 *              lists later (prism_plan_attach_lists).
 *   stream     cudaStream_t.
 *   out        receives the plan handle (host memory, freed by
 *              prism_plan_destroy).  Left NULL on error.
 */
PRISM_API int prism_plan(const prism_params* p, const void* Q, const void* K, const void* V,
               const float* a_map, void* workspace, size_t ws_bytes, void* stream,
               prism_plan_t* out);

/*
 * prism_plan_sharded -- prism_plan for inputs held as token shards, the layout
 * a sequence-parallel rank holds (the pages train with sequence parallelism 8:
 * page paper.rainbus.top, section "方法步骤详情").  The plan covers heads
 * head0 .. head0 + p->heads - 1 of the shards' heads_total heads and reads
 * their rows straight from the shards, so the sequence-to-head exchange that
 * would precede a head-sharded plan and the plan's reorder into block order are
 * one pass; everything after the plan (forward, backward, exports) is that of
 * a prism_plan over those heads' [p->heads][N][head_dim] tensors.
 * Arguments
 *   Q, K, V      host arrays of `shards` device pointers.  Shard s holds frames
 *                [s T/shards, (s + 1) T/shards) of every head as
 *                [heads_total][(T/shards) H W][head_dim] of `dtype`, raster
 *                order inside the shard; 16-byte aligned.  A pointer may be
 *                another GPU's memory mapped for peer access (symmetric
 *                memory, an IPC mapping): the kernels read it with plain
 *                loads, never a TMA multicast.
 *   shards       1 .. 16, dividing T.
 *   heads_total  heads held by each shard; head0 + p->heads <= heads_total.
 *   the rest     as prism_plan.
 * Returns PRISM_ERR_INVALID_ARG for a shard count that does not divide T, a
 * head range outside the shards, or a null or misaligned pointer.
 */
PRISM_API int prism_plan_sharded(const prism_params* p, const void* const* Q, const void* const* K,
                                 const void* const* V, int shards, int heads_total, int head0,
                                 const float* a_map, void* workspace, size_t ws_bytes, void* stream,
                                 prism_plan_t* out);

/*
 * prism_plan_import -- the same plan, but with stage 1's shapes and stage 3's
 * selection supplied by the caller instead of computed (a fixed-shape
 * comparator, a cached plan, or a plan computed elsewhere).  Runs stage 2
 * (reorder) and the pooling of stage 3, then builds the CSR lists from `sel`.
 *   shape_id  device uint8 [heads][Nz], values 0..15 (the candidate order: by
 *             volume 64, 128, 256, then lexicographic (b_T, b_H, b_W)).
 *   sel       device uint32 bitmap [heads][N/64][ceil((N/64)/32)]: bit j of
 *             row i set <=> key block j is in S_i; rows and bits beyond the
 *             head's block count are ignored.
 */
PRISM_API int prism_plan_import(const prism_params* p, const void* Q, const void* K, const void* V,
                      const uint8_t* shape_id, const uint32_t* sel,
                      void* workspace, size_t ws_bytes, void* stream, prism_plan_t* out);

/*
 * prism_plan_import_cuts -- prism_plan_import for plans with adaptive temporal
 * boundaries: zone_cut (device uint8 [heads][Nz], 0, 2, 4 or 6) gives each
 * zone's split frame and shape_id2 (device uint8 [heads][Nz]) the shape of the
 * part after it; shape_id then holds the first part's shape.  A shape whose
 * b_T does not divide its part's length, or a volume its part cannot tile, is
 * reported as PRISM_ERR_DEVICE_CHECK by prism_get_status.  NULL zone_cut (and
 * shape_id2) is prism_plan_import.
 */
PRISM_API int prism_plan_import_cuts(const prism_params* p, const void* Q, const void* K, const void* V,
                                     const uint8_t* shape_id, const uint8_t* zone_cut,
                                     const uint8_t* shape_id2, const uint32_t* sel, void* workspace,
                                     size_t ws_bytes, void* stream, prism_plan_t* out);

/*
 * prism_plan_import_sharded -- prism_plan_import_cuts for inputs held as token
 * shards (the layout and the head range of prism_plan_sharded): the given
 * shapes, splits (zone_cut and shape_id2 both NULL without adaptive temporal
 * boundaries) and selection, with the reorder reading every shard's rows.
 */
PRISM_API int prism_plan_import_sharded(const prism_params* p, const void* const* Q, const void* const* K,
                                        const void* const* V, int shards, int heads_total, int head0,
                                        const uint8_t* shape_id, const uint8_t* zone_cut,
                                        const uint8_t* shape_id2, const uint32_t* sel, void* workspace,
                                        size_t ws_bytes, void* stream, prism_plan_t* out);

/*
 * prism_plan_list_bytes -- for a plan made with a core-only workspace: the
 *   bytes its index lists need (0 once they are built).  Synchronises `stream`
 *   (reads each head's list lengths).
 * prism_plan_attach_lists -- builds the lists in `lists` (device, 16-byte
 *   aligned, >= prism_plan_list_bytes bytes, kept alive by the caller as long
 *   as the plan); asynchronous on `stream`.  prism_attn_fwd / prism_attn_bwd
 *   return PRISM_ERR_INVALID_ARG for a plan whose lists are not built;
 *   PRISM_ERR_WORKSPACE if `bytes` is too small.
 */
PRISM_API int prism_plan_list_bytes(prism_plan_t plan, size_t* bytes, void* stream);
PRISM_API int prism_plan_attach_lists(prism_plan_t plan, void* lists, size_t bytes, void* stream);

/*
 * prism_attn_fwd -- stages 4-5: for every query token q of block i,
 *   O_q = softmax_n(q . k_n / sqrt(D)) v_n over the tokens n of the key
 *   blocks in S_i (fp32 online softmax, fp16 tensor-core products with fp32
 *   accumulation), written back in raster order (inverse permutation).
 *   O    device [heads][N][head_dim] of `out_dtype`.
 *   lse  device fp32 [heads][N], log-sum-exp of the scaled logits, raster order.
 */
PRISM_API int prism_attn_fwd(prism_plan_t plan, void* O, float* lse, void* stream);

/*
 * prism_attn_bwd -- exact gradients of prism_attn_fwd with the plan fixed (the
 *   statistics, shapes and selection are detached: page xyznot.com/th, section
 *   on training).  dO, O, lse as produced/consumed by prism_attn_fwd.
 *   dO, dQ, dK, dV device [heads][N][head_dim] of `out_dtype`, raster order.
 */
PRISM_API int prism_attn_bwd(prism_plan_t plan, const void* dO, const void* O, const float* lse,
                   void* dQ, void* dK, void* dV, void* stream);

/*
 * prism_attn_fwd_sharded / prism_attn_bwd_sharded -- prism_attn_fwd and
 * prism_attn_bwd with O, dO, dQ, dK, dV held as token shards in the layout of
 * prism_plan_sharded (host arrays of `shards` device pointers, shard s holding
 * frames [s T/shards, (s + 1) T/shards) of `heads_total` heads as
 * [heads_total][(T/shards) H W][head_dim] of `out_dtype`; the plan's heads are
 * head0 .. head0 + heads - 1 there).  The rows of the plan's heads are written
 * (and O, dO read) in place, so a sequence-parallel rank needs no all-to-all
 * after the forward or around the backward: with peer-mapped shards the
 * kernels store and load other GPUs' rows with plain stores and loads.  The
 * LSE stays [heads][N] fp32 on this device.  Returns PRISM_ERR_INVALID_ARG for
 * a shard count that does not divide T, a head range outside the shards, or a
 * null or misaligned pointer.
 */
PRISM_API int prism_attn_fwd_sharded(prism_plan_t plan, void* const* O, int shards, int heads_total, int head0,
                                     float* lse, void* stream);
PRISM_API int prism_attn_bwd_sharded(prism_plan_t plan, const void* const* dO, const void* const* O,
                                     const float* lse, void* const* dQ, void* const* dK, void* const* dV,
                                     int shards, int heads_total, int head0, void* stream);

/*
 * prism_zone_shapes_noalloc -- stage 1 alone (zone statistics, block volume,
 *   snapped shape) for callers that cannot allocate device memory: a plugin
 *   that may only use the buffers another engine's memory plan hands it, a
 *   latency-critical path where cudaMalloc's implicit device synchronisation
 *   is not acceptable, or a deployment whose device memory is budgeted up
 *   front.  The paper has no counterpart: it is a packaging of prism_plan's
 *   first stage, computing the same shape ids and block counts.
 *   Inputs as for prism_plan (V device [heads][N][head_dim] of `dtype`; a_map
 *   device fp32 [T][H][W] or NULL).  Outputs (device, caller-allocated):
 *     shape_id  uint8 [heads][Nz], the candidate index per zone and head;
 *     nblocks   int32 [heads], blocks of the head (sum over zones of 512 / B).
 *   Whole zones only: p->cut_ratio must be 0 (PRISM_ERR_INVALID_ARG otherwise).
 *   Scratch: a file-scope static device array of 4 MiB (2^20 floats) that
 *   every GPU loading the library holds until the process exits.  Its use is
 *   2*Nz + Nz + 3*Nz + 4*heads*Nz floats (each part rounded up to 64 floats);
 *   larger problems return PRISM_ERR_SCRATCH_LIMIT (the 2K layer, Nz = 1,980,
 *   fits up to 130 heads).  No allocation of any kind is made.
 *   The first call on a device looks the array's device address up (one
 *   cudaGetSymbolAddress with that device current); make that first call
 *   before any stream capture.  Every call shares the one array and leaves its
 *   contents behind; each value is written before it is read, so nothing needs
 *   clearing, but calls whose kernels overlap on the GPU (other streams, other
 *   host threads) race on it and must be serialised by the caller.
 */
PRISM_API int prism_zone_shapes_noalloc(const prism_params* p, const void* V, const float* a_map,
                                        uint8_t* shape_id, int32_t* nblocks, void* stream);

/* ---- guidance map producer ---------------------------------------------- */
/*
 * prism_av_norm -- the audio-to-video cross-attention output norm that the
 *   next layer's prism_plan() reads as a_map (page paper.rainbus.top, section
 *   "前置知识", the dual-branch DiT paragraph: h_hat = CrossAttn(h, K_a, V_a)
 *   and its L2 norm per video position; page xyznot.com/id, section "Metode"
 *   1: a_{t,h,w} = ||h_hat_{t,h,w}||_2, cached from the previous layer):
 *     h_hat[head][n] = softmax_m(Qv[head][n] . Ka[head][m] / sqrt(D)) Va[head][m]
 *     a_map[n]       = sqrt(sum over heads and channels of h_hat[head][n][c]^2)
 *   i.e. the norm of the heads' concatenated outputs before the output
 *   projection (which belongs to the backbone's weights).  One launch covers
 *   every head; the map is written once per token (no atomics).
 * Arguments
 *   N          video tokens (T*H*W of the map, raster order), 1 .. 2^31 - 128.
 *   M          audio tokens, 1 .. 2^20 (the pages' audio is under 1K tokens).
 *   heads      1 .. 4096;  head_dim 64 or 128.
 *   Qv         device bf16 [heads][N][head_dim]: the video tokens' queries.
 *   Ka, Va     device bf16 [heads][M][head_dim]: the audio tokens' keys, values.
 *   a_map      device fp32 [N] (output): the map, ready for prism_plan.
 *   h_hat      device [heads][N][head_dim] of hhat_dtype (output), or NULL to
 *              produce the map alone.
 *   hhat_dtype PRISM_BF16 or PRISM_F32.
 *   dev_status device int32[4], zero before the call: a bounded device wait
 *              that gives up records PRISM_ERR_TIMEOUT and its site there
 *              (read and cleared by prism_status_read).
 * Tensor-core products take the bf16 inputs as they are and a bf16 P, with
 * fp32 accumulation and an fp32 online softmax.  All pointers 16-byte aligned.
 * Returns PRISM_ERR_INVALID_ARG for sizes or pointers outside the above,
 * PRISM_ERR_UNSUPPORTED without an sm_100 device, PRISM_ERR_CUDA if the launch
 * fails; asynchronous on `stream` otherwise.
 */
PRISM_API int prism_av_norm(int64_t N, int32_t M, int32_t heads, int32_t head_dim, const void* Qv,
                            const void* Ka, const void* Va, float* a_map, void* h_hat,
                            int32_t hhat_dtype, int32_t* dev_status, void* stream);

/* Synchronises `stream`, reads a device status block (int32[4], as passed to
 * prism_av_norm), clears it, and returns its status (PRISM_OK or
 * PRISM_ERR_TIMEOUT; PRISM_ERR_CUDA if the copy fails).  *site (if not NULL)
 * receives the site of a timed-out wait. */
PRISM_API int prism_status_read(int32_t* dev_status, int32_t* site, void* stream);

/* ---- inspection -------------------------------------------------------- */
#define PRISM_ITEM_SHAPE_ID   0  /* uint8  [heads][Nz]                         */
#define PRISM_ITEM_NBLOCKS    1  /* int32  [heads]                             */
#define PRISM_ITEM_BLK_START  2  /* int32  [heads][N/64 + 1] (first nblocks+1)  */
#define PRISM_ITEM_SEL_BITS   3  /* uint32 [heads][N/64][ceil(N/64 / 32)]       */
#define PRISM_ITEM_ROW_PTR    4  /* int32  [heads][N/64 + 1]  CSR              */
#define PRISM_ITEM_COL_IDX    5  /* int32  CSR key blocks: row i of head h at LIST_OFFSETS[0][h] + row_ptr[h][i] */
#define PRISM_ITEM_COL_PTR    6  /* int32  [heads][N/64 + 1]  CSC              */
#define PRISM_ITEM_ROW_IDX    7  /* int32  CSC query blocks: column j of head h at LIST_OFFSETS[1][h] + col_ptr[h][j] */
#define PRISM_ITEM_QBAR       8  /* fp32   [heads][N/64][head_dim]             */
#define PRISM_ITEM_KBAR       9  /* fp32   [heads][N/64][head_dim]             */
#define PRISM_ITEM_SRC       10  /* int32  [heads][N] raster token of each permuted slot */
#define PRISM_ITEM_ZONE_STATS 11 /* fp32   [heads][Nz][4] sigma2_T, sigma2_H, sigma2_W, rho_raw */
#define PRISM_ITEM_ZONE_CUT  12  /* uint8  [heads][Nz] split frame (0 = whole zone, 2, 4 or 6) */
#define PRISM_ITEM_SHAPE_ID2 13  /* uint8  [heads][Nz] shape of the part after the split (255 if none) */
#define PRISM_ITEM_ZONE_ENERGY 14 /* fp32  [heads][Nz][7] frame-difference energies e_t */
#define PRISM_ITEM_REGION_STATS 15 /* fp32 [heads][Nz][2][4] the parts' statistics (split zones) */
#define PRISM_ITEM_LIST_OFFSETS 16 /* int64 [4][heads]: head h's first entry in the CSR, CSC,
                                      forward and backward tile lists */
#define PRISM_ITEM_QKV_MAX   17  /* uint32 [heads][3]: fp32 bits of max |Q|, |K|, |V| of each head,
                                      which set the copies' power-of-two scales */
#define PRISM_ITEM_COUNT     18

/* Bytes of an item (0 for an unknown item). */
PRISM_API size_t prism_plan_item_bytes(prism_plan_t plan, int item);

/* Synchronises `stream` and copies an item into host memory (bytes must equal
 * prism_plan_item_bytes). */
PRISM_API int prism_plan_export(prism_plan_t plan, int item, void* host_dst, size_t bytes, void* stream);

/* Synchronises `stream`, then reads and clears the plan's device error word:
 * PRISM_OK, PRISM_ERR_TIMEOUT or PRISM_ERR_DEVICE_CHECK (or PRISM_ERR_CUDA). */
PRISM_API int prism_get_status(prism_plan_t plan, void* stream);

/* As prism_get_status, and writes the site of a timed-out wait (an id of the
 * kernel role and barrier, 0 if none) into *site when site is not NULL. */
PRISM_API int prism_get_status_ex(prism_plan_t plan, int32_t* site, void* stream);

/* Failure-detection self-test: launches one thread that waits on a barrier
 * nothing ever arrives at.  The bounded device wait gives up after about a
 * second, records PRISM_ERR_TIMEOUT (site 9001) in the plan's error word and
 * the kernel returns; the next prism_get_status reports it.  No fault and no
 * hang: the context stays usable. */
PRISM_API int prism_selftest_timeout(prism_plan_t plan, void* stream);

/* Frees the host handle (the workspace stays the caller's). */
PRISM_API void prism_plan_destroy(prism_plan_t plan);

/* Static description of a status code. */
PRISM_API const char* prism_status_string(int status);

/* ---- profiling ---------------------------------------------------------- */
/* Per-kernel CUDA-event timing of the attention launches (events recorded on
 * the caller's stream around each launch). */
#define PRISM_STAGE_FWD       0  /* k_attn_fwd                         */
#define PRISM_STAGE_BWD_PRE   1  /* dO scaling, D_i, block-order dO     */
#define PRISM_STAGE_BWD_DKDV  2  /* dK, dV per key tile                 */
#define PRISM_STAGE_BWD_DQ    3  /* dQ per query tile                   */
/* Plan stages, timed only for plans created while prism_profile_plans(1) is
 * in force (the plan is built inside prism_plan, before a handle exists). */
#define PRISM_STAGE_PLAN_STATS  4  /* audio terms + zone statistics of V    */
#define PRISM_STAGE_PLAN_SHAPES 5  /* finalize: g_d, B, l*, snapped shapes  */
#define PRISM_STAGE_PLAN_GATHER 6  /* block-order fp16 Q, K, V + pooled means */
#define PRISM_STAGE_PLAN_SELECT 7  /* block scores, Top-k u Top-p selection  */
#define PRISM_STAGE_PLAN_LISTS  8  /* CSR, CSC and the per-tile lists        */
#define PRISM_STAGE_COUNT       9

/* Turns per-stage timing on (1) or off (0) for later calls on this plan. */
PRISM_API int prism_profile_enable(prism_plan_t plan, int on);

/* Process-wide switch: plans created after prism_profile_plans(1) start with
 * timing on and record their own plan kernels under PRISM_STAGE_PLAN_*
 * (read back with prism_profile_read).  Returns the previous setting.  Not
 * synchronised with concurrent prism_plan calls on other host threads. */
PRISM_API int prism_profile_plans(int on);

/* Synchronises `stream`, writes the milliseconds spent per stage (and the
 * number of launches per stage into `launches`, may be NULL) since the last
 * read, and resets the accumulators.  ms has PRISM_STAGE_COUNT entries. */
PRISM_API int prism_profile_read(prism_plan_t plan, float* ms, int* launches, void* stream);

/* Number of kernels this plan has launched (plan, forward and backward). */
PRISM_API int64_t prism_launch_count(prism_plan_t plan);

/* Library version, e.g. "prism-b200 0.1 sm_100a". */
PRISM_API const char* prism_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PRISM_H */
