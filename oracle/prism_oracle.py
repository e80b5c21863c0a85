"""CPU oracle of Prism's dynamic sparse video self-attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the library never does.
It shares no code with the CUDA path.

Source: "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
Generation Model Training" (arXiv 2610.05416), as printed on the pages
xyznot.com/id/paper/2610.05416 (section "Metode" 1-3, the clean equations) and
paper.rainbus.top/paper/2610.05416 (section "方法步骤详情": Algorithm 1's
five stages and the hyperparameters).  Each function names the step it follows.

Precision.  Statistics, pooled means, logits and attention are accumulated in
float64.  Every quantity that decides an integer (the block volume B, the
snapped shape, the selected block set) is taken in float32, the precision of
the CUDA path: r, v_hat, a_bar and rho are rounded to float32 after their
float64 normalisation, and g, log2 g, l*, the snap distances, the softmax
probabilities and the Top-p prefix sums are float32 arithmetic.

Readings where the pages are silent (listed with their reasons in the design
notes of the repository):
  * "mean-pooled along axis d" = average over the plane orthogonal to d, giving
    the Z_d-long profile that the variance formula indexes by i;
  * r = (1/3, 1/3, 1/3) when the three directional variances sum to zero;
  * audio coupling a_bar(m) = zone mean of a, divided by its maximum over the
    zones (0 when that maximum is 0); v_hat_{a,d} = directional variance of
    the zone's slice means of a, divided by the sum over the three axes (0 when
    that sum is 0); a missing map (first layer) means a_bar = 0;
  * information density rho(m) = channel mean of [mean over frames of the
    spatial variance within the frame + variance of the frame differences],
    divided by its maximum over the zones of the head (0 when that max is 0);
    B = 256 if rho < tau256, else 128 if rho < tau128, else 64;
  * the candidate set C_B lists (b_T, b_H, b_W) in ascending lexicographic
    order; snapping takes the least squared log2 distance, ties to the lower
    index;
  * blocks tile the zone in raster order of block coordinates, tokens inside a
    block in raster (t, h, w) order; permuted position = 512 m + block * B +
    token;
  * selection: logits Qbar_i . Kbar_j / sqrt(D), softmax over all key blocks,
    order (P descending, j ascending); Top-p keeps the shortest prefix whose
    float32 running sum reaches p (p >= 1 keeps all, p <= 0 none); the union
    with Top-k of the same order is the first max(k, L) blocks;
  * adaptive temporal boundaries (optional): see zone_shapes_cut.

Parity status: the candidate set, the closed form l*, the snapping, the
directional statistics, the selection rule and the attention (forward and
backward) are pinned by the tests in tests/test_oracle_pins.py; the block-score
softmax (hand-worked values, torch float64), the tie margins (written-out
candidate distances, constructed threshold ties) and closed forms of the
statistics on hand-built fields by tests/test_oracle_selection_pins.py, with
planted mistakes that each of those checks catches; the adaptive temporal
boundaries by tests/test_oracle_cuts.py (closed-form energies, hard cuts at
every frame, per-token brute force on the parts, the partition's invariants);
the order of tokens inside a block by invariance (no result depends on it).
The rho formula, the a_bar / v_hat normalisations and the cut detector are
readings: their code is pinned to closed forms and to a per-token brute force,
the readings themselves are not fixed by the pages ("parity unpinned" for the
reading).
"""
from __future__ import annotations

import numpy as np

Z = 8  # macro-zone edge Z_T = Z_H = Z_W (section "Ide utama")
F32 = np.float32


# ---------------------------------------------------------------------------
# Candidate shapes (section "Metode" 2: edges from {2, 4, 8}, product B,
# 16 shapes over B in {64, 128, 256}).
# ---------------------------------------------------------------------------
def candidate_shapes():
    """All (b_T, b_H, b_W) with edges in {2,4,8} and volume 64, 128 or 256.

    Listed by volume, then lexicographically; the list index is the shape id.
    """
    out = []
    for vol in (64, 128, 256):
        for bt in (2, 4, 8):
            for bh in (2, 4, 8):
                for bw in (2, 4, 8):
                    if bt * bh * bw == vol:
                        out.append((bt, bh, bw))
    return out


SHAPES = candidate_shapes()


def shapes_of_volume(vol, L=Z):
    """Candidates of volume vol whose time edge b_T divides a region of L frames
    (every candidate for a whole 8-frame zone)."""
    return [(i, s) for i, s in enumerate(SHAPES) if s[0] * s[1] * s[2] == vol and L % s[0] == 0]


def max_volume(L):
    """Largest candidate volume that tiles a region of L frames (256 for 8 and 4
    frames, 128 for 2 and 6: those take b_T = 2 only)."""
    return max(s[0] * s[1] * s[2] for s in SHAPES if L % s[0] == 0)


# ---------------------------------------------------------------------------
# Stage 1: zone statistics ("Metode" 1; Algorithm 1 stage one)
# ---------------------------------------------------------------------------
def zones_of(X, T, H, W):
    """Raster [N, C] -> [Nz, 8(t), 8(h), 8(w), C], zones in raster (zt, zh, zw) order."""
    C = X.shape[-1]
    Y = X.reshape(T // Z, Z, H // Z, Z, W // Z, Z, C).transpose(0, 2, 4, 1, 3, 5, 6)
    return Y.reshape(-1, Z, Z, Z, C)


def directional_variance(Vz):
    """sigma^2_{v,d}(m) for d = T, H, W: [Nz, 3] float64.

    Profile along d: the mean of V over the plane orthogonal to d (one value
    per slice i = 1..Z_d and channel c); variance of the profile over i around
    its mean mu^{(d)}_{m,c}; average over the D channels.
    """
    Vz = np.asarray(Vz, dtype=np.float64)
    sig = np.empty((Vz.shape[0], 3))
    for d, plane in enumerate(((2, 3), (1, 3), (1, 2))):
        prof = Vz.mean(axis=plane)                      # [Nz, 8, D]
        mu = prof.mean(axis=1, keepdims=True)           # [Nz, 1, D]
        sig[:, d] = ((prof - mu) ** 2).mean(axis=1).mean(axis=-1)
    return sig


def ratio(sig):
    """r_{v,d} = sigma^2_d / sum_d' sigma^2_d'; (1/3,1/3,1/3) where the sum is 0."""
    tot = sig.sum(axis=1, keepdims=True)
    r = np.full_like(sig, 1.0 / 3.0)
    nz = tot[:, 0] > 0
    r[nz] = sig[nz] / tot[nz]
    return r


def audio_terms(a, T, H, W):
    """(a_bar [Nz], v_hat [Nz, 3]) from the cached A->V norm map a [T, H, W].

    The map is a float32 tensor; its values are taken as float32 and then
    summed in float64, so a constant map gives exactly zero variance.
    """
    a = np.asarray(a, dtype=np.float32).astype(np.float64)
    az = zones_of(a.reshape(-1, 1), T, H, W)[..., 0]
    mean = az.mean(axis=(1, 2, 3))                      # zone mean of a
    sig = np.empty((az.shape[0], 3))
    for d, plane in enumerate(((2, 3), (1, 3), (1, 2))):
        prof = az.mean(axis=plane)                      # [Nz, 8]
        sig[:, d] = ((prof - mean[:, None]) ** 2).mean(axis=1)
    tot = sig.sum(axis=1, keepdims=True)
    vhat = np.zeros_like(sig)
    nz = tot[:, 0] > 0
    vhat[nz] = sig[nz] / tot[nz]
    mx = mean.max()
    abar = mean / mx if mx > 0 else np.zeros_like(mean)
    return abar, vhat


def density_raw(Vz):
    """Unnormalised information density per zone: [Nz] float64.

    Channel mean of (mean over the 8 frames of the variance over the frame's
    8x8 tokens) + (variance over all 7x8x8 frame differences V[t+1]-V[t]).
    """
    Vz = np.asarray(Vz, dtype=np.float64)
    spatial = Vz.var(axis=(2, 3)).mean(axis=1)          # [Nz, D]
    diff = Vz[:, 1:] - Vz[:, :-1]                       # [Nz, 7, 8, 8, D]
    temporal = diff.var(axis=(1, 2, 3))                 # [Nz, D]
    return (spatial + temporal).mean(axis=-1)


def normalise_by_max(x):
    mx = x.max()
    return x / mx if mx > 0 else np.zeros_like(x)


# ---------------------------------------------------------------------------
# Stage 1 (cont.): volume quantisation and shape snapping ("Metode" 2)
# ---------------------------------------------------------------------------
def volume(rho32, tau128, tau256):
    """B(m) from the float32 density: 256 below tau256, 128 below tau128, else 64."""
    t128, t256 = F32(tau128), F32(tau256)
    return np.where(rho32 < t256, 256, np.where(rho32 < t128, 128, 64)).astype(np.int64)


def ideal_log_edges(g32, vol, alpha=0.5):
    """l*_d = -alpha log2 g_d + 1/3 (S + alpha sum_d' log2 g_d'), S = log2 B (float32).

    The pages' closed form is alpha = 1/2 ("Metode" 2); Table 10's ablation
    varies the exponent of b_d ~ g_d^-alpha, and the product stays B.
    """
    lg = np.log2(g32.astype(F32))
    S = np.log2(np.asarray(vol, dtype=F32))
    a = F32(alpha)
    inner = S + a * lg[..., 0] + a * lg[..., 1] + a * lg[..., 2]
    return (-a * lg + (inner / F32(3.0))[..., None]).astype(F32)


def snap(ell32, vol, L=Z):
    """Shape id of the candidate of volume vol nearest (squared log2 distance) to l*
    (among those that tile a region of L frames)."""
    best, best_d = -1, None
    for sid, s in shapes_of_volume(int(vol), L):
        e = np.log2(np.asarray(s, dtype=F32))
        d = (e - ell32).astype(F32)
        dist = F32(d[0] * d[0]) + F32(d[1] * d[1])
        dist = F32(dist + F32(d[2] * d[2]))
        if best_d is None or dist < best_d:
            best, best_d = sid, dist
    return best


def snap_margin(ell64, vol, L=Z):
    """Float64 gap between the two smallest snap distances (tie margin)."""
    ds = sorted(float(np.sum((np.log2(np.asarray(s, float)) - ell64) ** 2))
                for _, s in shapes_of_volume(int(vol), L))
    return ds[1] - ds[0] if len(ds) > 1 else np.inf


def rho_margin_of(rho64, tau128, tau256):
    """Float64 distance of the density to the nearer volume threshold (tie margin)."""
    rho64 = np.asarray(rho64, dtype=np.float64)
    return np.minimum(np.abs(rho64 - tau128), np.abs(rho64 - tau256))


SHAPE_DYNAMIC, SHAPE_ISOTROPIC, SHAPE_FIXED = 0, 1, 2


def zone_shapes(V, a, T, H, W, eps, tau128=0.5, tau256=0.25, alpha=0.5, shape_mode=SHAPE_DYNAMIC,
                fixed_shape=0, cut_ratio=0.0):
    """Stage one for one head: V [N, D] raster, a [T,H,W] or None.

    Returns dict with shape_id [Nz], B [Nz], g [Nz,3] (float32), rho [Nz]
    (float32) and the float64 decision margins rho_margin, snap_margin.
    Variants (Table 10's ablation): alpha is the mapping exponent; the
    isotropic mode takes g_d equal on the three axes (B still from rho); the
    fixed mode gives every zone candidate fixed_shape.  cut_ratio > 0 turns on
    the adaptive temporal boundaries (zone_shapes_cut); 0 keeps every zone whole.
    """
    Vz = zones_of(np.asarray(V, dtype=np.float64), T, H, W)
    if cut_ratio > 0:
        return zone_shapes_cut(Vz, a, T, H, W, eps, tau128, tau256, alpha, shape_mode, cut_ratio)
    r = ratio(directional_variance(Vz))
    if a is None:
        abar = np.zeros(Vz.shape[0])
        vhat = np.zeros((Vz.shape[0], 3))
    else:
        abar, vhat = audio_terms(a, T, H, W)
    g32 = (r.astype(F32) + abar.astype(F32)[:, None] * vhat.astype(F32) + F32(eps)).astype(F32)
    g64 = r + abar[:, None] * vhat + eps
    if shape_mode == SHAPE_ISOTROPIC:
        g32 = np.ones_like(g32)
        g64 = np.ones_like(g64)
    rho64 = normalise_by_max(density_raw(Vz))
    rho32 = rho64.astype(F32)
    B = volume(rho32, tau128, tau256)
    ell = ideal_log_edges(g32, B.astype(F32), alpha)
    sid = np.array([snap(ell[m], B[m]) for m in range(len(B))], dtype=np.int64)
    lg = np.log2(g64)
    ell64 = -alpha * lg + (np.log2(B) + alpha * lg.sum(axis=1))[:, None] / 3.0
    rho_margin = rho_margin_of(rho64, tau128, tau256)
    smargin = np.array([snap_margin(ell64[m], B[m]) for m in range(len(B))])
    if shape_mode == SHAPE_ISOTROPIC:
        smargin = np.full(len(B), np.inf)      # the tie rule decides exactly
    if shape_mode == SHAPE_FIXED:
        sid = np.full(len(B), int(fixed_shape), dtype=np.int64)
        B = np.full(len(B), int(np.prod(SHAPES[int(fixed_shape)])), dtype=np.int64)
        rho_margin = np.full(len(B), np.inf)
        smargin = np.full(len(B), np.inf)
    nz = len(B)
    return dict(shape_id=sid, B=B, g=g32, rho=rho32, r=r, abar=abar, vhat=vhat,
                ell=ell, rho_margin=rho_margin, snap_margin=smargin,
                cut=np.zeros(nz, np.int64), shape_id2=np.full(nz, -1, np.int64), cut_margin=np.full(nz, np.inf))


# ---------------------------------------------------------------------------
# Adaptive temporal zone boundaries.  Page paper.rainbus.top, section
# "独立分析的弱点" item (1) and section "未来方向" (the authors' first
# direction): a macro-zone with a fixed 8-frame window that spans a shot cut or
# a fast zoom mixes unrelated content under one block shape; detect the cut from
# frame differences and split the zone there (page xyznot.com/th, limitations,
# names the same failure mode).  Reading (the pages give no formula):
#   * per zone and head, the frame-difference energy e_t = mean over the zone's
#     64 tokens and D channels of (V[t+1] - V[t])^2, t = 0..6;
#   * a cut follows the largest e_t* (lowest t on ties) when e_t* exceeds
#     cut_ratio times the median of the seven energies (float32 decision);
#   * the boundary t* + 1 snaps to the nearest of {2, 4, 6} (3 and 5 to 4): the
#     time edges of the candidate blocks are 2, 4 or 8, so a part must hold an
#     even number of frames;
#   * each part (frames [0, c) and [c, 8)) is a region planned like a zone:
#     its own directional variances (the T profile has the part's length),
#     density (its frames and frame differences) and audio terms; rho and a_bar
#     are normalised by their maxima over the head's regions; the volume is
#     capped at the largest that tiles the part (128 for 2 or 6 frames) and the
#     shape is the nearest candidate whose b_T divides the part's length.
# ---------------------------------------------------------------------------
CUT_SNAP = {1: 2, 2: 2, 3: 4, 4: 4, 5: 4, 6: 6, 7: 6}


def frame_diff_energy(Vz):
    """e_t = mean over the zone's 64 tokens and D channels of (V[t+1] - V[t])^2: [Nz, 7] float64."""
    Vz = np.asarray(Vz, dtype=np.float64)
    d = Vz[:, 1:] - Vz[:, :-1]
    return (d * d).mean(axis=(2, 3, 4))


def zone_cuts(e, cut_ratio):
    """Split position per zone (0 = whole zone, else 2, 4 or 6) and a relative
    float64 margin of the decision (distance of e_t* to the threshold and to
    the runner-up energy; infinite for a zone without frame changes)."""
    e = np.asarray(e, dtype=np.float64)
    e32 = e.astype(F32)
    cut = np.zeros(e.shape[0], np.int64)
    margin = np.full(e.shape[0], np.inf)
    for m in range(e.shape[0]):
        t = int(np.argmax(e32[m]))
        med = np.sort(e32[m])[3]
        if e32[m, t] > F32(F32(cut_ratio) * med):
            cut[m] = CUT_SNAP[t + 1]
        srt = np.sort(e[m])
        if srt[-1] > 0:
            margin[m] = min(abs(srt[-1] - cut_ratio * srt[3]), srt[-1] - srt[-2]) / srt[-1]
    return cut, margin


def zone_regions(cut):
    """[(zone, t0, t1)] in zone order, parts in time order."""
    out = []
    for m, c in enumerate(cut):
        out += [(m, 0, Z)] if c == 0 else [(m, 0, int(c)), (m, int(c), Z)]
    return out


def region_audio(az, regions):
    """Audio terms of each region: zone-style mean and directional slice variances."""
    araw, vhat = np.empty(len(regions)), np.zeros((len(regions), 3))
    for k, (m, t0, t1) in enumerate(regions):
        x = az[m, t0:t1]                                        # [L, 8, 8]
        mean = x.mean()
        sig = np.array([((x.mean(axis=p) - mean) ** 2).mean() for p in ((1, 2), (0, 2), (0, 1))])
        araw[k] = mean
        if sig.sum() > 0:
            vhat[k] = sig / sig.sum()
    return araw, vhat


def zone_shapes_cut(Vz, a, T, H, W, eps, tau128, tau256, alpha, shape_mode, cut_ratio):
    """Stage one with adaptive temporal boundaries (see the reading above)."""
    e = frame_diff_energy(Vz)
    cut, cut_margin = zone_cuts(e, cut_ratio)
    regions = zone_regions(cut)
    sig = np.stack([directional_variance(Vz[m:m + 1, t0:t1])[0] for m, t0, t1 in regions])
    rraw = np.array([density_raw(Vz[m:m + 1, t0:t1])[0] for m, t0, t1 in regions])
    r = ratio(sig)
    if a is None:
        abar, vhat = np.zeros(len(regions)), np.zeros((len(regions), 3))
    else:
        a64 = np.asarray(a, dtype=np.float32).astype(np.float64)
        araw, vhat = region_audio(zones_of(a64.reshape(-1, 1), T, H, W)[..., 0], regions)
        abar = normalise_by_max(araw)
    g32 = (r.astype(F32) + abar.astype(F32)[:, None] * vhat.astype(F32) + F32(eps)).astype(F32)
    g64 = r + abar[:, None] * vhat + eps
    if shape_mode == SHAPE_ISOTROPIC:
        g32, g64 = np.ones_like(g32), np.ones_like(g64)
    rho64 = normalise_by_max(rraw)
    rho32 = rho64.astype(F32)
    L = np.array([t1 - t0 for _, t0, t1 in regions])
    B = np.minimum(volume(rho32, tau128, tau256), [max_volume(x) for x in L])
    ell = ideal_log_edges(g32, B.astype(F32), alpha)
    rsid = np.array([snap(ell[k], B[k], L[k]) for k in range(len(regions))], dtype=np.int64)
    lg = np.log2(g64)
    ell64 = -alpha * lg + (np.log2(B) + alpha * lg.sum(axis=1))[:, None] / 3.0
    rmargin = rho_margin_of(rho64, tau128, tau256)
    smargin = np.array([snap_margin(ell64[k], B[k], L[k]) for k in range(len(regions))])
    if shape_mode == SHAPE_ISOTROPIC:
        smargin = np.full(len(regions), np.inf)
    nz = Vz.shape[0]
    sid, sid2 = np.zeros(nz, np.int64), np.full(nz, -1, np.int64)
    zr, zs = np.full(nz, np.inf), np.full(nz, np.inf)
    for k, (m, t0, _t1) in enumerate(regions):
        if t0 == 0:
            sid[m] = rsid[k]
        else:
            sid2[m] = rsid[k]
        zr[m] = min(zr[m], rmargin[k])
        zs[m] = min(zs[m], smargin[k])
    return dict(shape_id=sid, shape_id2=sid2, cut=cut, cut_margin=cut_margin, energy=e,
                rho_margin=zr, snap_margin=zs, regions=regions, region_shape=rsid, region_B=B,
                region_rho=rho32, region_g=g32, region_r=r, region_abar=abar, region_vhat=vhat,
                region_L=L)


# ---------------------------------------------------------------------------
# Stage 2: token reorder (Algorithm 1 stage two)
# ---------------------------------------------------------------------------
def _local_order(shape, t0=0, L=Z):
    """Zone-local raster indices (lt*64 + lh*8 + lw) of frames [t0, t0 + L) in
    block-contiguous order."""
    bt, bh, bw = shape
    out = []
    for kt in range(L // bt):
        for kh in range(Z // bh):
            for kw in range(Z // bw):
                for lt in range(bt):
                    for lh in range(bh):
                        for lw in range(bw):
                            out.append(((t0 + kt * bt + lt) * Z + kh * bh + lh) * Z + kw * bw + lw)
    return np.array(out, dtype=np.int64)


_LOCAL = [_local_order(s) for s in SHAPES]


def partition(shape_id, T, H, W, cut=None, shape_id2=None):
    """src [N] (raster token of each permuted position) and block starts [N_b + 1].

    With cuts, zone m's frames [0, c) take shape_id[m] and frames [c, 8)
    shape_id2[m]; the first part's blocks come first."""
    zh_n, zw_n = H // Z, W // Z
    src = np.empty(T * H * W, dtype=np.int64)
    starts = [0]
    for m, sid in enumerate(shape_id):
        zt, rem = divmod(m, zh_n * zw_n)
        zh, zw = divmod(rem, zw_n)
        c = 0 if cut is None else int(cut[m])
        parts = [(0, Z, int(sid))] if c == 0 else [(0, c, int(sid)), (c, Z, int(shape_id2[m]))]
        pos = 512 * m
        for t0, t1, s in parts:
            loc = _LOCAL[s] if t1 - t0 == Z else _local_order(SHAPES[s], t0, t1 - t0)
            lt, lh, lw = loc // 64, (loc // 8) % 8, loc % 8
            src[pos: pos + len(loc)] = ((zt * Z + lt) * H + zh * Z + lh) * W + zw * Z + lw
            vol = int(np.prod(SHAPES[s]))
            starts.extend(pos + vol * (k + 1) for k in range(len(loc) // vol))
            pos += len(loc)
    return src, np.array(starts, dtype=np.int64)


def pool(X, src, starts):
    """Block means (float64) of X [N, D] raster over the permuted blocks."""
    Xp = np.asarray(X, dtype=np.float64)[src]
    sums = np.add.reduceat(Xp, starts[:-1], axis=0)
    return sums / np.diff(starts)[:, None]


# ---------------------------------------------------------------------------
# Stage 3: block scoring and hybrid Top-k U Top-p ("Metode" 3)
# ---------------------------------------------------------------------------
def block_probs(Qbar, Kbar):
    """P_i = softmax_j(Qbar_i . Kbar_j / sqrt(D)) with float32 logits: (s32, P32)."""
    D = Qbar.shape[1]
    s = (np.asarray(Qbar, np.float64) @ np.asarray(Kbar, np.float64).T / np.sqrt(D)).astype(F32)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    P = (e / e.sum(axis=1, keepdims=True)).astype(F32)
    return s, P


def select_row(P_row, k, p):
    """Selected key blocks (ascending) of one query block: first max(k, L) of the order."""
    nb = P_row.shape[0]
    order = np.argsort(-P_row, kind="stable")           # P descending, j ascending
    if p >= 1.0:
        L = nb
    elif p <= 0.0:
        L = 0
    else:
        cum = np.cumsum(P_row[order], dtype=F32)        # sequential float32 sum
        hit = np.nonzero(cum >= F32(p))[0]
        L = int(hit[0]) + 1 if hit.size else nb
    cnt = max(min(int(k), nb), L)
    return np.sort(order[:cnt]), order, cnt


def k_of_fraction(frac, nb):
    """k = ceil(frac * N_b) with the product in float32 (the pages' "Top-k 95%"
    is a sparsity: frac = 0.05 keeps 5% of the key blocks)."""
    return int(np.ceil(F32(frac) * F32(nb)))


def select(Qbar, Kbar, k, p, k_frac=0.0):
    """List of selected key-block arrays for every query block, plus (s32, P32).
    k_frac > 0 replaces k by k_of_fraction(k_frac, N_b)."""
    s, P = block_probs(Qbar, Kbar)
    if k_frac > 0:
        k = k_of_fraction(k_frac, P.shape[1])
    sel = [select_row(P[i], k, p)[0] for i in range(P.shape[0])]
    return sel, s, P


# ---------------------------------------------------------------------------
# Whole plan for one head
# ---------------------------------------------------------------------------
def plan_head(Q, K, V, a, T, H, W, k, p, eps, tau128=0.5, tau256=0.25, shape_id=None, alpha=0.5,
              shape_mode=SHAPE_DYNAMIC, fixed_shape=0, k_frac=0.0, cut_ratio=0.0, cut=None, shape_id2=None):
    """Stages one to three for one head.  Q, K, V: [N, D] raster.  shape_id (and,
    with adaptive boundaries, cut and shape_id2) replace stage one's result."""
    st = zone_shapes(V, a, T, H, W, eps, tau128, tau256, alpha, shape_mode, fixed_shape, cut_ratio)
    sid = st["shape_id"] if shape_id is None else np.asarray(shape_id)
    cut = st["cut"] if cut is None else np.asarray(cut)
    sid2 = st["shape_id2"] if shape_id2 is None else np.asarray(shape_id2)
    src, starts = partition(sid, T, H, W, cut, sid2)
    Qbar, Kbar = pool(Q, src, starts), pool(K, src, starts)
    sel, s, P = select(Qbar, Kbar, k, p, k_frac)
    return dict(stats=st, shape_id=sid, cut=cut, shape_id2=sid2, src=src, starts=starts, Qbar=Qbar,
                Kbar=Kbar, sel=sel, logits=s, P=P)


def block_of_token(src, starts):
    """Block id of every raster token."""
    nb = len(starts) - 1
    bid_perm = np.repeat(np.arange(nb), np.diff(starts))
    out = np.empty_like(bid_perm)
    out[src] = bid_perm
    return out


def token_mask(src, starts, sel):
    """Dense [N, N] bool mask M[q, n] = block(n) in S_{block(q)} (raster order)."""
    nb = len(starts) - 1
    bsel = np.zeros((nb, nb), dtype=bool)
    for i, js in enumerate(sel):
        bsel[i, js] = True
    bt = block_of_token(src, starts)
    return bsel[bt][:, bt]


# ---------------------------------------------------------------------------
# Stage 4-5: sparse attention over the selected blocks, output in raster order
# ---------------------------------------------------------------------------
def attention_fwd(Q, K, V, src, starts, sel):
    """O [N, D] and LSE [N] (float64, raster order) of attention restricted to S_i."""
    Q, K, V = (np.asarray(x, np.float64) for x in (Q, K, V))
    D = Q.shape[1]
    O = np.empty_like(Q)
    lse = np.empty(Q.shape[0])
    for i, js in enumerate(sel):
        qi = src[starts[i]:starts[i + 1]]
        keys = np.concatenate([src[starts[j]:starts[j + 1]] for j in js])
        s = Q[qi] @ K[keys].T
        s /= np.sqrt(D)                                  # logits
        m = s.max(axis=1, keepdims=True)
        s -= m
        np.exp(s, out=s)                                 # exp(logit - row max)
        z = s.sum(axis=1, keepdims=True)
        s /= z                                           # softmax over the row's keys
        O[qi] = s @ V[keys]
        lse[qi] = (m + np.log(z))[:, 0]
    return O, lse


def block_grads(Q, K, V, dO, O, lse, src, starts, sel, i, dQ, dK, dV):
    """Gradient contributions of query block i (float64, raster order):
    dQ rows of the block, and its terms of dK, dV over the keys of S_i."""
    D = Q.shape[1]
    sc = 1.0 / np.sqrt(D)
    qi = src[starts[i]:starts[i + 1]]
    keys = np.concatenate([src[starts[j]:starts[j + 1]] for j in sel[i]])
    Kk, Vk, Qi, g = K[keys], V[keys], Q[qi], dO[qi]
    P = Qi @ Kk.T
    P *= sc
    P -= lse[qi][:, None]
    np.exp(P, out=P)                                     # P = exp(S / sqrt(D) - LSE)
    dV[keys] += P.T @ g
    dS = g @ Vk.T                                        # dP
    dS -= (g * O[qi]).sum(axis=1, keepdims=True)         # dP - D_i
    dS *= P                                              # dS = P o (dP - D)
    dQ[qi] = dS @ Kk * sc
    dK[keys] += dS.T @ Qi * sc


def attention_bwd(Q, K, V, dO, src, starts, sel):
    """dQ, dK, dV (float64, raster order): exact gradients with the selection fixed."""
    Q, K, V, dO = (np.asarray(x, np.float64) for x in (Q, K, V, dO))
    O, lse = attention_fwd(Q, K, V, src, starts, sel)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for i in range(len(sel)):
        block_grads(Q, K, V, dO, O, lse, src, starts, sel, i, dQ, dK, dV)
    return dQ, dK, dV


def block_selection_matrix(sel, nb):
    """Boolean [nb, nb]: entry (i, j) is True when key block j is in S_i."""
    bsel = np.zeros((nb, nb), dtype=bool)
    for i, js in enumerate(sel):
        bsel[i, js] = True
    return bsel


def attention_rows(Q, K, V, src, starts, sel, rows, dO=None, chunk=64):
    """Forward (and dQ when dO is given) for selected raster query rows only,
    from the masked definition: row q attends to every key n whose block is in
    S_block(q), with a softmax over exactly those keys.

    Rows are taken `chunk` at a time against all N keys (masked logits are
    -inf), so no key is gathered.  Returns O [len(rows), D], LSE [len(rows)]
    and optionally dQ [len(rows), D] (float64).
    """
    Q, K, V = (np.asarray(x, np.float64) for x in (Q, K, V))
    D = Q.shape[1]
    sc = 1.0 / np.sqrt(D)
    rows = np.asarray(rows, dtype=np.int64)
    bt = block_of_token(src, starts)
    bsel = block_selection_matrix(sel, len(starts) - 1)
    O = np.empty((len(rows), D))
    lse = np.empty(len(rows))
    dQ = np.empty((len(rows), D)) if dO is not None else None
    for r0 in range(0, len(rows), chunk):
        rr = rows[r0:r0 + chunk]
        mask = bsel[bt[rr]][:, bt]                                 # [r, N]
        P = Q[rr] @ K.T
        P *= sc
        P[~mask] = -np.inf                                         # keys outside the selection
        m = P.max(axis=1, keepdims=True)
        P -= m
        np.exp(P, out=P)
        z = P.sum(axis=1, keepdims=True)
        P /= z                                                     # softmax over the selected keys
        O[r0:r0 + len(rr)] = P @ V
        lse[r0:r0 + len(rr)] = (m + np.log(z))[:, 0]
        if dO is not None:
            g = np.asarray(dO[rr], np.float64)
            dS = g @ V.T                                           # dP
            dS -= (g * O[r0:r0 + len(rr)]).sum(axis=1, keepdims=True)
            dS *= P                                                # P o (dP - D)
            dQ[r0:r0 + len(rr)] = dS @ K * sc
    return O, lse, dQ


def attention_key_rows(Q, K, V, dO, src, starts, sel, key_rows):
    """dK and dV [len(key_rows), D] (float64) of selected raster key rows.

    Key n receives, from every query row q whose block selects block(n), the
    terms P[q, n] dO_q (dV) and P[q, n] (dP[q, n] - D_q) Q_q / sqrt(D) (dK),
    where P[q, .] is q's softmax over all keys of its selection (its full LSE),
    dP[q, n] = dO_q . V_n and D_q = dO_q . O_q.  The query blocks that select
    a sampled key's block are evaluated whole, one at a time (practical when
    the selections are short).
    """
    Q, K, V, dO = (np.asarray(x, np.float64) for x in (Q, K, V, dO))
    D = Q.shape[1]
    sc = 1.0 / np.sqrt(D)
    key_rows = np.asarray(key_rows, dtype=np.int64)
    bt = block_of_token(src, starts)
    nb = len(starts) - 1
    bsel = block_selection_matrix(sel, nb)
    dK = np.zeros((len(key_rows), D))
    dV = np.zeros((len(key_rows), D))
    kblk = bt[key_rows]
    users = np.nonzero(bsel[:, np.unique(kblk)].any(axis=1))[0]   # query blocks that select any of them
    for i in users:
        qi = src[starts[i]:starts[i + 1]]
        keys = np.concatenate([src[starts[j]:starts[j + 1]] for j in sel[i]])
        s = Q[qi] @ K[keys].T * sc
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        P = e / e.sum(axis=1, keepdims=True)                      # [|B_i|, |keys|]
        Oi = P @ V[keys]
        g = dO[qi]
        Di = (g * Oi).sum(axis=1)
        col = {int(n): c for c, n in enumerate(keys)}
        for r in np.nonzero(bsel[i, kblk])[0]:
            n = int(key_rows[r])
            p = P[:, col[n]]
            dV[r] += p @ g
            dK[r] += (p * (g @ V[n] - Di)) @ Q[qi] * sc
    return dK, dV


# ---------------------------------------------------------------------------
# Guidance map producer: the audio-to-video cross-attention output norm.
# Page paper.rainbus.top, section "前置知识" (the dual-branch DiT paragraph): the
# video hidden state takes in audio through h_hat = CrossAttn(h, K_a, V_a), and
# the L2 norm of that output measures how much audio a video position absorbed.
# Page xyznot.com/id, section "Metode" 1: a_{t,h,w} = ||h_hat_{t,h,w}||_2, cached
# from the previous layer (page xyznot.com/th, section on limitations: the
# self-attention runs before the cross-attention inside a block, hence the
# one-layer lag).  Reading (the pages print no formula for the multi-head
# case): h_hat of a token is the concatenation over heads of
# softmax(q_h K_{a,h}^T / sqrt(D)) V_{a,h}, taken before the output projection
# (which needs the backbone's weights), and the norm runs over all heads'
# channels.
def av_cross_attn(Qv, Ka, Va):
    """Per-head cross-attention outputs h_hat [heads, N, D] (float64).

    Qv [heads, N, D]: the video tokens' queries; Ka, Va [heads, M, D]: the
    audio tokens' keys and values.  Softmax over the M audio tokens, logits
    scaled by 1/sqrt(D), max subtracted before exp."""
    Qv, Ka, Va = (np.asarray(x, np.float64) for x in (Qv, Ka, Va))
    heads, N, D = Qv.shape
    out = np.empty((heads, N, D))
    for h in range(heads):
        for r0 in range(0, N, 4096):
            s = Qv[h, r0:r0 + 4096] @ Ka[h].T / np.sqrt(D)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            out[h, r0:r0 + 4096] = (e / e.sum(axis=1, keepdims=True)) @ Va[h]
    return out


def av_norm_map(Qv, Ka, Va):
    """The guidance map a [N] = ||h_hat||_2 over the concatenated heads, and
    h_hat [heads, N, D] (float64)."""
    hh = av_cross_attn(Qv, Ka, Va)
    return np.sqrt((hh * hh).sum(axis=(0, 2))), hh


def av_norm_rows(Qv, Ka, Va, rows):
    """a and h_hat [heads, len(rows), D] for the given token rows only."""
    rows = np.asarray(rows)
    return av_norm_map(np.asarray(Qv)[:, rows], Ka, Va)
