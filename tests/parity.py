"""Comparison rules between the CUDA path and the CPU oracle.

Integer decisions (block volume, shape, selected set) must agree exactly,
except where the oracle's own margin shows a near-tie: a shape may differ only
where |rho - tau| or the gap between the two nearest candidates is below
1e-5; a selected set may differ only in blocks whose logit lies within 1e-5
of the boundary block's logit, and its size only as far as moving p by 1e-5
moves the Top-p prefix.  Attention outputs and gradients from bf16 inputs
must reach relative L2 <= 1e-2 and max-abs <= 3e-2 against the oracle
(gradients: max-abs 3e-2 plus half a bf16 ulp of the tensor's largest
magnitude, close_grad).
"""
import numpy as np

TIE = 1e-5
REL_L2 = 1e-2
MAX_ABS = 3e-2
# Gradients: the max-abs bar holds at unit scale; the elements may in addition
# carry half an ulp of the pages' 16-bit operand format (bf16: 2^-9) of the
# compared tensor's largest magnitude.  The backward is linear in dO, so a purely
# absolute bar would depend on the caller's scale of dO; the operating point's dK
# reaches 170 at unit-variance dO, and an element is a sum of terms of that size
# that may cancel, so one fp16 rounding of a dominant dS term (2^-12 relative)
# alone is 0.04 whatever the element's own size.
GRAD_RTOL = 2.0 ** -9


def bits_to_sets(words, nb, nwords):
    rows = []
    w = np.asarray(words, dtype=np.uint32).reshape(-1, nwords)
    for i in range(nb):
        b = np.unpackbits(w[i].view(np.uint8), bitorder="little")[:nb]
        rows.append(np.nonzero(b)[0])
    return rows


def sets_to_bits(sel, nb_max, nwords):
    out = np.zeros((nb_max, nwords), dtype=np.uint32)
    for i, js in enumerate(sel):
        for j in js:
            out[i, j >> 5] |= np.uint32(1) << np.uint32(j & 31)
    return out


def shapes_agree(gpu_sid, st, gpu_cut=None, gpu_sid2=None):
    """(exact matches, accepted near-tie mismatches, bad zones).  With adaptive
    temporal boundaries the split position and the second part's shape are
    compared too; a split decision may differ only where the oracle's relative
    cut margin is below the tie bound."""
    bad, tie = [], []
    cut_m = st.get("cut_margin")
    for m, (g, o) in enumerate(zip(gpu_sid, st["shape_id"])):
        same = int(g) == int(o)
        if gpu_cut is not None:
            same = same and int(gpu_cut[m]) == int(st["cut"][m])
            if same and int(st["cut"][m]):
                same = int(gpu_sid2[m]) == int(st["shape_id2"][m])
        if not same:
            near = st["rho_margin"][m] < TIE or st["snap_margin"][m] < TIE
            if cut_m is not None and cut_m[m] < TIE:
                near = True
            (tie if near else bad).append(m)
    return len(gpu_sid) - len(bad) - len(tie), tie, bad


def _prefix_len(cum, p):
    if p >= 1.0:
        return len(cum)
    if p <= 0.0:
        return 0
    hit = np.nonzero(cum >= np.float32(p))[0]
    return int(hit[0]) + 1 if hit.size else len(cum)


def selection_agrees(gpu_set, logits, P, k, p):
    """True if the GPU's set for one row is the oracle's up to near-ties."""
    nb = len(P)
    order = np.argsort(-P, kind="stable")
    cum = np.cumsum(P[order], dtype=np.float32)
    kk = min(int(k), nb)
    lo = max(kk, _prefix_len(cum, p - TIE)) if 0 < p < 1 else max(kk, _prefix_len(cum, p))
    hi = max(kk, _prefix_len(cum, p + TIE)) if 0 < p < 1 else lo
    n = len(gpu_set)
    if not (lo <= n <= hi):
        return False
    want = set(order[:n].tolist())
    got = set(np.asarray(gpu_set).tolist())
    if want == got:
        return True
    edge = logits[order[n - 1]]
    return all(abs(float(logits[j]) - float(edge)) <= TIE for j in want ^ got)


def close(a, b, rel=REL_L2, mabs=MAX_ABS):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rl2 = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    ma = float(np.max(np.abs(a - b))) if a.size else 0.0
    return rl2 <= rel and ma <= mabs, rl2, ma


def close_grad(a, b, rel=REL_L2, mabs=MAX_ABS, rtol=GRAD_RTOL):
    """Gradient comparison: relative L2 <= rel over the tensor and, per element,
    |a - b| <= mabs + rtol max|b|.  Returns (ok, relL2, max-abs, max-abs as a
    fraction of the bound)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rl2 = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    ma = float(np.abs(a - b).max()) if a.size else 0.0
    bound = mabs + rtol * (float(np.abs(b).max()) if b.size else 0.0)
    return rl2 <= rel and ma <= bound, rl2, ma, ma / bound
