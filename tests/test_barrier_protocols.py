"""Models of the attention kernels' mbarrier protocols, checked on the host.

Covered: the forward (k_attn_fwd), the backward (k_bwd_dkdv, with and without
the fused dQ drain; k_bwd_dq for head_dim 64) and the guidance-map producer
(k_av_norm).

Each kernel role (TMA producer lanes, MMA issuers, softmax groups) is written
as the sequence of its barrier operations, in the order and with the phase
parities the kernel source uses: ('wait', barrier, k) waits for the k-th
completion of the barrier (parity k & 1), ('arrive', barrier) arrives once.
Completions are immediate in the model (an MMA commit arrives when issued, a
TMA load completes when issued), and the roles are interleaved at random.  A
correct protocol never deadlocks and never waits on a barrier that has already
completed two or more phases past the awaited one (a parity wait would then
return at the wrong phase).  The kernels also bound every wait in time; these
models check that no wait should ever need that bound.
"""
import random

import pytest


def run(roles, counts, seed):
    """None if the interleaving completes, else a description of the failure."""
    rng = random.Random(seed)
    gens = [r() for r in roles]
    cur = [next(g, None) for g in gens]
    arrivals = {}
    done = lambda b: arrivals.get(b, 0) // counts.get(b, 1)
    while any(c is not None for c in cur):
        ready = []
        for i, c in enumerate(cur):
            if c is None:
                continue
            if c[0] == "arrive":
                ready.append(i)
                continue
            k = done(c[1])
            if k >= c[2] + 2:
                return f"role {i} waits for phase {c[2]} of {c[1]} after {k} completions"
            if k >= c[2] + 1:
                ready.append(i)
        if not ready:
            return f"deadlock at {cur}"
        i = rng.choice(ready)
        if cur[i][0] == "arrive":
            arrivals[cur[i][1]] = arrivals.get(cur[i][1], 0) + 1
        cur[i] = next(gens[i], None)
    return None


# ---------------------------------------------------------------- forward
def forward_roles(n, KST=2, VST=2):
    """k_attn_fwd: two softmax groups take the key tiles alternately (steps
    j = g mod 2), S released after it is read (s_free), QK and PV issuers."""
    def producer_k():
        yield ("arrive", "q")
        for j in range(n):
            s = j % KST
            if j >= KST:
                yield ("wait", f"k_empty{s}", j // KST - 1)
            yield ("arrive", f"k_full{s}")

    def producer_v():
        for j in range(n):
            s = j % VST
            if j >= VST:
                yield ("wait", f"v_empty{s}", j // VST - 1)
            yield ("arrive", f"v_full{s}")

    def qk():
        if n:
            yield ("wait", "q", 0)
        for j in range(n):
            b = j & 1
            if j >= 2:
                yield ("wait", f"s_free{b}", (j - 2) >> 1)
            yield ("wait", f"k_full{j % KST}", j // KST)
            yield ("arrive", f"s_full{b}")
            yield ("arrive", f"k_empty{j % KST}")

    def pv():
        for j in range(n):
            b = j & 1
            yield ("wait", f"p_full{b}", j >> 1)
            yield ("wait", f"v_full{j % VST}", j // VST)
            yield ("arrive", f"pv_done{b}")
            yield ("arrive", f"v_empty{j % VST}")

    def group(g):
        def f():
            cnt = 0
            for j in range(g, n, 2):
                yield ("wait", f"s_full{g}", j >> 1)
                yield ("arrive", f"s_free{g}")
                if cnt:
                    yield ("wait", f"pv_done{g}", (j - 2) >> 1)
                yield ("arrive", f"p_full{g}")
                cnt += 1
            for gg in (g, g ^ 1):                 # own group's last product first
                if n > gg:
                    jl = gg + 2 * ((n - 1 - gg) // 2)
                    yield ("wait", f"pv_done{gg}", jl >> 1)
        return f

    return [producer_k, producer_v, qk, pv, group(0), group(1)]


@pytest.mark.parametrize("n", list(range(0, 10)) + [31, 64])
def test_forward_protocol(n):
    for seed in range(200):
        assert run(forward_roles(n), {}, seed) is None, (n, seed)


# ------------------------------------------------------- guidance map
def av_roles(heads, MT, ST=2):
    """k_av_norm: steps j = head * MT + key tile; Q double-buffered by head, K/V
    rings, S double-buffered, two O accumulators alternating by head (lagged
    epilogue), rescale waits on the previous product."""
    J = heads * MT

    def producer_qk():
        for j in range(J):
            h, kt = divmod(j, MT)
            if kt == 0:
                if h >= 2:
                    yield ("wait", f"q_empty{h & 1}", (h >> 1) - 1)
                yield ("arrive", f"q_full{h & 1}")
            if j >= ST:
                yield ("wait", f"k_empty{j % ST}", j // ST - 1)
            yield ("arrive", f"k_full{j % ST}")

    def producer_v():
        for j in range(J):
            if j >= ST:
                yield ("wait", f"v_empty{j % ST}", j // ST - 1)
            yield ("arrive", f"v_full{j % ST}")

    def mma():
        for j in range(J + 1):
            if j < J:
                h, kt = divmod(j, MT)
                if kt == 0:
                    yield ("wait", f"q_full{h & 1}", h >> 1)
                yield ("wait", f"k_full{j % ST}", j // ST)
                yield ("arrive", f"s_full{j & 1}")
                yield ("arrive", f"k_empty{j % ST}")
                if kt == MT - 1:
                    yield ("arrive", f"q_empty{h & 1}")
            if j >= 1:
                jj = j - 1
                hh, kt = divmod(jj, MT)
                yield ("wait", f"p_full{jj & 1}", jj >> 1)
                yield ("wait", f"v_full{jj % ST}", jj // ST)
                if kt == 0 and hh >= 2:
                    yield ("wait", f"o_free{hh & 1}", (hh >> 1) - 1)
                yield ("arrive", f"pv_done{jj & 1}")
                yield ("arrive", f"v_empty{jj % ST}")

    def softmax(rescale_every_step):
        def f():
            for j in range(J):
                h, kt = divmod(j, MT)
                yield ("wait", f"s_full{j & 1}", j >> 1)
                if kt > 0 and rescale_every_step:
                    yield ("wait", f"pv_done{(j - 1) & 1}", (j - 1) >> 1)
                yield ("arrive", f"p_full{j & 1}")
                if kt == 0 and h > 0:
                    yield ("wait", f"pv_done{(j - 1) & 1}", (j - 1) >> 1)
                    yield ("arrive", f"o_free{(h - 1) & 1}")
            yield ("wait", f"pv_done{(J - 1) & 1}", (J - 1) >> 1)
        return f

    return [producer_qk, producer_v, mma], softmax


@pytest.mark.parametrize("heads,MT", [(1, 1), (2, 1), (3, 2), (4, 8), (5, 3), (40, 8)])
@pytest.mark.parametrize("rescale", [False, True])
def test_guidance_map_protocol(heads, MT, rescale):
    roles, softmax = av_roles(heads, MT)
    for seed in range(60 if heads < 40 else 8):
        assert run(roles + [softmax(rescale)], {}, seed) is None, (heads, MT, seed)


# ------------------------------------------------------------- backward
def backward_roles(U, fuse=True, ST=3):
    """k_bwd_dkdv: 64-query units of a key tile, a 3-stage Q/dO ring, S^T/dP^T
    double-buffered in TMEM; issuer A (S^T, dP^T), issuer B (dV and dK with
    P^T and dS^T read from TMEM, then dQ^T), softmax (P'^T over dP^T and dS^T
    over S^T in TMEM, dS^T also into shared memory when fused), dQ^T drain
    (fuse)."""
    def producer():
        yield ("arrive", "kv")
        for u in range(U):
            s = u % ST
            if u >= ST:
                yield ("wait", f"st_empty{s}", u // ST - 1)
            yield ("arrive", f"st_full{s}")

    def issuer_a():
        yield ("wait", "kv", 0)
        for u in range(U):
            b = u & 1
            yield ("wait", f"st_full{u % ST}", u // ST)
            if u >= 2:
                yield ("wait", f"pd_done{b}", (u - 2) >> 1)          # S^T over dS^T(u - 2)
                yield ("wait", f"dq_free{b}" if fuse else f"pd_done{b}", (u - 2) >> 1)
            yield ("arrive", f"s_full{b}")

    def issuer_b():
        for u in range(U):
            b = u & 1
            yield ("wait", f"p_full{b}", u >> 1)
            yield ("arrive", f"pd_done{b}")
            yield ("arrive", f"st_empty{u % ST}")
            if fuse:
                yield ("arrive", f"dq_full{b}")
        yield ("arrive", "acc_done")

    def softmax():
        for u in range(U):
            b = u & 1
            yield ("wait", f"s_full{b}", u >> 1)
            yield ("wait", f"st_full{u % ST}", u // ST)
            if fuse and u >= 2:
                yield ("wait", f"dq_full{b}", (u - 2) >> 1)          # dS^T(u - 2) in shared memory read
            yield ("arrive", f"p_full{b}")
        yield ("wait", "acc_done", 0)

    def drain():
        for u in range(U):
            b = u & 1
            yield ("wait", f"dq_full{b}", u >> 1)
            yield ("arrive", f"dq_free{b}")

    return [producer, issuer_a, issuer_b, softmax] + ([drain] if fuse else [])


@pytest.mark.parametrize("U", list(range(1, 10)) + [33, 100])
@pytest.mark.parametrize("fuse", [True, False])
def test_backward_protocol(U, fuse):
    for seed in range(150):
        assert run(backward_roles(U, fuse), {}, seed) is None, (U, fuse, seed)


def dq_roles(U, ST=2):
    """k_bwd_dq (head_dim 64): one 128-query tile, 64-key units; one issuer
    (S and dP of unit u, then dQ += dS K of unit u - 1), the softmax forms dS."""
    def producer():
        yield ("arrive", "q")
        for u in range(U):
            if u >= ST:
                yield ("wait", f"st_empty{u % ST}", u // ST - 1)
            yield ("arrive", f"st_full{u % ST}")

    def issuer():
        yield ("wait", "q", 0)
        for u in range(U + 1):
            if u < U:
                yield ("wait", f"st_full{u % ST}", u // ST)
                if u >= 2:
                    yield ("wait", f"s_free{u & 1}", (u - 2) >> 1)
                yield ("arrive", f"s_full{u & 1}")
            if u >= 1:
                uu = u - 1
                yield ("wait", f"ds_full{uu & 1}", uu >> 1)
                yield ("arrive", f"dq_done{uu & 1}")
                yield ("arrive", f"st_empty{uu % ST}")

    def softmax():
        for u in range(U):
            b = u & 1
            yield ("wait", f"s_full{b}", u >> 1)
            yield ("arrive", f"s_free{b}")
            if u >= 2:
                yield ("wait", f"dq_done{b}", (u - 2) >> 1)
            yield ("arrive", f"ds_full{b}")
        if U:
            yield ("wait", f"dq_done{(U - 1) & 1}", (U - 1) >> 1)

    return [producer, issuer, softmax]


@pytest.mark.parametrize("U", list(range(0, 9)) + [40])
def test_dq_protocol(U):
    for seed in range(150):
        assert run(dq_roles(U), {}, seed) is None, (U, seed)


def test_model_catches_a_wrong_parity():
    """A planted mistake: the PV issuer of the forward waiting on p_full with the
    step's own parity shifted by one phase deadlocks (the model is not vacuous)."""
    roles = forward_roles(6)

    def pv_wrong():
        for j in range(6):
            yield ("wait", f"p_full{j & 1}", (j >> 1) + 1)
            yield ("wait", f"v_full{j % 2}", j // 2)
            yield ("arrive", f"pv_done{j & 1}")
            yield ("arrive", f"v_empty{j % 2}")

    roles[3] = pv_wrong
    assert run(roles, {}, 0) is not None
