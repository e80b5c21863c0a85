#!/usr/bin/env python
"""Prism sparse video self-attention benchmark on B200.

One step = one head-layer of the 2K training workload (grid 72x88x160,
1,013,760 tokens, head_dim 128, bf16 inputs, Top-k 16, Top-p 0.9): the plan
(zone statistics, shapes, reorder, pooling, selection), the sparse attention
forward and its backward, heads processed in sequence.  With N GPUs (one
process each, launched by torchrun) every rank runs its own heads: weak
scaling, no collective on the data path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl prism|reference]

Prints one JSON line (rank 0).  `value` is milliseconds per head-layer for the
whole job (lower is better); the dominant kernel's roofline, the end-to-end
number through the C ABI with host buffers, and the CPU oracle baseline ride
along.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Prism sparse-attn fwd+bwd ms/head-layer @1M tokens; achieved tensor TFLOP/s"
UNIT = "ms/head-layer"


def args_():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["prism", "reference"], default="prism")
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--grid", type=int, nargs=3, default=None, metavar=("T", "H", "W"),
                    help="override the grid (smaller cases for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="attention sample budget of the CPU oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense same-shape comparison (torch SDPA and all-blocks Prism)")
    # variants of the pages' ablation and operating point (defaults: the workload's method)
    ap.add_argument("--top-k", type=int, default=None)
    ap.add_argument("--top-p", type=float, default=None)
    ap.add_argument("--topk-frac", type=float, default=0.0,
                    help="k as a fraction of each head's blocks (the pages' Top-k 95%% = 0.05)")
    ap.add_argument("--alpha", type=float, default=0.5, help="shape-mapping exponent (1/2: the method)")
    ap.add_argument("--shape-mode", choices=["dynamic", "isotropic", "fixed"], default="dynamic")
    ap.add_argument("--fixed-shape", type=int, default=3, help="candidate index for --shape-mode fixed")
    ap.add_argument("--cut-ratio", type=float, default=0.0,
                    help="adaptive temporal zone boundaries: split a zone where its largest frame-difference "
                         "energy exceeds this multiple of the median (0: whole zones, the method)")
    ap.add_argument("--shot-cuts", type=int, nargs="*", default=[],
                    help="frames where the synthetic fields start a new shot")
    ap.add_argument("--av-tokens", type=int, default=1000,
                    help="audio tokens of the guidance-map producer leg (the pages: under 1K)")
    ap.add_argument("--no-av", action="store_true", help="skip the guidance-map producer leg")
    ap.add_argument("--no-op", action="store_true",
                    help="skip the leg at the pages' operating point (k = 5%% of the blocks, Top-p 0.2)")
    ap.add_argument("--sweep", action="store_true",
                    help="the 2K inference sweep instead of the step: forward only on grid 64x88x152, "
                         "peaked (Q, K x3) and diffuse (x0.5) logits, Top-k 8/16/32 x Top-p 0.8/0.9/0.95")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers
def head_order(rank, world, need, heads):
    """The heads a rank processes, in order: `need` consecutive heads starting
    at rank * need (mod heads), so ranks work on different heads while
    rank * need < heads."""
    return [(rank * need + i) % heads for i in range(need)]


def max_over_ranks(value, world, device=None):
    """Max of a per-rank float over all ranks (the job's time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def selected_pairs(pl, head=0):
    """Pi = sum_i |B_i| * sum_{j in S_i} |B_j| of a plan (exported, host)."""
    import numpy as np
    p = pl.params
    N = p.T * p.H * p.W
    NB = N // 64
    words = (NB + 31) // 32
    nb = int(pl.export("nblocks")[head])
    st = pl.export("blk_start").reshape(-1, NB + 1)[head, :nb + 1].astype(np.int64)
    size = np.diff(st)
    bits = pl.export("sel_bits").reshape(-1, NB, words)[head, :nb]
    sel = np.unpackbits(bits.view(np.uint8), axis=1, bitorder="little")[:, :nb].astype(np.int64)
    keys = sel @ size
    return int((size * keys).sum()), nb, float(sel.sum(1).mean())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *exc):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        import statistics
        rows = []
        self.f.flush()
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        mx = max(r[1] for r in rows)
        load = [r[0] for r in rows if r[0] > 0.5 * mx] or [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


KERNEL_TU = {"k_bwd_dkdv": "prism_attn_bwd.cu", "k_attn_fwd": "prism_attn_fwd.cu",
             "k_av_norm": "prism_av_norm.cu"}


def source_digest(kernel):
    """First 16 hex digits of sha256 over the kernel's translation unit, then
    csrc/prism_dev.cuh and csrc/prism_internal.h (None for an unknown kernel)."""
    import hashlib
    tu = KERNEL_TU.get(kernel)
    if tu is None:
        return None
    m = hashlib.sha256()
    for f in (tu, "prism_dev.cuh", "prism_internal.h"):
        with open(os.path.join(ROOT, "dynamic_block_sparse_indicator_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


TRAFFIC_PROFILE = "dram_traffic_k_bwd_dkdv_grid16x64x144_grid16x64x288.md"


def measured_traffic(kernel, pairs, path=None):
    """DRAM bytes of one launch of `kernel` at `pairs` selected token pairs,
    scaled from the committed one-launch ncu captures on small grids (the table
    in profiles/dram_traffic_k_bwd_dkdv_grid16x64x144_grid16x64x288.md gives the captured
    bytes and the captured grid's selected pairs) by the ratio of selected pairs
    (the kernel's traffic per launch follows its work: every unit loads one Q/dO
    tile and every (key tile, chunk) one K/V tile and one dK/dV reduce); of
    several captures the one on the largest grid (most selected pairs).  None
    if the kernel's sources changed since the capture (their hash no longer
    matches) or there is no capture."""
    path = path or os.path.join(ROOT, "profiles", TRAFFIC_PROFILE)
    digest = source_digest(kernel)
    if digest is None or not os.path.exists(path):
        return None
    best = None                       # the capture with the most selected pairs
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) == 6 and cells[0] == kernel and cells[5] == digest:
            row = (float(cells[4]), float(cells[1]) + float(cells[2]))
            best = row if best is None or row[0] > best[0] else best
    return None if best is None else best[1] * float(pairs) / best[0]


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        return {}


# --------------------------------------------------------- CPU oracle leg
def variant_of(a):
    """The oracle's keyword arguments for the command line's variant flags."""
    mode = {"dynamic": 0, "isotropic": 1, "fixed": 2}[a.shape_mode]
    return dict(alpha=a.alpha, shape_mode=mode, fixed_shape=a.fixed_shape, k_frac=a.topk_frac,
                cut_ratio=a.cut_ratio)


def workload_of(a):
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    over = {k: v for k, v in (("top_k", a.top_k), ("top_p", a.top_p)) if v is not None}
    if a.grid:
        over.update(T=a.grid[0], H=a.grid[1], W=a.grid[2])
    if a.shot_cuts:
        over.update(shot_cuts=list(a.shot_cuts))
    return syn.workload(a.workload, **over)


def oracle_head_ms(Qh, Kh, Vh, dOh, a, w, budget_s, seed=0, variant=None):
    """The oracle on one head: full plan, then forward + backward on a seeded
    sample of query blocks until `budget_s` elapses; the attention time is
    extrapolated to the head by the share of selected pairs.  Returns
    (ms per head-layer, description, threads)."""
    import numpy as np
    from oracle import prism_oracle as po
    t0 = time.perf_counter()
    pl = po.plan_head(Qh, Kh, Vh, a, w.T, w.H, w.W, w.top_k, w.top_p, w.eps, **(variant or {}))
    t_plan = time.perf_counter() - t0
    src, st, sel = pl["src"], pl["starts"], pl["sel"]
    size = np.diff(st)
    pairs = np.array([size[i] * size[js].sum() for i, js in enumerate(sel)], dtype=np.float64)
    rng = np.random.default_rng(seed)
    order = rng.permutation(len(sel))
    # O and LSE of the sampled blocks come from the oracle forward on those rows
    O = np.zeros_like(Qh)
    lse = np.zeros(Qh.shape[0])
    dQ, dK, dV = np.zeros_like(Qh), np.zeros_like(Kh), np.zeros_like(Vh)
    t1 = time.perf_counter()
    done, pi_s = 0, 0.0
    for i in order:
        qi = src[st[i]:st[i + 1]]
        keys = np.concatenate([src[st[j]:st[j + 1]] for j in sel[i]])
        s = Qh[qi] @ Kh[keys].T / np.sqrt(Qh.shape[1])
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        O[qi] = (e / z) @ Vh[keys]
        lse[qi] = (m + np.log(z))[:, 0]
        po.block_grads(Qh, Kh, Vh, dOh, O, lse, src, st, sel, i, dQ, dK, dV)
        done += 1
        pi_s += pairs[i]
        if time.perf_counter() - t1 > budget_s:
            break
    t_attn = (time.perf_counter() - t1) * pairs.sum() / pi_s
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        threads = os.cpu_count() or 1
    desc = (f"full oracle plan of one head ({t_plan:.1f} s) + forward and backward of {done} of "
            f"{len(sel)} query blocks ({100 * pi_s / pairs.sum():.2f}% of the selected pairs), "
            f"attention time extrapolated by pair share")
    return 1e3 * (t_plan + t_attn), desc, threads


def operating_point_leg(Q, K, V, dO, amap, w, h, peak, steps=3):
    """The pages' operating point (k = 5% of each head's blocks, Top-p 0.2; page
    paper.rainbus.top, "方法步骤详情") on one head of the same workload: plan +
    forward + backward per head-layer, 1 warm-up and `steps` timed steps (CUDA
    events), TFLOP/s over the selected pairs' 14 D Pi flops of the attention."""
    import torch
    from dynamic_block_sparse_indicator_b200 import _lib
    prm = _lib.make_params(w.T, w.H, w.W, 1, w.head_dim, _lib.PRISM_BF16, 0, 0.2, w.eps,
                           out_dtype=_lib.PRISM_F32, top_k_frac=0.05)
    sl = slice(h, h + 1)
    ws = torch.empty(_lib.core_bytes(prm), dtype=torch.uint8, device=Q.device)

    def run(prof):
        pl = _lib.plan(Q[sl], K[sl], V[sl], amap, prm, workspace=ws, compact=True)
        if prof:
            pl.profile(True)
        O, lse = pl.attn_fwd()
        pl.attn_bwd(dO[sl], O, lse)
        return pl

    pl = run(False)
    Pi, nb, sel = selected_pairs(pl)
    del pl
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stage = {}
    e0.record()
    plans = [run(True) for _ in range(steps)]
    e1.record()
    torch.cuda.synchronize()
    for pl in plans:
        for k, (ms, _n) in pl.profile_read().items():
            stage[k] = stage.get(k, 0.0) + ms / steps
    ms = e0.elapsed_time(e1) / steps
    attn = stage["fwd"] + stage["bwd_pre"] + stage["bwd_dkdv"] + stage["bwd_dq"]
    tf = 14 * w.head_dim * Pi / (attn * 1e-3) / 1e12
    return {"top_k_frac": 0.05, "top_p": 0.2, "ms_per_head_layer": ms,
            "stages_ms": {k: stage[k] for k in ("fwd", "bwd_dkdv", "bwd_dq")},
            "attention_tflops": tf, "frac_of_sustained": tf / peak, "selected_pairs": Pi,
            "pair_density": Pi / float(w.N) ** 2, "mean_selected_blocks": sel, "blocks_per_head": nb,
            "note": "plan with the core workspace and index lists sized from their counts"}


# ------------------------------------------------------------- main paths
def emit(d):
    print(json.dumps(d), flush=True)


def run_reference(a, rank, world):
    """The oracle on the host cores, on the same workload and metric."""
    if rank != 0:
        return
    import numpy as np
    import torch
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    w = workload_of(a)
    var = variant_of(a)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    heads = min(w.heads, a.steps + 1)
    Q, K, V = syn.make_qkv(w, device=dev, heads=heads)
    dO = syn.make_dout(w, device=dev, heads=heads, out_dtype=torch.bfloat16)
    amap = syn.make_amap(w, device=dev).cpu().numpy()
    host = lambda t, h: t[h].to("cpu", torch.float64).numpy()
    # warm-up steps: a one-second sample on head 0
    for _ in range(a.warmup):
        oracle_head_ms(host(Q, 0), host(K, 0), host(V, 0), host(dO, 0), amap, w, 1.0, variant=var)
    vals, desc, threads = [], "", 1
    t0 = time.perf_counter()
    for s in range(a.steps):
        h = s % heads
        ms, desc, threads = oracle_head_ms(host(Q, h), host(K, h), host(V, h), host(dO, h), amap, w,
                                           a.cpu_seconds / 4, seed=s, variant=var)
        vals.append(ms)
    wall = time.perf_counter() - t0
    v = float(np.mean(vals))
    # value: the oracle's time for a whole head-layer, extrapolated from each
    # step's bounded sample (a full 1M-token head takes the oracle hours);
    # ms_per_step: what each step actually took, so steps x ms_per_step is the
    # timed region this run really spent
    emit({"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
          "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * wall / max(a.steps, 1),
          "value_extrapolated_from_sample": True, "higher_is_better": False,
          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
          "config": {"workload": w.name(), "grid": [w.T, w.H, w.W], "tokens": w.N,
                     "head_dim": w.head_dim, "top_k": w.top_k, "top_p": w.top_p,
                     "top_k_frac": a.topk_frac, "alpha": a.alpha, "shape_mode": a.shape_mode},
          "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                           "sample": desc, "wall_s": wall},
          "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})


def dense_same_shape(Q, K, V, dO, amap, w, ws, O, lse, dQ, dK, dV, h, peak):
    """Dense attention over all N tokens of one head, fwd + bwd (14 D N^2 flops):
    torch SDPA (flash and cuDNN back ends, where available) and this library with
    every block selected (k >= N_b, p = 1)."""
    import torch
    from dynamic_block_sparse_indicator_b200 import _lib
    D, N = w.head_dim, w.N
    flops = 14.0 * D * float(N) ** 2
    out = {"flops": flops, "tokens": N}

    def timed(fn, reps=1):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    q = Q[h:h + 1].unsqueeze(0).to(torch.bfloat16).detach().requires_grad_(True)
    k = K[h:h + 1].unsqueeze(0).to(torch.bfloat16).detach().requires_grad_(True)
    v = V[h:h + 1].unsqueeze(0).to(torch.bfloat16).detach().requires_grad_(True)
    g = dO[h:h + 1].unsqueeze(0).to(torch.bfloat16)
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        backends = {"sdpa_flash": SDPBackend.FLASH_ATTENTION, "sdpa_cudnn": SDPBackend.CUDNN_ATTENTION}
    except ImportError:
        backends = {}
    for name, be in backends.items():
        try:
            def run():
                with sdpa_kernel([be]):
                    o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
                torch.autograd.backward(o, g)
                q.grad = k.grad = v.grad = None
            ms = timed(run)
            out[name] = {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12}
        except Exception as exc:  # noqa: BLE001
            out[name] = {"unavailable": str(exc).splitlines()[0][:160]}
    del q, k, v, g
    params = _lib.make_params(w.T, w.H, w.W, 1, D, _lib.PRISM_BF16, 1 << 30, 1.0, w.eps,
                              out_dtype=_lib.PRISM_F32)

    last = []

    def prism_all():
        pl = _lib.plan(Q[h:h + 1], K[h:h + 1], V[h:h + 1], amap, params, workspace=ws)
        pl.attn_fwd(O, lse)
        pl.attn_bwd(dO[h:h + 1], O, lse, dQ, dK, dV)
        last[:] = [pl]

    ms = timed(prism_all)
    st = last[0].status()
    if st:
        raise RuntimeError(f"device status (all blocks): {_lib.status_string(st)}")
    last.clear()
    out["prism_all_blocks"] = {"ms": ms, "tflops": flops / (ms * 1e-3) / 1e12,
                               "fraction_of_peak": flops / (ms * 1e-3) / 1e12 / peak,
                               "note": "plan + fwd + bwd with k >= N_b and p = 1 (every block selected)"}
    return out


def guidance_map_leg(w, M, pk, reps=5):
    """The guidance map producer (prism_av_norm) on the layer's video grid: one
    launch over all heads of the audio-to-video cross-attention (4 N M D flops per
    head), timed alone with CUDA events on the launching stream, with h_hat
    written in bf16 (the fused producer of a model) and with the map alone."""
    import torch
    from dynamic_block_sparse_indicator_b200 import _lib
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    Qv, Ka, Va = syn.make_av_inputs(w, M, device="cuda")
    heads, N, D = Qv.shape
    amap = torch.empty(N, dtype=torch.float32, device="cuda")
    hh = torch.empty(heads, N, D, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    flops = 4.0 * N * M * D * heads
    burst = pk.get("bf16_tflops") or 1590.0
    sust = pk.get("bf16_tflops_sustained") or 1400.0
    out = {"workload": f"grid{w.T}x{w.H}x{w.W} ({N} video tokens), {M} audio tokens, {heads} heads, "
                       f"head_dim {D}, bf16 inputs", "flops": flops, "launches_per_call": 1}
    for name, hbuf in (("with_hhat_bf16", hh), ("map_only", None)):
        for _ in range(2):
            _lib.av_norm(Qv, Ka, Va, a_map=amap, h_hat=hbuf, status=status)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            _lib.av_norm(Qv, Ka, Va, a_map=amap, h_hat=hbuf, status=status)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        tf = flops / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "frac_of_burst": tf / burst, "frac_of_sustained": tf / sust}
    st, site = _lib.status_read(status)
    if st:
        raise RuntimeError(f"guidance map: device status {_lib.status_string(st)} at site {site}")
    ach = out["with_hhat_bf16"]["tflops"]
    out["roofline"] = {"kernel": "k_av_norm", "bound": "tensor", "achieved": ach, "peak": burst,
                       "unit": "TFLOP/s", "frac": ach / burst,
                       "peak_source": "measured burst bf16 (timed alone)" if pk else "fallback",
                       "traffic": None, "traffic_note": "no DRAM capture of this kernel"}
    del Qv, Ka, Va, amap, hh
    torch.cuda.empty_cache()
    return out


def run_sweep(a):
    """The 2K inference sweep (workload 4: grid 64x88x152, 856,064 tokens, head_dim 128,
    bf16, forward only), one head per point: plan + forward timed with CUDA events
    (1 warm-up, `--steps` timed), TFLOP/s = 4 D Pi / forward time, mean selected
    blocks per query block.  Prints one JSON line with every point."""
    import numpy as np
    import torch
    from dynamic_block_sparse_indicator_b200 import _lib
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    pk = peaks()
    peak = pk.get("bf16_tflops_sustained") or 1400.0
    points = []
    for regime, scale in (("peaked", 3.0), ("diffuse", 0.5)):
        w0 = syn.workload(4, qk_scale=scale)
        Q, K, V = syn.make_qkv(w0, device="cuda", heads=1)
        amap = syn.make_amap(w0, device="cuda")
        for k in (8, 16, 32):
            for p in (0.8, 0.9, 0.95):
                params = _lib.make_params(w0.T, w0.H, w0.W, 1, w0.head_dim, _lib.PRISM_BF16, k, p, w0.eps,
                                          out_dtype=_lib.PRISM_F32)
                pl = _lib.plan(Q, K, V, amap, params)
                O, lse = pl.attn_fwd()
                torch.cuda.synchronize()
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                tp, tf = 0.0, 0.0
                for _ in range(a.steps):
                    ev[0].record()
                    pl = _lib.plan(Q, K, V, amap, params)
                    ev[1].record()
                    pl.attn_fwd(O, lse)
                    ev[2].record()
                    torch.cuda.synchronize()
                    tp += ev[0].elapsed_time(ev[1])
                    tf += ev[1].elapsed_time(ev[2])
                st = pl.status()
                if st:
                    raise RuntimeError(f"device status: {_lib.status_string(st)}")
                Pi, nb, sel = selected_pairs(pl)
                fwd_ms = tf / a.steps
                tfl = 4.0 * w0.head_dim * Pi / (fwd_ms * 1e-3) / 1e12
                points.append({"regime": regime, "top_k": k, "top_p": p, "plan_ms": tp / a.steps,
                               "fwd_ms": fwd_ms, "ms_per_head_layer": tp / a.steps + fwd_ms,
                               "tflops": tfl, "fraction_of_sustained": tfl / peak,
                               "blocks_per_head": nb, "mean_selected_blocks": sel,
                               "pair_density": Pi / float(w0.N) ** 2})
        del Q, K, V
        torch.cuda.empty_cache()
    emit({"mode": "sweep", "metric": "Prism sparse-attn forward ms/head-layer, 2K inference sweep",
          "unit": "ms/head-layer", "higher_is_better": False, "data": "synthetic", "steps": a.steps,
          "config": {"workload": "grid64x88x152_h1_d128_bf16", "tokens": 856064, "head_dim": 128},
          "peak_tflops": peak, "sweep": points})


def run_prism(a, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from dynamic_block_sparse_indicator_b200 import _lib
    from dynamic_block_sparse_indicator_b200 import synthetic as syn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload_of(a)
    mode = {"dynamic": _lib.PRISM_SHAPE_DYNAMIC, "isotropic": _lib.PRISM_SHAPE_ISOTROPIC,
            "fixed": _lib.PRISM_SHAPE_FIXED}[a.shape_mode]
    variant = dict(alpha=a.alpha, shape_mode=mode, fixed_shape=a.fixed_shape, top_k_frac=a.topk_frac,
                   cut_ratio=a.cut_ratio)
    lib = _lib.load()
    need = a.warmup + a.steps
    heads = min(w.heads, need)
    # this rank's heads: offsets by rank, so ranks work on different heads
    order = head_order(rank, world, need, w.heads)
    gen_heads = max(order) + 1
    Q, K, V = syn.make_qkv(w, device=dev, heads=gen_heads)
    dO = syn.make_dout(w, device=dev, heads=gen_heads, out_dtype=torch.bfloat16).float()
    amap = syn.make_amap(w, device=dev)
    params = _lib.make_params(w.T, w.H, w.W, 1, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p,
                              w.eps, out_dtype=_lib.PRISM_F32, **variant)
    ws = torch.empty(_lib.workspace_bytes(params), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    O = torch.empty(1, w.N, w.head_dim, **f32)
    lse = torch.empty(1, w.N, **f32)
    dQ, dK, dV = (torch.empty(1, w.N, w.head_dim, **f32) for _ in range(3))

    def step(h, prof=False, pev=None):
        if pev is not None:
            pev[0].record()
        pl = _lib.plan(Q[h:h + 1], K[h:h + 1], V[h:h + 1], amap, params, workspace=ws)
        if pev is not None:
            pev[1].record()
        if prof:
            pl.profile(True)
        pl.attn_fwd(O, lse)
        pl.attn_bwd(dO[h:h + 1], O, lse, dQ, dK, dV)
        return pl

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for i in range(a.warmup):
        pl = step(order[i])
    barrier()
    st = pl.status()
    if st:
        raise RuntimeError(f"device status after warm-up: {_lib.status_string(st)}")
    del pl
    # ---------------------------------------------------------- timed region
    stage_ms = {k: 0.0 for k in _lib.Plan.STAGES}
    stage_n = {k: 0 for k in _lib.Plan.STAGES}
    plan_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(a.steps)]
    launches = 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    plans = []
    _lib.profile_plans(True)          # the timed plans also time their own kernels
    with ClockSampler(local_rank) as clk:
        barrier()
        e0.record()
        for i in range(a.steps):
            pl = step(order[a.warmup + i], prof=True, pev=plan_ev[i])
            plans.append(pl)
        e1.record()
        barrier()
    _lib.profile_plans(False)
    clocks = clk.summary()
    elapsed = e0.elapsed_time(e1)
    elapsed_max = max_over_ranks(elapsed, world, dev)
    for pl in plans:
        for k, (ms, n) in pl.profile_read().items():
            stage_ms[k] += ms
            stage_n[k] += n
        launches += pl.launches()
        st = pl.status()
        if st:
            raise RuntimeError(f"device status: {_lib.status_string(st)}")
    plan_ms = sum(a_.elapsed_time(b_) for a_, b_ in plan_ev)
    del plans, pl
    # selected pairs of the timed heads (plans are deterministic: re-plan, untimed)
    pis = []
    for i in range(a.steps):
        h = order[a.warmup + i]
        pl = _lib.plan(Q[h:h + 1], K[h:h + 1], V[h:h + 1], amap, params, workspace=ws)
        pis.append(selected_pairs(pl))
        del pl
    Pi = float(np.mean([p[0] for p in pis]))
    nb_mean = float(np.mean([p[1] for p in pis]))
    sel_mean = float(np.mean([p[2] for p in pis]))
    D = w.head_dim
    # head_dim 128 folds dQ into the dK/dV kernel (10 D Pi there, the dQ stage is a
    # scatter); head_dim 64 keeps a separate dQ kernel (8 D Pi + 2 D Pi)
    fused = D == 128
    flops = {"fwd": 4 * D * Pi, "bwd_dkdv": (10 if fused else 8) * D * Pi,
             "bwd_dq": 0.0 if fused else 2 * D * Pi}
    pk = peaks()
    peak = pk.get("bf16_tflops_sustained") or 1400.0
    peak_src = "measured sustained bf16 (fp16 operands, same kind::f16 rate)" if pk else "fallback"
    per_launch = {k: stage_ms[k] / max(stage_n[k], 1) for k in stage_ms}
    dom = max(("fwd", "bwd_dkdv", "bwd_dq"), key=lambda k: stage_ms[k])
    ach = flops[dom] / (per_launch[dom] * 1e-3) / 1e12
    attn_ms = (stage_ms["fwd"] + stage_ms["bwd_pre"] + stage_ms["bwd_dkdv"] + stage_ms["bwd_dq"]) / a.steps
    attn_tflops = 14 * D * Pi / (attn_ms * 1e-3) / 1e12
    value = elapsed_max / (a.steps * world)
    # plan kernels against their own bounds: HBM for the statistics (one read of
    # V) and the gather stage (Q, K, V read once for the per-head power-of-two
    # scales, then read again and written as the scaled fp16 copies); plain ALU
    # for the block scores (2 D N_b^2 flops + N_b^2 exp)
    hbm = pk.get("hbm_gbs") or 6650.0
    per_head = lambda k: stage_ms[k] / a.steps
    stats_bytes = 2.0 * D * w.N + 4.0 * w.N
    gather_bytes = 18.0 * D * w.N
    plan_kernels = {
        "stats": {"ms": per_head("plan_stats"), "bytes": stats_bytes,
                  "GB/s": stats_bytes / (per_head("plan_stats") * 1e-3) / 1e9 if per_head("plan_stats") else None},
        "shapes": {"ms": per_head("plan_shapes")},
        "gather": {"ms": per_head("plan_gather"), "bytes": gather_bytes,
                   "GB/s": gather_bytes / (per_head("plan_gather") * 1e-3) / 1e9 if per_head("plan_gather") else None},
        "select": {"ms": per_head("plan_select"), "flops": 2.0 * D * nb_mean ** 2, "exp": nb_mean ** 2,
                   "GFLOP/s": 2.0 * D * nb_mean ** 2 / (per_head("plan_select") * 1e-3) / 1e9
                   if per_head("plan_select") else None},
        "lists": {"ms": per_head("plan_lists")},
        "hbm_peak_GB/s": hbm, "peak_source": "measured" if pk.get("hbm_gbs") else "fallback",
    }
    # ------------------------------------------------- the pages' operating point
    op = None
    if world == 1 and not a.no_op:
        op = operating_point_leg(Q, K, V, dO, amap, w, order[a.warmup], peak)
    # ------------------------------------------- dense attention of the same shape
    dense = None
    if world == 1 and not a.no_dense:
        dense = dense_same_shape(Q, K, V, dO, amap, w, ws, O, lse, dQ, dK, dV, order[a.warmup], peak)
    # ------------------------------------- guidance map producer (next layer's a)
    av = None
    if world == 1 and not a.no_av:
        av = guidance_map_leg(w, a.av_tokens, pk)
    # --------------------------------------------------- end to end (host)
    # Through the C ABI from pinned host buffers: every step copies its inputs
    # (Q, K, V, dO, the map) to the device and reads its results (O, LSE, dQ, dK,
    # dV) back.  The copies run on a side stream against two device buffer sets,
    # so step i + 1's upload and step i's download overlap step i's kernels; the
    # timed region runs from before the first upload to after the last download.
    e2e = None
    if a.e2e_steps > 0:
        pin = lambda t: t.cpu().pin_memory()
        hin = dict(q=pin(Q[:1]), k=pin(K[:1]), v=pin(V[:1]), do=pin(dO[:1]), a=pin(amap))
        f32 = dict(dtype=torch.float32, device=dev)
        din = [{k_: torch.empty_like(v_, device=dev) for k_, v_ in hin.items()} for _ in range(2)]
        dout = [dict(O=torch.empty(1, w.N, D, **f32), lse=torch.empty(1, w.N, **f32),
                     dQ=torch.empty(1, w.N, D, **f32), dK=torch.empty(1, w.N, D, **f32),
                     dV=torch.empty(1, w.N, D, **f32)) for _ in range(2)]
        hout = [{k_: torch.empty(tuple(v_.shape), dtype=v_.dtype).pin_memory() for k_, v_ in dout[0].items()}
                for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for x in hin.values())
        d2h = sum(x.numel() * x.element_size() for x in hout[0].values())
        main, cs = torch.cuda.current_stream(), torch.cuda.Stream()
        up = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        down = [torch.cuda.Event() for _ in range(2)]

        def upload(b):
            with torch.cuda.stream(cs):
                for k_, v_ in hin.items():
                    din[b][k_].copy_(v_, non_blocking=True)
                up[b].record(cs)

        barrier()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(main)
        cs.wait_event(x0)
        upload(0)
        for i in range(a.e2e_steps):
            b = i & 1
            main.wait_event(up[b])
            if i >= 2:
                main.wait_event(down[b])          # step i - 2's results have been read back
            d, o = din[b], dout[b]
            pl = _lib.plan(d["q"], d["k"], d["v"], d["a"], params, workspace=ws)
            pl.attn_fwd(o["O"], o["lse"])
            pl.attn_bwd(d["do"], o["O"], o["lse"], o["dQ"], o["dK"], o["dV"])
            done[b].record(main)
            if i + 1 < a.e2e_steps:
                if i >= 1:
                    cs.wait_event(done[b ^ 1])    # step i - 1 has finished with that input set
                upload(b ^ 1)
            with torch.cuda.stream(cs):
                cs.wait_event(done[b])
                for k_, v_ in o.items():
                    hout[b][k_].copy_(v_, non_blocking=True)
                down[b].record(cs)
        main.wait_stream(cs)
        x1.record(main)
        barrier()
        st = pl.status()
        if st:
            raise RuntimeError(f"device status (end to end): {_lib.status_string(st)}")
        te = max_over_ranks(x0.elapsed_time(x1), world, dev)
        e2e = {"value": te / (a.e2e_steps * world), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "copies": "side stream, two device buffer sets: uploads and downloads overlap the kernels"}
        del din, dout, hout, hin
    # --------------------------------------------------- CPU oracle baseline
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        h = order[a.warmup]
        host = lambda t: t[h].to("cpu", torch.float64).numpy()
        ms, desc, threads = oracle_head_ms(host(Q), host(K), host(V), host(dO),
                                           amap.cpu().numpy(), w, a.cpu_seconds, variant=variant_of(a))
        cpu = {"value": ms, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
        try:                                      # the same on one core
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                ms1, desc1, _ = oracle_head_ms(host(Q), host(K), host(V), host(dO), amap.cpu().numpy(), w,
                                               a.cpu_seconds / 2, variant=variant_of(a))
            cpu["single_core"] = {"value": ms1, "unit": UNIT, "cores": 1, "sample": desc1}
        except ImportError:
            cpu["single_core"] = None
    if rank == 0:
        emit({"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
              "warmup": a.warmup, "ms_per_step": elapsed_max / a.steps, "higher_is_better": False,
              "scaling": "weak", "vs_baseline": None, "dtype": "fp16-operand tensor cores, fp32 accumulate",
              "data": "synthetic",
              "config": {"workload": w.name(), "grid": [w.T, w.H, w.W], "tokens": w.N,
                         "heads_in_sequence": True, "head_dim": D, "input_dtype": "bf16",
                         "output_dtype": "fp32", "top_k": w.top_k, "top_p": w.top_p,
                         "top_k_frac": a.topk_frac, "alpha": a.alpha, "shape_mode": a.shape_mode,
                         **({"cut_ratio": a.cut_ratio, "shot_cuts": list(a.shot_cuts)} if a.cut_ratio else {}),
                         **({"fixed_shape": a.fixed_shape} if a.shape_mode == "fixed" else {}),
                         "l2": "inputs larger than L2 (259 MB per tensor per head)"},
              "tflops": {"fwd_bwd_selected": attn_tflops,
                         "fraction_of_peak": attn_tflops / peak},
              "stages_ms_per_head": {"plan": plan_ms / a.steps,
                                     **{k: stage_ms[k] / a.steps for k in stage_ms}},
              "plan_stats": {"blocks_per_head": nb_mean, "mean_selected_blocks": sel_mean,
                             "selected_pairs": Pi, "pair_density": Pi / float(w.N) ** 2},
              "roofline": {"kernel": {"fwd": "k_attn_fwd", "bwd_dkdv": "k_bwd_dkdv",
                                      "bwd_dq": "k_dq_finalize" if fused else "k_bwd_dq"}[dom],
                           "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                           "frac": ach / peak, "peak_source": peak_src,
                           "traffic": measured_traffic(
                               {"fwd": "k_attn_fwd", "bwd_dkdv": "k_bwd_dkdv"}.get(dom, ""), Pi),
                           "traffic_note": "DRAM bytes per launch from a one-launch ncu capture on a small "
                                           "grid, scaled by selected pairs (profiles/" + TRAFFIC_PROFILE
                                           + "); null once the kernel changed since"},
              "plan_kernels": plan_kernels, "dense_same_shape": dense, "operating_point": op,
              "guidance_map": av,
              "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": launches, "clocks": clocks})


def main():
    a = args_()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank, world)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=600))
    try:
        if a.sweep:
            if rank == 0:
                run_sweep(a)
            return
        run_prism(a, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
