"""Seeded synthetic inputs for Prism's video self-attention workloads.

This module only draws inputs: Gaussian-smoothed random value fields, the
localised "fast-varying" zones, the audio-to-video cross-attention norm map
and the output gradient.  It holds none of the method's arithmetic, so both
the CUDA path and the CPU oracle can be fed from it.

Workloads (grid T x H x W, heads, head_dim, dtype, top-k, top-p, eps):

  0  8 x 16 x 16      (2,048 tokens),   2 heads, D=64,  fp32, k=4,  p=0.9, eps=1e-6
  1  24 x 48 x 80     (92,160 tokens),  40 heads, D=128, bf16, k=8,  p=0.9, eps=1e-4
  2  32 x 72 x 128    (294,912 tokens), 40 heads, D=128, bf16, k=16, p=0.9, eps=1e-4
  3  72 x 88 x 160    (1,013,760 tokens), 40 heads, D=128, bf16, k=16, p=0.9, eps=1e-4
  4  64 x 88 x 152    (856,064 tokens), 40 heads, D=128, bf16, forward sweep

Recipe for one tensor (Q, K or V), per head and channel:
  * white N(0,1) noise on the T x H x W grid, smoothed by a separable Gaussian
    (sigma = 3 tokens, radius 9, replicate padding at the grid edges), then
    divided by its own standard deviation;
  * plus N(0, 0.3^2) noise;
  * inside each localised zone an extra N(0,1) component per channel that
    varies along one axis only: per frame ("T-fast"), per row ("H-fast") or
    per column ("W-fast"), constant over the other two axes of the zone;
  * for the 2K workloads, 85 % of the zones (chosen by seed, never a
    localised one) are near-uniform: the smoothed field is scaled by 0.1 and
    the noise standard deviation is 0.03.
Inputs of the audio-to-video cross-attention that produces the norm map
(make_av_inputs): the video queries Qv are a further tensor of the recipe
above (seed id 5); the audio keys and values Ka, Va [heads, M, D] are, per head
and channel, white N(0,1) noise over the M audio tokens smoothed by a 1-D
Gaussian (sigma 3 tokens, radius 9, replicate padding), divided by its std,
plus N(0, 0.3^2) (seed ids 6 and 7).
Shot cuts (optional, `shot_cuts`): from each listed frame on, the recipe's field
is replaced by a fresh draw (a new shot); local cuts (`local_cuts`, (zt, zh, zw,
local frame)): the same inside one zone from a local frame on.
The audio norm map is 0.05 everywhere, raised to a Gaussian blob
0.05 + 0.95 exp(-|x - c|^2 / (2 * 3^2)) around the centre c of every localised
zone (blobs combine by max).  dO is N(0,1).  Seeds: workload id x 1000 +
tensor id (Q=0, K=1, V=2, dO=3, zone choice=4).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass
class Workload:
    wid: int
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    dtype: str  # "f32" or "bf16"
    top_k: int
    top_p: float
    eps: float
    n_tfast: int = 0
    n_hfast: int = 0
    n_wfast: int = 0
    uniform_frac: float = 0.0
    qk_scale: float = 1.0
    fixed_zones: list = field(default_factory=list)  # explicit (zt, zh, zw, axis)
    shot_cuts: list = field(default_factory=list)    # global frames where a new shot starts
    local_cuts: list = field(default_factory=list)   # (zt, zh, zw, local frame): a zone changes content

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def zones(self) -> int:
        return (self.T // 8) * (self.H // 8) * (self.W // 8)

    def name(self) -> str:
        return (f"grid{self.T}x{self.H}x{self.W}_h{self.heads}_d{self.head_dim}_"
                f"{self.dtype}_k{self.top_k}_p{self.top_p}")


def workload(wid: int, **over) -> Workload:
    """The five workloads of the hot path (see the module docstring)."""
    if wid == 0:
        w = Workload(0, 8, 16, 16, 2, 64, "f32", 4, 0.9, 1e-6,
                     fixed_zones=[(0, 1, 1, 0)])
    elif wid == 1:
        w = Workload(1, 24, 48, 80, 40, 128, "bf16", 8, 0.9, 1e-4, n_tfast=6)
    elif wid == 2:
        w = Workload(2, 32, 72, 128, 40, 128, "bf16", 16, 0.9, 1e-4,
                     n_tfast=4, n_hfast=4, n_wfast=4)
    elif wid == 3:
        w = Workload(3, 72, 88, 160, 40, 128, "bf16", 16, 0.9, 1e-4,
                     n_tfast=12, n_hfast=6, n_wfast=6, uniform_frac=0.85)
    elif wid == 4:
        w = Workload(4, 64, 88, 152, 40, 128, "bf16", 16, 0.9, 1e-4,
                     n_tfast=12, n_hfast=6, n_wfast=6, uniform_frac=0.85)
    else:
        raise ValueError(f"unknown workload {wid}")
    for k, v in over.items():
        setattr(w, k, v)
    return w


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zone_layout(w: Workload, device="cpu"):
    """Localised zones [(zt, zh, zw, axis)] and a bool mask [Nz] of near-uniform zones."""
    zt_n, zh_n, zw_n = w.T // 8, w.H // 8, w.W // 8
    nz = zt_n * zh_n * zw_n
    if w.fixed_zones:
        loc = list(w.fixed_zones)
        uniform = torch.zeros(nz, dtype=torch.bool)
        return loc, uniform
    g = _gen(w.wid * 1000 + 4, "cpu")
    order = torch.randperm(nz, generator=g).tolist()
    axes = [0] * w.n_tfast + [1] * w.n_hfast + [2] * w.n_wfast
    loc = []
    for z, ax in zip(order[: len(axes)], axes):
        zt, rem = divmod(z, zh_n * zw_n)
        zh, zw = divmod(rem, zw_n)
        loc.append((zt, zh, zw, ax))
    uniform = torch.zeros(nz, dtype=torch.bool)
    n_uni = int(round(w.uniform_frac * nz))
    if n_uni:
        uniform[torch.tensor(order[len(axes): len(axes) + n_uni], dtype=torch.long)] = True
    return loc, uniform


def _blur_axis(x: torch.Tensor, dim: int, taps: torch.Tensor) -> torch.Tensor:
    r = (taps.numel() - 1) // 2
    xt = x.movedim(dim, -1)
    shp = xt.shape
    y = xt.reshape(-1, 1, shp[-1])
    y = F.pad(y, (r, r), mode="replicate")
    y = F.conv1d(y, taps.view(1, 1, -1))
    return y.reshape(shp).movedim(-1, dim)


def _base_field(w: Workload, g: torch.Generator, uniform_tok, device) -> torch.Tensor:
    """Smoothed unit-std field plus noise (near-uniform zones damped): [D, T, H, W]."""
    D, T, H, W = w.head_dim, w.T, w.H, w.W
    sigma, radius = 3.0, 9
    k = torch.arange(-radius, radius + 1, dtype=torch.float32, device=device)
    taps = torch.exp(-(k * k) / (2 * sigma * sigma))
    taps = taps / taps.sum()
    x = torch.randn(D, T, H, W, generator=g, device=device)
    for dim in (1, 2, 3):
        x = _blur_axis(x, dim, taps)
    x = x / x.flatten(1).std(dim=1).clamp_min(1e-12).view(D, 1, 1, 1)
    noise = torch.randn(D, T, H, W, generator=g, device=device)
    if uniform_tok is not None:
        u = uniform_tok.view(1, T, H, W)
        return torch.where(u, x * 0.1, x) + torch.where(u, noise * 0.03, noise * 0.3)
    return x + 0.3 * noise


def _field_one_head(w: Workload, g: torch.Generator, loc, uniform_tok, device) -> torch.Tensor:
    """One head of one tensor: [N, D] float32 in raster token order.

    Shot cuts: from each cut frame on, every frame is a fresh draw of the base
    field (a new shot).  Local cuts: inside one zone, from a local frame on, the
    tokens are a fresh draw (content that changes abruptly in one region, as in
    a fast zoom)."""
    D, T, H, W = w.head_dim, w.T, w.H, w.W
    x = _base_field(w, g, uniform_tok, device)
    for c in sorted(w.shot_cuts):
        x[:, c:] = _base_field(w, g, uniform_tok, device)[:, c:]
    for (zt, zh, zw, tl) in w.local_cuts:
        y = _base_field(w, g, uniform_tok, device)
        sl = (slice(None), slice(8 * zt + tl, 8 * zt + 8), slice(8 * zh, 8 * zh + 8), slice(8 * zw, 8 * zw + 8))
        x[sl] = y[sl]
    for (zt, zh, zw, ax) in loc:
        comp = torch.randn(D, 8, generator=g, device=device)
        sl = (slice(None), slice(8 * zt, 8 * zt + 8), slice(8 * zh, 8 * zh + 8),
              slice(8 * zw, 8 * zw + 8))
        if ax == 0:
            x[sl] += comp.view(D, 8, 1, 1)
        elif ax == 1:
            x[sl] += comp.view(D, 1, 8, 1)
        else:
            x[sl] += comp.view(D, 1, 1, 8)
    return x.permute(1, 2, 3, 0).reshape(T * H * W, D)


def _uniform_tokens(w: Workload, uniform: torch.Tensor, device):
    if not bool(uniform.any()):
        return None
    zt_n, zh_n, zw_n = w.T // 8, w.H // 8, w.W // 8
    u = uniform.view(zt_n, 1, zh_n, 1, zw_n, 1).expand(zt_n, 8, zh_n, 8, zw_n, 8)
    return u.reshape(w.T, w.H, w.W).to(device)


def make_qkv(w: Workload, device="cpu", heads=None, out_dtype=None):
    """Q, K, V as [heads, N, D] tensors (float32 or bfloat16, per the workload)."""
    heads = w.heads if heads is None else heads
    dt = out_dtype or (torch.float32 if w.dtype == "f32" else torch.bfloat16)
    loc, uniform = zone_layout(w)
    utok = _uniform_tokens(w, uniform, device)
    out = []
    for tid in range(3):
        g = _gen(w.wid * 1000 + tid, device)
        t = torch.empty(heads, w.N, w.head_dim, dtype=dt, device=device)
        for h in range(heads):
            f = _field_one_head(w, g, loc, utok, device)
            if tid < 2 and w.qk_scale != 1.0:
                f = f * w.qk_scale
            t[h] = f.to(dt)
        out.append(t)
    return tuple(out)


def make_amap(w: Workload, device="cpu") -> torch.Tensor:
    """Audio-to-video cross-attention norm map a [T, H, W] float32."""
    loc, _ = zone_layout(w)
    t = torch.arange(w.T, dtype=torch.float32, device=device).view(-1, 1, 1)
    h = torch.arange(w.H, dtype=torch.float32, device=device).view(1, -1, 1)
    x = torch.arange(w.W, dtype=torch.float32, device=device).view(1, 1, -1)
    a = torch.full((w.T, w.H, w.W), 0.05, dtype=torch.float32, device=device)
    for (zt, zh, zw, _ax) in loc:
        ct, ch, cw = 8 * zt + 3.5, 8 * zh + 3.5, 8 * zw + 3.5
        d2 = (t - ct) ** 2 + (h - ch) ** 2 + (x - cw) ** 2
        a = torch.maximum(a, 0.05 + 0.95 * torch.exp(-d2 / (2 * 3.0 ** 2)))
    return a


def make_dout(w: Workload, device="cpu", heads=None, out_dtype=None) -> torch.Tensor:
    heads = w.heads if heads is None else heads
    dt = out_dtype or (torch.float32 if w.dtype == "f32" else torch.bfloat16)
    g = _gen(w.wid * 1000 + 3, device)
    t = torch.empty(heads, w.N, w.head_dim, dtype=dt, device=device)
    for h in range(heads):
        t[h] = torch.randn(w.N, w.head_dim, generator=g, device=device).to(dt)
    return t


def make_av_inputs(w: Workload, M: int, device="cpu", heads=None, out_dtype=torch.bfloat16,
                   qk_scale: float = 1.0):
    """Qv [heads, N, D], Ka, Va [heads, M, D] for the norm-map producer (bf16 by default)."""
    heads = w.heads if heads is None else heads
    loc, uniform = zone_layout(w)
    utok = _uniform_tokens(w, uniform, device)
    g = _gen(w.wid * 1000 + 5, device)
    Qv = torch.empty(heads, w.N, w.head_dim, dtype=out_dtype, device=device)
    for h in range(heads):
        Qv[h] = (_field_one_head(w, g, loc, utok, device) * qk_scale).to(out_dtype)
    sigma, radius = 3.0, 9
    k = torch.arange(-radius, radius + 1, dtype=torch.float32, device=device)
    taps = torch.exp(-(k * k) / (2 * sigma * sigma))
    taps = taps / taps.sum()
    out = []
    for tid in (6, 7):
        ga = _gen(w.wid * 1000 + tid, device)
        x = torch.randn(heads, w.head_dim, M, generator=ga, device=device)
        x = _blur_axis(x, 2, taps)
        x = x / x.std(dim=2, keepdim=True).clamp_min(1e-12) if M > 1 else x
        x = x + 0.3 * torch.randn(heads, w.head_dim, M, generator=ga, device=device)
        if tid == 6 and qk_scale != 1.0:
            x = x * qk_scale
        out.append(x.transpose(1, 2).contiguous().to(out_dtype))
    return Qv, out[0], out[1]


def roundtrip_float(t: torch.Tensor):
    """Exact float64 numpy copy of a tensor's values (bf16 values are exact in f64)."""
    return t.detach().to("cpu", torch.float64).numpy()


__all__ = ["Workload", "workload", "zone_layout", "make_qkv", "make_amap", "make_dout", "make_av_inputs",
           "roundtrip_float"]

