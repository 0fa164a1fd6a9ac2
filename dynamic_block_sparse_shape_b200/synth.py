"""Seeded synthetic inputs shaped like the Prism workloads.

This module only draws numbers: smooth sinusoid fields over the (t, h, w)
token grid, Gaussian noise, per-zone anisotropic oscillations for the video
features, and Gaussian "sound-source" blobs for the a2v residual norm. It holds
none of the method's arithmetic (no zone statistics, pooling, scoring,
selection or attention), so the CPU oracle and the CUDA path can both take
their inputs from it.

Every generator takes a ``torch.Generator`` and a device; the same seed and
device give the same tensors. Token order is raster (t, h, w): token id
``n = (t * H + h) * W + w``. Q/K/V are ``[N, heads, head_dim]``; features and
residuals are ``[N, C]``.

Workloads (sizes from the Prism pages: 720p / 1080p / 2K joint video-audio
training, 24 heads of width 128, 3072-wide hidden states):

* ``tiny``: grid 4x8x8, 2 heads, d=64, fp32, N(0,1) + one sinusoid per channel.
* ``720p``: grid 16x48x80, 24 heads, d=128, bf16, Q/K = 8 sinusoids + noise.
* ``1080p``: grid 16x72x128, plus video features and an a2v residual.
* ``2k``: grid 32x72x128, the 1080p recipe on the 2K latent grid.
* ``720p-latent`` / ``2k-latent``: grids 16x45x80 and 32x90x160, the real
  latent sizes of 720p and 2K frames, whose 45 / 90 rows are not a whole
  number of 8-token zones; the 1080p recipe otherwise.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

TWO_PI = 2.0 * math.pi


@dataclass(frozen=True)
class Workload:
    name: str
    grid: tuple  # (T, H, W) latent token grid
    heads: int
    head_dim: int
    dtype: str  # "bf16" or "fp32"
    zone: tuple  # (Zt, Zh, Zw)
    top_k: int
    cdf_threshold: float
    backward: bool
    features: str  # "none" | "q" | "synthetic"
    residual: bool
    amplitude: float = 1.0
    seed: int = 0
    shapes: str = "default"  # "default" candidate list, or "fixed444"
    extra: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        T, H, W = self.grid
        return T * H * W


WORKLOADS = {
    "tiny": Workload("tiny", (4, 8, 8), 2, 64, "fp32", (4, 8, 8), 1, 0.20, True, "none", False, seed=0,
                     shapes="fixed444"),
    "720p": Workload("720p", (16, 48, 80), 24, 128, "bf16", (8, 8, 8), 4, 0.20, False, "q", False, seed=1),
    "1080p": Workload("1080p", (16, 72, 128), 24, 128, "bf16", (8, 8, 8), 4, 0.20, False, "synthetic", True,
                      seed=2),
    "2k": Workload("2k", (32, 72, 128), 24, 128, "bf16", (8, 8, 8), 4, 0.20, True, "synthetic", True, seed=3),
    # the 2K grid with 2 heads and Q as the feature input: every attention tensor (151 MB) is still
    # larger than L2, and the whole working set (~1.3 GB) is small enough for profiler captures
    "2k-2h": Workload("2k-2h", (32, 72, 128), 2, 128, "bf16", (8, 8, 8), 4, 0.20, True, "q", False, seed=3),
    # the 2K grid with the full video features and a2v residual ([N, 3072] bf16 each, as in the 2K
    # training step) but 2 heads: the zone statistics stream their full 2K inputs while the whole
    # working set (~4.8 GB) stays small enough for profiler captures of the selection path
    "2k-stats": Workload("2k-stats", (32, 72, 128), 2, 128, "bf16", (8, 8, 8), 4, 0.20, True, "synthetic", True,
                         seed=3),
    # the real VAE latent grids (16x spatial, 4x temporal downsampling): 720p gives 45 x 80 tokens per frame,
    # 2K (2560 x 1440) 90 x 160; 45 and 90 are not multiples of the 8-token zone, so the last zone row is clipped
    "720p-latent": Workload("720p-latent", (16, 45, 80), 24, 128, "bf16", (8, 8, 8), 4, 0.20, True, "synthetic",
                            True, seed=5),
    "2k-latent": Workload("2k-latent", (32, 90, 160), 24, 128, "bf16", (8, 8, 8), 4, 0.20, True, "synthetic", True,
                          seed=6),
}


def sweep_workloads():
    """The 45-point selection/sparsity sweep on the 2K grid."""
    out = []
    for amp in (0.25, 1.0, 4.0):
        for k in (1, 4, 16):
            for tau in (0.05, 0.10, 0.20, 0.40, 1.0):
                out.append(Workload(f"2k-sweep-a{amp}-k{k}-t{tau}", (32, 72, 128), 24, 128, "bf16", (8, 8, 8), k,
                                    tau, True, "synthetic", True, amplitude=amp, seed=4))
    return out


def make_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _axes(grid, device):
    T, H, W = grid
    t = torch.arange(T, device=device, dtype=torch.float32) / T
    h = torch.arange(H, device=device, dtype=torch.float32) / H
    w = torch.arange(W, device=device, dtype=torch.float32) / W
    return t, h, w


def sinusoid_field(grid, channels, n_terms, amplitude, fmax, gen, device, out=None):
    """Sum over ``n_terms`` of (amplitude/sqrt(n_terms)) * sin(2 pi f.x + phi) per channel.

    x = (t/T, h/H, w/W); f has independent integer components in [0, fmax]; phi
    is uniform in [0, 2 pi). Returns fp32 ``[T*H*W, channels]`` (added into
    ``out`` when given).
    """
    T, H, W = grid
    freqs = torch.randint(0, fmax + 1, (n_terms, channels, 3), generator=gen, device=device).float()
    phase = torch.rand((n_terms, channels), generator=gen, device=device) * TWO_PI
    t, h, w = _axes(grid, device)
    if out is None:
        out = torch.zeros((T, H, W, channels), device=device, dtype=torch.float32)
    else:
        out = out.view(T, H, W, channels)
    a = amplitude / math.sqrt(n_terms)
    for i in range(n_terms):
        pt = TWO_PI * t[:, None] * freqs[i, :, 0][None, :] + phase[i][None, :]  # [T, C]
        ph = TWO_PI * h[:, None] * freqs[i, :, 1][None, :]  # [H, C]
        pw = TWO_PI * w[:, None] * freqs[i, :, 2][None, :]  # [W, C]
        for ti in range(T):  # one time slice at a time keeps temporaries small
            arg = pt[ti][None, None, :] + ph[:, None, :] + pw[None, :, :]
            out[ti].add_(torch.sin(arg), alpha=a)
    return out.view(T * H * W, channels)


def qkv(wl: Workload, device="cpu", dtype=None):
    """Q, K, V (and dO when the workload has a backward) for a workload."""
    gen = make_generator(wl.seed, device)
    T, H, W = wl.grid
    N, C = wl.n_tokens, wl.heads * wl.head_dim
    tdt = dtype or (torch.float32 if wl.dtype == "fp32" else torch.bfloat16)
    out = {}
    if wl.name == "tiny":
        for name in ("q", "k", "v"):
            x = torch.randn((N, C), generator=gen, device=device)
            sinusoid_field(wl.grid, C, 1, 1.0, 2, gen, device, out=x)
            out[name] = x.view(N, wl.heads, wl.head_dim).to(tdt)
    else:
        for name in ("q", "k"):
            x = torch.randn((N, C), generator=gen, device=device).mul_(0.5)
            sinusoid_field(wl.grid, C, 8, wl.amplitude, 4, gen, device, out=x)
            out[name] = x.view(N, wl.heads, wl.head_dim).to(tdt)
            del x
        out["v"] = torch.randn((N, C), generator=gen, device=device).view(N, wl.heads, wl.head_dim).to(tdt)
    if wl.backward:
        out["do"] = torch.randn((N, C), generator=gen, device=device).view(N, wl.heads, wl.head_dim).to(tdt)
    return out


def video_features(wl: Workload, channels=3072, device="cpu", base_amplitude=0.5):
    """Video hidden states ``[N, channels]`` bf16 with per-zone anisotropy.

    A global 8-term sinusoid field (amplitude 1, frequencies up to 4 cycles per
    grid side) plus, in every zone, one oscillation per axis with a period of
    4 tokens and a random phase per (zone, axis, channel). Each zone draws a
    dominant axis and a ratio rho in {1, 2, 4}; the dominant axis's oscillation
    has amplitude rho * base_amplitude, the others base_amplitude.
    """
    gen = make_generator(1000 + wl.seed, device)
    T, H, W = wl.grid
    Zt, Zh, Zw = wl.zone
    # zones tile the grid rounded up (the last one per axis may be clipped)
    nt, nh, nw = -(-T // Zt), -(-H // Zh), -(-W // Zw)
    nz = nt * nh * nw
    x = sinusoid_field(wl.grid, channels, 8, 1.0, 4, gen, device)  # fp32 [N, C]
    dom = torch.randint(0, 3, (nz,), generator=gen, device=device)
    rho = torch.tensor([1.0, 2.0, 4.0], device=device)[torch.randint(0, 3, (nz,), generator=gen, device=device)]
    amp = torch.full((nz, 3), base_amplitude, device=device)
    amp[torch.arange(nz, device=device), dom] *= rho
    psi = torch.rand((nz, 3, channels), generator=gen, device=device) * TWO_PI
    x = x.view(T, H, W, channels)
    tt = torch.arange(T, device=device)
    hh = torch.arange(H, device=device)
    ww = torch.arange(W, device=device)
    for ti in range(T):
        zt = ti // Zt
        zh = hh // Zh  # [H]
        zw = ww // Zw  # [W]
        zid = (zt * nh + zh[:, None]) * nw + zw[None, :]  # [H, W]
        lt = float(ti % Zt)
        lh = (hh % Zh).float()[:, None].expand(H, W)
        lw = (ww % Zw).float()[None, :].expand(H, W)
        q = math.pi / 2.0
        comp = amp[zid, 0, None] * torch.sin(q * lt + psi[zid, 0])
        comp += amp[zid, 1, None] * torch.sin(q * lh[..., None] + psi[zid, 1])
        comp += amp[zid, 2, None] * torch.sin(q * lw[..., None] + psi[zid, 2])
        x[ti].add_(comp)
        del comp
    del tt
    return x.view(T * H * W, channels).to(torch.bfloat16)


def a2v_residual(wl: Workload, channels=3072, device="cpu", n_blobs=4, sigma=6.0, peak=5.0, floor_std=0.1):
    """A synthetic a2v bridge residual ``[N, channels]`` bf16.

    Per-token target norm = |N(0, floor_std^2)| + sum over ``n_blobs`` Gaussian
    blobs (std ``sigma`` tokens, height ``peak``) centred at uniform random
    (t, h, w) positions; each token's direction is uniform on the sphere.
    Also returns the blob centres.
    """
    gen = make_generator(2000 + wl.seed, device)
    T, H, W = wl.grid
    N = T * H * W
    centres = torch.rand((n_blobs, 3), generator=gen, device=device) * torch.tensor(
        [T, H, W], device=device, dtype=torch.float32)
    base = torch.randn((N,), generator=gen, device=device).mul_(floor_std).abs_()
    t = torch.arange(T, device=device, dtype=torch.float32)
    h = torch.arange(H, device=device, dtype=torch.float32)
    w = torch.arange(W, device=device, dtype=torch.float32)
    norm = base.view(T, H, W)
    for b in range(n_blobs):
        ct, ch, cw = centres[b]
        d2 = (t - ct)[:, None, None] ** 2 + (h - ch)[None, :, None] ** 2 + (w - cw)[None, None, :] ** 2
        norm = norm + peak * torch.exp(-d2 / (2.0 * sigma * sigma))
    norm = norm.reshape(N)
    out = torch.empty((N, channels), device=device, dtype=torch.bfloat16)
    chunk = 1 << 15
    for s in range(0, N, chunk):
        e = min(N, s + chunk)
        g = torch.randn((e - s, channels), generator=gen, device=device)
        g.mul_((norm[s:e] / g.norm(dim=1))[:, None])
        out[s:e] = g.to(torch.bfloat16)
    return out, centres


def candidates_for(wl: Workload):
    """Candidate (bt, bh, bw) shapes: the 10 power-of-two 64-token boxes that
    fit an 8x8x8 zone, or the single (4,4,4) of the fixed-shape workload."""
    if wl.shapes == "fixed444":
        return [(4, 4, 4)]
    return list(DEFAULT_CANDIDATES)


# The 10 boxes (2^a, 2^b, 2^c), a+b+c = 6, each exponent in 0..3, in a fixed
# order: isotropic first, the two shapes the Prism walkthrough names next.
DEFAULT_CANDIDATES = (
    (4, 4, 4), (8, 2, 4), (8, 4, 2), (4, 8, 2), (2, 8, 4), (2, 4, 8), (4, 2, 8), (1, 8, 8), (8, 1, 8), (8, 8, 1),
)
