"""Seeded synthetic inputs for the heterogeneous-attention path.

This module holds input generation only -- none of the method's arithmetic --
and is the one piece of code that both the CUDA path's callers and the fp64
oracle's callers share.  It depends on numpy/scipy only.

The paper measures on Wan2.1-1.3B (81x480x832 pixels) and Wan2.2-5B
(121x704x1280) latents ("Where Compute Matters: Heterogeneous Attention for
Efficient Video Diffusion", §4 Evaluation Setting; Table 5).  No model, prompt
or video is used here: the named workloads below stand in for them with the
latent-grid shapes those resolutions give, iid Gaussian Q/K/V and a seeded
uncertainty field.
"""
from dataclasses import dataclass, field, replace
from typing import Tuple

import numpy as np

# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: Tuple[int, int, int]          # (T, H, W) latent grid, token i = (t*H + h)*W + w
    win: Tuple[int, int, int]           # local window (wt, wh, ww), odd sizes
    rho: float                          # dense fraction per sample
    u_kind: str                         # "uniform" | "smooth" | "clustered"
    qkv_seed: int
    u_seeds: Tuple[int, ...]            # one seed per sample; () = continue the Q/K/V generator
    x_seed: int = 3                     # hidden states for the uncertainty head
    w_seed: int = 4                     # head weights
    C: int = 0                          # head input width (model dim)
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def M(self) -> int:
        a, b, c = self.win
        return a * b * c


TINY = Workload("tiny-4x8x8", B=1, H=2, d=64, grid=(4, 8, 8), win=(3, 3, 3),
                rho=0.25, u_kind="uniform", qkv_seed=0, u_seeds=(), C=128)
WAN21 = Workload("wan2.1-1.3b-21x30x52", B=1, H=12, d=128, grid=(21, 30, 52),
                 win=(3, 9, 9), rho=0.2, u_kind="smooth", qkv_seed=1,
                 u_seeds=(2,), C=1536)
WAN22 = Workload("wan2.2-5b-31x22x40", B=1, H=24, d=128, grid=(31, 22, 40),
                 win=(3, 9, 9), rho=0.2, u_kind="smooth", qkv_seed=1,
                 u_seeds=(2,), C=3072)
SWEEP_RHOS = (0.05, 0.1, 0.2, 0.35, 0.5)
BATCHED = Workload("wan2.1-1.3b-batched-b2", B=2, H=12, d=128,
                   grid=(21, 30, 52), win=(3, 9, 9), rho=0.2, u_kind="smooth",
                   qkv_seed=1, u_seeds=(5, 6), C=1536)
# The Wan2.1-1.3B layer at 720p (81 frames -> 21 latent frames, 720x1280 ->
# 45x80 after the 16x spatial compression and 2x2 patchify): N = 75600, the
# resolution at which the paper puts self-attention at 82% of compute.
WAN21_720P = Workload("wan2.1-1.3b-720p-21x45x80", B=1, H=12, d=128,
                      grid=(21, 45, 80), win=(3, 9, 9), rho=0.2, u_kind="smooth",
                      qkv_seed=1, u_seeds=(2,), C=1536)


def sweep(rho: float, u_kind: str) -> Workload:
    """The routing/load-balance sweep at the Wan2.1 shape."""
    assert u_kind in ("uniform", "clustered")
    return replace(WAN21, name="wan2.1-sweep-%s-rho%.2f" % (u_kind, rho),
                   rho=rho, u_kind=u_kind, u_seeds=(7,))


ALL = {w.name: w for w in (TINY, WAN21, WAN22, BATCHED, WAN21_720P)}

# the window sizes the paper's window ablation compares (its default 11^3,
# plus 9^3 and 13^3), at the Wan2.1 latent shape
WINDOW_CUBES = (9, 11, 13)


def window_cube(n: int) -> Workload:
    """The Wan2.1 workload with an n x n x n local window."""
    return replace(WAN21, name="wan2.1-1.3b-window%d" % n, win=(n, n, n))


def scaled(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (for tests that must finish in seconds)."""
    return replace(w, name=w.name + "-scaled", **kw)


# ---------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even on the bit pattern)
# ---------------------------------------------------------------------------


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the exactly equal fp32 values."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def make_qkv(w: Workload):
    """Q, K, V iid N(0,1) fp32, rounded to bf16: returns three uint16 [B,H,N,d]."""
    rng = _rng(w.qkv_seed)
    shape = (w.B, w.H, w.N, w.d)
    out = []
    for _ in range(3):
        out.append(bf16_bits(rng.standard_normal(shape, dtype=np.float32)))
    return tuple(out)


def _smooth_field(rng, grid, sigma=3.0, noise=0.1):
    from scipy.ndimage import gaussian_filter
    z = rng.standard_normal(grid)
    z = gaussian_filter(z, sigma=sigma, mode="reflect", truncate=4.0)
    z = (z - z.mean()) / z.std()
    z = z + rng.normal(0.0, noise, size=grid)
    return z.astype(np.float32).ravel()


def _clustered_field(rng, grid, nblobs=4, sigma=4.0, noise=0.01):
    T, H, W = grid
    c0 = rng.uniform([0.0, 0.0], [H - 1.0, W - 1.0], size=(nblobs, 2))
    vel = rng.uniform(-1.0, 1.0, size=(nblobs, 2))
    hh, ww = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    f = np.zeros(grid)
    for t in range(T):
        c = c0 + vel * t
        for b in range(nblobs):
            d2 = (hh - c[b, 0]) ** 2 + (ww - c[b, 1]) ** 2
            f[t] += np.exp(-d2 / (2.0 * sigma * sigma))
    f = f + rng.normal(0.0, noise, size=grid)
    return f.astype(np.float32).ravel()


def make_u(w: Workload) -> np.ndarray:
    """The per-sample uncertainty vector from the previous step: fp32 [B,N]."""
    u = np.zeros((w.B, w.N), np.float32)
    if not w.u_seeds:
        # one generator draws Q, K, V and then u (single-seed workloads)
        assert w.u_kind == "uniform"
        rng = _rng(w.qkv_seed)
        for _ in range(3):
            rng.standard_normal((w.B, w.H, w.N, w.d), dtype=np.float32)
        return rng.random((w.B, w.N), dtype=np.float32)
    for b in range(w.B):
        rng = _rng(w.u_seeds[b % len(w.u_seeds)] + (b // len(w.u_seeds)) * 1000)
        if w.u_kind == "uniform":
            u[b] = rng.random(w.N, dtype=np.float32)
        elif w.u_kind == "smooth":
            u[b] = _smooth_field(rng, w.grid)
        elif w.u_kind == "clustered":
            u[b] = _clustered_field(rng, w.grid)
        else:
            raise ValueError(w.u_kind)
    return u


def make_head(w: Workload, B: int = None):
    """Hidden states X ~ N(0,1) as bf16 [B,N,C] and weights w ~ N(0, 1/C) fp32."""
    B = w.B if B is None else B
    rng = _rng(w.x_seed)
    X = bf16_bits(rng.standard_normal((B, w.N, w.C), dtype=np.float32))
    wv = (_rng(w.w_seed).standard_normal(w.C) / np.sqrt(w.C)).astype(np.float32)
    return X, wv
