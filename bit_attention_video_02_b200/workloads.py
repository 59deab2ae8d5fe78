"""Seeded synthetic Q/K/V generators shaped like video-DiT attention inputs.

This module holds no step of the attention method: it only draws random numbers
(torch generators, seeded) and casts them to bf16.  Both the CUDA path and the
CPU oracle are fed the same bytes from here.

The pages' own workloads (Wan2.2 / MiniMax-H3 activations) are not available;
these recipes stand in for them.  Shapes follow the Wan latent grid
(21 x 45 x 80 = 75,600 tokens, flattened t-major) and the other clip shapes named
for the five workloads:

  1  tiny correctness  B=1 H=2  N=1024           N(0,1); V: 1% tokens x20 on 8 channels
  2  mixture           B=1 H=8  N=8192           32-centroid Gaussian mixture, sigma 0.3;
                                                 V: 0.5% tokens x30 on 4..16 channels
  3  Wan-shaped layer  B=1 H=40 N=75600 (21x45x80) 16 sinusoids of (t,h,w) per channel,
                                                 + N(0, 0.2^2); V: 1% tokens x25
  4  denoising steps   B=1 H=24 N=32768 (8x64x64)  base as 3, outliers as 2,
                                                 X_s = X_{s-1} + N(0, 0.05^2), 4 steps
  5  long clip         B=1 H=24 N=122880 (60x32x64) as 3 (noise 0.2), V: 1% tokens x25
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    B: int
    H: int
    N: int
    k: int                      # V-Smooth clusters
    recipe: str                 # "gauss" | "mixture" | "sinusoid"
    grid: tuple | None = None   # (T, Hg, Wg) for sinusoid recipes
    steps: int = 1
    v_out_frac: float = 0.01
    v_out_scale: float = 20.0
    v_out_channels: tuple = (8, 8)   # inclusive range of outlier channels per head
    noise: float = 0.2
    step_noise: float = 0.05
    d: int = HEAD_DIM

    @property
    def seed(self) -> int:
        return 1000 + self.cid

    @property
    def flops(self) -> float:
        """Dense attention work 4*B*H*N^2*d (QK^T and PV) for one step."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d

    def describe(self) -> str:
        g = "x".join(map(str, self.grid)) if self.grid else "-"
        return (f"cfg{self.cid} {self.name}: B={self.B} H={self.H} N={self.N} d={self.d} "
                f"grid={g} k={self.k} steps={self.steps}")


WORKLOADS = {
    1: Workload(1, "tiny", 1, 2, 1024, k=8, recipe="gauss", v_out_frac=0.01,
                v_out_scale=20.0, v_out_channels=(8, 8)),
    2: Workload(2, "mixture", 1, 8, 8192, k=32, recipe="mixture", v_out_frac=0.005,
                v_out_scale=30.0, v_out_channels=(4, 16)),
    3: Workload(3, "wan_layer", 1, 40, 75600, k=32, recipe="sinusoid", grid=(21, 45, 80),
                v_out_frac=0.01, v_out_scale=25.0, v_out_channels=(4, 16), noise=0.2),
    4: Workload(4, "denoise_steps", 1, 24, 32768, k=32, recipe="sinusoid", grid=(8, 64, 64),
                steps=4, v_out_frac=0.005, v_out_scale=30.0, v_out_channels=(4, 16),
                noise=0.2, step_noise=0.05),
    5: Workload(5, "long_clip", 1, 24, 122880, k=32, recipe="sinusoid", grid=(60, 32, 64),
                v_out_frac=0.01, v_out_scale=25.0, v_out_channels=(4, 16), noise=0.2),
}


def shrink(w: Workload, H: int | None = None, N: int | None = None) -> Workload:
    """Same recipe at a smaller size (for CPU-time oracle comparisons)."""
    grid = w.grid
    if N is not None and grid is not None:
        # keep a (t, h, w) structure: fold the token count into a T x 8 x W grid
        grid = (max(1, N // 64), 8, 8) if N % 64 == 0 and N >= 64 else (1, 1, N)
    return replace(w, H=H if H is not None else w.H, N=N if N is not None else w.N, grid=grid)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _coords(grid, N, device):
    T, Hg, Wg = grid
    n = torch.arange(N, device=device, dtype=torch.float32)
    t = torch.div(n, Hg * Wg, rounding_mode="floor")
    rem = n - t * (Hg * Wg)
    h = torch.div(rem, Wg, rounding_mode="floor")
    w = rem - h * Wg
    return t, h, w


def _sinusoid_head(g, coords, N, d, noise, device):
    t, h, w = coords
    x = torch.zeros(N, d, device=device, dtype=torch.float32)
    om = torch.rand(16, 3, d, generator=g, device=device) * 0.5
    ph = torch.rand(16, d, generator=g, device=device) * (2 * math.pi)
    for s in range(16):
        arg = (t[:, None] * om[s, 0][None, :] + h[:, None] * om[s, 1][None, :]
               + w[:, None] * om[s, 2][None, :] + ph[s][None, :])
        x += torch.sin(arg)
    x += noise * torch.randn(N, d, generator=g, device=device)
    return x


def _mixture_head(g, N, d, device):
    cents = torch.randn(32, d, generator=g, device=device)
    pick = torch.randint(0, 32, (N,), generator=g, device=device)
    return cents[pick] + 0.3 * torch.randn(N, d, generator=g, device=device)


def _inject_v_outliers(g, v, w: Workload):
    N, d = v.shape
    n_out = int(math.ceil(w.v_out_frac * N))
    if n_out == 0:
        return v
    toks = torch.randperm(N, generator=g, device=v.device)[:n_out]
    lo, hi = w.v_out_channels
    nch = int(torch.randint(lo, hi + 1, (1,), generator=g, device=v.device).item())
    chans = torch.randperm(d, generator=g, device=v.device)[:nch]
    v[toks[:, None], chans[None, :]] *= w.v_out_scale
    return v


def make_qkv(w: Workload, device="cpu", step: int = 0):
    """Q, K, V as bf16 tensors [B, H, N, d] on `device`, for denoising step `step`."""
    device = torch.device(device)
    g = _gen(device, w.seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    out = []
    coords = _coords(w.grid, N, device) if w.recipe == "sinusoid" else None
    for tensor in range(3):
        x = torch.empty(B, H, N, d, device=device, dtype=torch.float32)
        for b in range(B):
            for hh in range(H):
                if w.recipe == "gauss":
                    xh = torch.randn(N, d, generator=g, device=device)
                elif w.recipe == "mixture":
                    xh = _mixture_head(g, N, d, device)
                else:
                    xh = _sinusoid_head(g, coords, N, d, w.noise, device)
                if tensor == 2:
                    xh = _inject_v_outliers(g, xh, w)
                x[b, hh] = xh
        out.append(x)
    # denoising-step drift: X_s = X_{s-1} + N(0, step_noise^2), drawn in step order
    for s in range(1, step + 1):
        for x in out:
            x += w.step_noise * torch.randn(x.shape, generator=g, device=device)
    return tuple(x.to(torch.bfloat16) for x in out)


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a CPU bf16 tensor's bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
