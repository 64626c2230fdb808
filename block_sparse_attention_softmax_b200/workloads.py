"""Seeded synthetic inputs for the block-sparse attention path.

The pages measure on video-DiT self-attention (Wan2.1-1.3B at 480p, Wan2.1-14B
at 720p, and a 245K-token Waver-class sequence: SpargeAttention2 §4, SLA2
"実験結果", Veda §4). No model or dataset is available here, so these
generators stand in for those activations: Q and K carry i.i.d. N(0,1) noise
plus a smooth 3-D positional field over the (t, y, x) latent grid, which gives
nearby tokens larger q·k and therefore the local, peaked block scores that
real video attention shows. V is i.i.d. N(0,1).

This module holds no arithmetic of the attention method itself: it only draws
random numbers. Both the CUDA path and the CPU oracle consume the same bytes.

Positional field, per head h and channel c (integer frequencies keep it smooth
at the scale of the whole grid):

    P_c(t, y, x) = sqrt(2) * cos(2*pi*(f_t*t/T + f_y*y/Hh + f_x*x/W) + phi_c)
    f_t, f_y, f_x ~ U{0, 1, 2},   phi_c ~ U(0, 2*pi)

Q = Z_q + A*P, K = Z_k + A*P with A = 1/sigma = 2 (sigma = 0.5 read as the
ratio of noise std to positional std). Every draw comes from one
torch.Generator seeded per workload, head by head, so any device reproduces
its own stream and memory stays bounded by one head at a time.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    bq: int
    bk: int
    topk: float          # Top-k fraction of key blocks per row, in (0, 1]
    topp: float          # Top-p cumulative-probability target, in [0, 1]
    kind: str            # "iid" | "local" | "sink"
    grid: tuple | None   # (T, Hh, W) latent grid, raster t-major; None for iid
    linear: bool         # run the elu+1 linear branch and the alpha blend
    seed: int
    description: str = ""

    @property
    def n_qb(self) -> int:
        return -(-self.N // self.bq)

    @property
    def n_kb(self) -> int:
        return -(-self.N // self.bk)

    def with_n(self, grid):
        """Same recipe on a smaller latent grid (for tests that need small N)."""
        n = grid[0] * grid[1] * grid[2]
        return replace(self, grid=tuple(grid), N=n, name=f"{self.name}@{n}")


POS_AMPLITUDE = 2.0      # 1 / sigma with sigma = 0.5
SINK_KEYS = 4            # sink tokens per head
SINK_GAIN = 8.0          # sink keys are scaled by this factor
FLAT_HEAD_FRAC = 0.25    # share of heads whose Q is shrunk towards uniform logits
FLAT_Q_GAIN = 0.05

WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 1024, 64, 64, 64, 0.10, 0.9, "iid", None, False, 1235,
                     "B=1 H=2 N=1024 d=64, i.i.d. N(0,1), 64x64 blocks, Top-k 10% + Top-p 0.9"),
    "wan13b_480p": Workload("wan13b_480p", 1, 12, 32760, 128, 128, 64, 0.05, 0.9, "local",
                            (21, 30, 52), False, 1236,
                            "Wan2.1-1.3B-480p-shaped self-attention, 21x30x52 grid"),
    "wan14b_720p": Workload("wan14b_720p", 1, 40, 75600, 128, 128, 64, 0.03, 0.85, "local",
                            (21, 45, 80), True, 1237,
                            "Wan2.1-14B-720p-shaped, 21x45x80 grid, + elu+1 linear branch"),
    "sink_skew": Workload("sink_skew", 1, 40, 75600, 128, 128, 64, 0.05, 0.9, "sink",
                          (21, 45, 80), False, 1238,
                          "14B-720p geometry with sink keys and near-uniform heads"),
    "long_245k": Workload("long_245k", 1, 40, 245760, 128, 128, 64, 0.05, 0.9, "local",
                          (30, 64, 128), False, 1239,
                          "245,760 tokens, 30x64x128 grid"),
}


def _grid_coords(grid, device):
    T, Hh, W = grid
    t = torch.arange(T, device=device, dtype=torch.float32)
    y = torch.arange(Hh, device=device, dtype=torch.float32)
    x = torch.arange(W, device=device, dtype=torch.float32)
    tt, yy, xx = torch.meshgrid(t / T, y / Hh, x / W, indexing="ij")
    return torch.stack([tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)], 1)  # [N, 3]


def make_inputs(wl: Workload, device="cpu", seed: int | None = None):
    """Return dict(q, k, v [B,H,N,d] bf16 contiguous, alpha [H,d] fp32 or None)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else seed)
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    q = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    coords = _grid_coords(wl.grid, device) if wl.kind in ("local", "sink") else None
    flat_heads = set()
    if wl.kind == "sink":
        n_flat = int(round(FLAT_HEAD_FRAC * H))
        perm = torch.randperm(H, generator=g, device=device).tolist()
        flat_heads = set(perm[:n_flat])
    for b in range(B):
        for h in range(H):
            zq = torch.randn(N, d, generator=g, device=device)
            zk = torch.randn(N, d, generator=g, device=device)
            zv = torch.randn(N, d, generator=g, device=device)
            if coords is not None:
                f = torch.randint(0, 3, (d, 3), generator=g, device=device).float()
                phi = torch.rand(d, generator=g, device=device) * (2 * math.pi)
                pos = math.sqrt(2.0) * torch.cos(2 * math.pi * (coords @ f.T) + phi)
                zq += POS_AMPLITUDE * pos
                zk += POS_AMPLITUDE * pos
                del pos
            if wl.kind == "sink":
                sinks = torch.randperm(N, generator=g, device=device)[:SINK_KEYS]
                zk[sinks] *= SINK_GAIN
                if h in flat_heads:
                    zq *= FLAT_Q_GAIN
            q[b, h] = zq.to(torch.bfloat16)
            k[b, h] = zk.to(torch.bfloat16)
            v[b, h] = zv.to(torch.bfloat16)
    alpha = None
    if wl.linear:
        alpha = torch.rand(H, d, generator=g, device=device, dtype=torch.float32)
    return {"q": q, "k": k, "v": v, "alpha": alpha, "flat_heads": sorted(flat_heads)}


def random_qkv(B, H, N, d, seed, device="cpu", scale=1.0):
    """Plain i.i.d. N(0, scale^2) bf16 Q/K/V for edge-case tests."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = [(torch.randn(B, H, N, d, generator=g, device=device) * scale).to(torch.bfloat16)
           for _ in range(3)]
    return out
