"""Seeded synthetic inputs for the packed-KV-cache context-attention path.

This module only draws numbers and lays them out.  It holds none of the
method's arithmetic: the token counts ``n`` and ``n_c`` of each workload are
written here as literal values, and checking them against the pages'
formulas is the oracle's job.  Both the CUDA path (through the tests and the
bench) and the oracle take their inputs from here, and from nowhere else.

Workloads follow the setting of the PackForcing pages (Wan2.1-T2V-1.3B,
832x480 at 16 FPS, 4-latent-frame blocks of 30x52 patches, 12 heads of 128
dims; "Implementation Details" and Sec. 3.2 "Compressed Mid Tokens"):

* ``tiny``      1 head, 6x8-patch blocks (n=192, n_c=4), 8-block pool, top-3.
* ``layer``     one layer at the pages' scale: n=6,240, n_c=182, pool 40, top-16.
* ``step30``    the same per-layer shapes with a 116-block pool, 30 layers.
* ``dense``     a 748,800-key full-resolution context, no mid pool.
* ``stress16`` / ``stress64``  batch 2, a 1,000-block pool, top-16 / top-64.
* ``ragged_a`` / ``ragged_b`` / ``ragged_c``  small test shapes whose block
  and pool sizes are not multiples of any tile size, to exercise ragged tails
  (``ragged_c`` has an odd number of 128-row query tiles).

Values are N(0,1) drawn by torch's generators and rounded to bf16.  Planted
mid blocks follow the recipe K~ = 0.8 * mean_i(Q_i) + 0.2 * N(0,1), with the
mean taken over the current block's queries, per head.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    block_frames: int
    h: int
    w: int
    n: int            # tokens per full-resolution block (literal value)
    n_c: int          # tokens per compressed mid block (literal value)
    sink_blocks: int
    recent_blocks: int
    pool_blocks: int  # live compressed mid blocks when attention runs
    mid_capacity: int
    n_top: int
    planted: int
    delta_lo: int
    delta_hi: int
    layers: int = 1
    rope_split: tuple = (44, 42, 42)
    rope_base: float = 10000.0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 4, 6, 8, 192, 4, 2, 1, 8, 8, 3, 3, 5, 5),
    "layer": Workload("layer", 1, 12, 128, 4, 30, 52, 6240, 182, 2, 1, 40, 40, 16, 16, 1, 32),
    "step30": Workload("step30", 1, 12, 128, 4, 30, 52, 6240, 182, 2, 1, 116, 116, 16, 16, 4, 4,
                       layers=30),
    "dense": Workload("dense", 1, 12, 128, 4, 30, 52, 6240, 182, 0, 119, 0, 0, 0, 0, 0, 0),
    "stress16": Workload("stress16", 2, 12, 128, 4, 30, 52, 6240, 182, 2, 1, 1000, 1000, 16, 16,
                         1, 64),
    "stress64": Workload("stress64", 2, 12, 128, 4, 30, 52, 6240, 182, 2, 1, 1000, 1000, 64, 64,
                         1, 64),
    # small shapes for parity at oracle-friendly sizes: n and n_c are not
    # multiples of 32, the pool is not a multiple of anything.
    "ragged_a": Workload("ragged_a", 2, 2, 128, 4, 6, 10, 240, 4, 2, 1, 13, 13, 5, 5, 1, 32),
    "ragged_b": Workload("ragged_b", 1, 3, 128, 2, 9, 13, 234, 6, 1, 2, 11, 16, 4, 4, 1, 32),
    # an odd number (3) of 128-row query tiles: the last tile is split along the context
    "ragged_c": Workload("ragged_c", 2, 3, 128, 4, 6, 14, 336, 6, 2, 1, 9, 9, 4, 4, 1, 32),
}

SEED_BASE = 1000


def nominal_seed(workload_index: int, layer: int = 0) -> int:
    """Seed rule: 1000 + 100 * workload index + layer."""
    return SEED_BASE + 100 * workload_index + layer


def _bf16_normal(gen: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_layer(wl: Workload, seed: int, device="cpu", with_values: bool = True) -> dict:
    """Draw one layer's inputs.

    Returns a dict of bf16 tensors on ``device`` (layout ``[B, L, H, D]``
    token-major, or ``[B, blocks, L, H, D]`` for per-block stores) plus the
    planted mid-block indices and the RoPE shift ``delta``:

    ``Q, K_cur, V_cur``           [B, n, H, D]      current block
    ``sink_K, sink_V``            [B, S, n, H, D]   full-resolution sink blocks
    ``mid_K, mid_V``              [B, P, n_c, H, D] compressed pool, oldest first
    ``recent_K, recent_V``        [B, R, n, H, D]   full-resolution recent blocks
    ``recent_Kc, recent_Vc``      [B, R, n_c, H, D] their compressed backups
    ``planted``                   [B, planted] int64, ascending
    ``delta``                     int
    """
    B, H, D, n, nc = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c
    S, R, P = wl.sink_blocks, wl.recent_blocks, wl.pool_blocks
    dev = torch.device(device)
    # one generator per tensor, so that skipping a tensor leaves the others as they are
    names = ["Q", "K_cur", "V_cur", "sink_K", "sink_V", "recent_K", "recent_V",
             "recent_Kc", "recent_Vc", "mid_K", "mid_V", "plant_noise", "plant_idx"]
    sub = {name: seed * 64 + i for i, name in enumerate(names)}

    def draw(name, shape):
        return bf16_normal(shape, sub[name], dev)

    out = {}
    out["Q"] = draw("Q", (B, n, H, D))
    out["K_cur"] = draw("K_cur", (B, n, H, D))
    out["V_cur"] = draw("V_cur", (B, n, H, D)) if with_values else None
    out["sink_K"] = draw("sink_K", (B, S, n, H, D))
    out["sink_V"] = draw("sink_V", (B, S, n, H, D)) if with_values else None
    out["recent_K"] = draw("recent_K", (B, R, n, H, D))
    out["recent_V"] = draw("recent_V", (B, R, n, H, D)) if with_values else None
    out["recent_Kc"] = draw("recent_Kc", (B, R, nc, H, D))
    out["recent_Vc"] = draw("recent_Vc", (B, R, nc, H, D))
    mid_K = draw("mid_K", (B, P, nc, H, D))
    out["mid_V"] = draw("mid_V", (B, P, nc, H, D)) if with_values else None

    cpu = torch.Generator(device="cpu").manual_seed(sub["plant_idx"])
    planted = torch.zeros((B, wl.planted), dtype=torch.int64)
    if P > 0 and wl.planted > 0:
        qmean = out["Q"].float().mean(dim=1)                      # [B, H, D]
        ngen = (torch.Generator(device="cpu") if dev.type == "cpu"
                else torch.Generator(device=dev)).manual_seed(sub["plant_noise"])
        for b in range(B):
            idx = torch.randperm(P, generator=cpu)[: wl.planted].sort().values
            planted[b] = idx
            noise = torch.randn((len(idx), nc, H, D), generator=ngen, device=dev)
            mid_K[b, idx.to(dev)] = (0.8 * qmean[b][None, None] + 0.2 * noise).to(torch.bfloat16)
    out["mid_K"] = mid_K
    out["planted"] = planted
    if wl.delta_hi > 0:
        out["delta"] = int(torch.randint(wl.delta_lo, wl.delta_hi + 1, (1,), generator=cpu))
    else:
        out["delta"] = 0
    return out


def make_block(wl: Workload, seed: int, device="cpu") -> dict:
    """One generated block as the cache receives it: full K/V and compressed Kc/Vc."""
    B, H, D, n, nc = wl.batch, wl.heads, wl.head_dim, wl.n, wl.n_c
    return {
        "K": bf16_normal((B, n, H, D), seed * 64 + 0, device),
        "V": bf16_normal((B, n, H, D), seed * 64 + 1, device),
        "Kc": bf16_normal((B, nc, H, D), seed * 64 + 2, device),
        "Vc": bf16_normal((B, nc, H, D), seed * 64 + 3, device),
    }


def bf16_normal(shape, seed: int, device="cpu") -> torch.Tensor:
    """A plain seeded N(0,1) bf16 tensor."""
    dev = torch.device(device)
    gen = (torch.Generator(device="cpu") if dev.type == "cpu"
           else torch.Generator(device=dev)).manual_seed(seed)
    return _bf16_normal(gen, shape, dev)
