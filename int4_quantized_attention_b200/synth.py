"""Seeded synthetic inputs for the RotateAttention INT4 attention path.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no RoPE, rotation, quantisation or attention), so both
the CUDA path and the CPU oracle may take their inputs from it.

The pages describe the workloads only by model family (Wan2.2, HunyuanVideo:
"RotateAttention" review page, abstract and Sec. 5.1), and the paper's own
observation is that Q/K outliers sit on a few channels inside each 3D-RoPE
segment and are shared by Q and K (Fig. 2 caption).  Model activations are not
available, so each configuration below stands in for them with Gaussian data
whose per-channel scale is shared by Q and K:

* ``tiny``:  4 channels per RoPE segment (chosen per head) scaled by 8.
* ``half``:  per-(head, channel) lognormal(0, 1) scale.
* ``wan`` / ``hunyuan``: per-(head, channel) lognormal(0, 1.5) scale.
* ``wan_flat``: a stress case, not one of the pages' workloads: the Wan
  shapes with every Q/K channel scaled by 0.3, so the logits of a row stay
  within about one unit of each other and almost every P code is non-zero
  (no 64-key half of exponentials can be skipped).
* V is N(0, 1) everywhere.

Recipe (fixed, so that any consumer reproduces the same bytes):
``numpy.random.Generator(PCG64(seed))``; draw the channel scales first (the
outlier-channel choice for ``tiny``), then Q for every head in order, then K,
then V, each head as ``standard_normal((N, d), float32)``; multiply Q and K by
the scale vector of their head in float32 and round to float16 (RNE).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

D_HEAD = 128


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: shapes, RoPE split, rotation mode and input recipe."""

    name: str
    B: int
    H: int
    F: int
    Hh: int
    W: int
    n_text: int
    split: tuple
    rot: str                 # "none" | "interleaved" | "half"
    dist: str                # "outlier8" | "lognormal1" | "lognormal1.5"
    seed: int
    d: int = D_HEAD
    theta: float = 10000.0
    p_mode: str = "range"    # P quantisation: "range" (the method) | "symmetric"
    v_rot: int = 0           # 1: Hadamard on V inside the INT4 path (undone on O)
    blocks: Optional[tuple] = None   # rot "blocks_*": d/2 x (r00, r01, r10, r11), flattened

    @property
    def N(self) -> int:
        return self.F * self.Hh * self.W + self.n_text

    @property
    def ops(self) -> float:
        """Dense work of one attention call: 4·N²·d·H·B integer ops."""
        return 4.0 * self.N * self.N * self.d * self.H * self.B

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny and half-rotation parity cases, the two video-DiT
# shaped cases, and the mixed-precision schedule (which reuses the Wan shapes).
CONFIGS = {
    "tiny": Config("tiny", 1, 2, 4, 8, 8, 0, (44, 42, 42), "interleaved", "outlier8", 101),
    "half": Config("half", 1, 4, 8, 16, 16, 0, (44, 42, 42), "half", "lognormal1", 102),
    "wan": Config("wan", 1, 40, 21, 45, 80, 0, (44, 42, 42), "interleaved", "lognormal1.5", 103),
    "hunyuan": Config("hunyuan", 1, 24, 33, 45, 80, 256, (16, 56, 56), "half", "lognormal1.5", 104),
    "wan_flat": Config("wan_flat", 1, 40, 21, 45, 80, 0, (44, 42, 42), "interleaved", "const0.3", 105),
}

def random_pair_blocks(seed: int, d: int = D_HEAD) -> tuple:
    """d/2 seeded 2x2 orthogonal blocks (a rotation or a reflection each),
    flattened row-major: stand-ins for learned rotations."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(d // 2):
        t = rng.uniform(-np.pi, np.pi)
        c, s = np.cos(t), np.sin(t)
        out += [c, -s, s, c] if rng.random() < 0.5 else [c, s, s, -c]
    return tuple(float(v) for v in out)


def _channel_scales(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    """Per-(head, channel) float32 scale shared by Q and K."""
    H, d = cfg.B * cfg.H, cfg.d
    if cfg.dist == "outlier8":
        sc = np.ones((H, d), np.float32)
        offs = np.cumsum((0,) + tuple(cfg.split))
        for h in range(H):
            for s in range(3):
                ch = rng.choice(cfg.split[s], size=4, replace=False)
                sc[h, offs[s] + ch] = 8.0
        return sc
    if cfg.dist == "lognormal1":
        return rng.lognormal(0.0, 1.0, size=(H, d)).astype(np.float32)
    if cfg.dist == "lognormal1.5":
        return rng.lognormal(0.0, 1.5, size=(H, d)).astype(np.float32)
    if cfg.dist == "normal":
        return np.ones((H, d), np.float32)
    if cfg.dist == "const0.3":
        return np.full((H, d), 0.3, np.float32)
    raise ValueError(f"unknown distribution {cfg.dist!r}")


def make_qkv(cfg: Config, seed: Optional[int] = None, heads: Optional[int] = None):
    """Return fp16 numpy arrays q, k, v of shape [B, H, N, d] (C order).

    ``heads`` limits generation to the first ``heads`` heads of the recipe
    (same bytes as the full draw for those heads is NOT guaranteed; it is
    its own recipe used for bounded CPU samples).
    """
    rng = np.random.Generator(np.random.PCG64(cfg.seed if seed is None else seed))
    scales = _channel_scales(cfg, rng)
    BH = cfg.B * cfg.H if heads is None else heads
    N, d = cfg.N, cfg.d
    out = []
    for which in range(3):
        t = np.empty((BH, N, d), np.float16)
        for h in range(BH):
            x = rng.standard_normal((N, d), dtype=np.float32)
            if which < 2:
                x *= scales[h][None, :]
            t[h] = x.astype(np.float16)
        out.append(t.reshape((cfg.B, cfg.H, N, d) if heads is None else (1, BH, N, d)))
    return out[0], out[1], out[2]


def sample_rows(cfg: Config, frac: float = 0.01, seed: int = 7, full_heads=None):
    """Seeded (head, row) sample used for parity at full size.

    All rows of the heads in ``full_heads`` (default first and last) plus a
    ``frac`` sample of rows in every other head, always including the last row
    (the ragged tail) of every head.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    BH, N = cfg.B * cfg.H, cfg.N
    if full_heads is None:
        full_heads = (0, BH - 1)
    rows = {}
    for h in range(BH):
        if h in full_heads:
            rows[h] = np.arange(N, dtype=np.int64)
        else:
            k = max(1, int(round(frac * N)))
            r = rng.choice(N, size=k, replace=False)
            rows[h] = np.unique(np.concatenate([r, [N - 1]])).astype(np.int64)
    return rows
