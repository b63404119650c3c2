"""Seeded synthetic video-shaped Q/K/V (inputs only; holds none of the method).

Tokens sit on an F x H x W latent grid in row-major (f, h, w) order.  Each batch
element scatters ``n_seeds`` Voronoi seed points uniformly in the continuous box
[0,F) x [0,H) x [0,W); a token belongs to its nearest seed (Euclidean distance in
grid units, ties to the lower seed) and seed i carries centroid i mod C.  Every
head draws its own centroids mu_c ~ N(0, I_d) and value map W_v ~ N(0, 1/d):

    q = a * mu_z + N(0, 0.5^2),   k = a * mu_z + N(0, 0.5^2)   (independent noise)
    v = W_v mu_z + N(0, 1)

with a = 2.0 unless the workload's centroid scale was calibrated (the 32,760-token
workload: a is bisected so that the median query needs ~6.2% of keys for 90% of
its softmax mass, the per-query support statistic the huashangw.com article
reports for Wan2.2).  The 108,000-token workload adds a slow per-frame drift
mu_c + 0.1 * f * u_c with u_c ~ N(0, I_d).  Values are rounded once to bf16; both
the CUDA path and the oracle read the same bf16 bits.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
CALIBRATION_FILE = os.path.join(_HERE, "calibration.json")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: tuple           # (F, H, W)
    d: int
    n_centroids: int
    n_seeds: int
    block: int
    density: float
    n_kgroups: int
    n_qgroups: int
    n_samples: int
    n_probes: int
    eig_rank: int
    sub_rank: int
    kmeans_iters: int
    ridge_lambda: float = 1e-2
    centroid_scale: float = 2.0
    calibrated: bool = False
    drift: float = 0.0
    frame_causal: bool = False

    @property
    def N(self) -> int:
        f, h, w = self.grid
        return f * h * w

    @property
    def frames(self) -> int:
        return self.grid[0]


def _groups(n: int, block: int) -> int:
    return (n + 2 * block - 1) // (2 * block)


def _make(name, B, H, grid, d, C, S, block, density, **kw):
    n = grid[0] * grid[1] * grid[2]
    g = kw.pop("groups", _groups(n, block))
    base = dict(n_kgroups=g, n_qgroups=g, n_samples=max(64, d), n_probes=64,
                eig_rank=d // 4, sub_rank=d // 4, kmeans_iters=5)
    base.update(kw)
    return Workload(name=name, B=B, H=H, grid=grid, d=d, n_centroids=C, n_seeds=S,
                    block=block, density=density, **base)


WORKLOADS = {
    # 1024 tokens, the case the oracle finishes in seconds
    "tiny": _make("tiny", 1, 2, (4, 16, 16), 64, 16, 16, 64, 0.25, groups=8,
                  n_samples=64, sub_rank=16, kmeans_iters=8),
    "mid": _make("mid", 1, 12, (8, 32, 32), 64, 64, 64, 64, 0.25, kmeans_iters=8),
    "wan": _make("wan", 1, 40, (21, 30, 52), 128, 128, 256, 128, 0.25,
                 calibrated=True),
    "long": _make("long", 1, 24, (30, 45, 80), 128, 256, 512, 128, 0.25,
                  calibrated=True, drift=0.1),
    "world": _make("world", 4, 16, (16, 32, 32), 128, 128, 256, 128, 0.25,
                   calibrated=True, frame_causal=True),
    # the 1024-token case with the frame-causal mask (4 frames of 256 tokens)
    "tiny_causal": _make("tiny_causal", 1, 2, (4, 16, 16), 64, 16, 16, 64, 0.25, groups=8,
                         n_samples=64, sub_rank=16, kmeans_iters=8, frame_causal=True),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    if w.calibrated and "centroid_scale" not in overrides:
        w = replace(w, centroid_scale=calibrated_scale())
    return replace(w, **overrides) if overrides else w


def calibrated_scale() -> float:
    with open(CALIBRATION_FILE) as f:
        return float(json.load(f)["centroid_scale"])


# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = ((b >> 16) & 1) + np.uint32(0x7FFF)
    return ((b + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def voronoi_centroid_ids(grid, n_seeds: int, n_centroids: int, rng) -> np.ndarray:
    F, H, W = grid
    seeds = rng.random((n_seeds, 3)) * np.array([F, H, W], np.float64)
    f, h, w = np.meshgrid(np.arange(F), np.arange(H), np.arange(W), indexing="ij")
    coords = np.stack([f, h, w], axis=-1).reshape(-1, 3).astype(np.float64)
    out = np.empty(coords.shape[0], np.int64)
    for s0 in range(0, coords.shape[0], 8192):
        c = coords[s0:s0 + 8192]
        d2 = ((c[:, None, :] - seeds[None, :, :]) ** 2).sum(axis=2)
        out[s0:s0 + 8192] = np.argmin(d2, axis=1)
    return out % n_centroids


def frame_index(grid) -> np.ndarray:
    F, H, W = grid
    return np.repeat(np.arange(F, dtype=np.int32), H * W)


def _head_rng(seed: int, b: int, h: int, stream: int = 0):
    return np.random.default_rng([int(seed), int(b), int(h), int(stream), 0x5EED])


def head_base(w: Workload, seed: int, b: int, h: int, cid: np.ndarray):
    """mu_z per token (with drift) and the head's value map."""
    rng = _head_rng(seed, b, h)
    mu = rng.standard_normal((w.n_centroids, w.d), dtype=np.float32)
    wv = rng.standard_normal((w.d, w.d), dtype=np.float32) / np.float32(math.sqrt(w.d))
    base = mu[cid]
    if w.drift:
        u = rng.standard_normal((w.n_centroids, w.d), dtype=np.float32)
        fr = frame_index(w.grid).astype(np.float32)
        base = base + np.float32(w.drift) * fr[:, None] * u[cid]
    return base, wv, rng


def generate(w: Workload, seed: int = 0, heads=None, scale=None):
    """Q, K, V as bf16 bit arrays [B, H, N, d] (uint16).

    heads: optional list of (b, h) to generate (others left zero) -- lets tests
    build one head of a large workload cheaply."""
    a = np.float32(w.centroid_scale if scale is None else scale)
    N, d = w.N, w.d
    shape = (w.B, w.H, N, d)
    qb = np.zeros(shape, np.uint16)
    kb = np.zeros(shape, np.uint16)
    vb = np.zeros(shape, np.uint16)
    want = None if heads is None else set(heads)
    for b in range(w.B):
        cid = voronoi_centroid_ids(w.grid, w.n_seeds, w.n_centroids,
                                   np.random.default_rng([int(seed), int(b), 0x0B0B]))
        for h in range(w.H):
            if want is not None and (b, h) not in want:
                continue
            base, wv, rng = head_base(w, seed, b, h, cid)
            half = np.float32(0.5)
            q = a * base + half * rng.standard_normal((N, d), dtype=np.float32)
            k = a * base + half * rng.standard_normal((N, d), dtype=np.float32)
            v = base @ wv.T + rng.standard_normal((N, d), dtype=np.float32)
            qb[b, h] = f32_to_bf16_bits(q)
            kb[b, h] = f32_to_bf16_bits(k)
            vb[b, h] = f32_to_bf16_bits(v)
    return qb, kb, vb


def perturb(bits: np.ndarray, sigma: float, seed: int, step: int) -> np.ndarray:
    """World-model rollout step: add N(0, sigma^2) to every element (re-rounded)."""
    rng = np.random.default_rng([int(seed), int(step), 0xD1F7])
    x = bf16_bits_to_f32(bits) + np.float32(sigma) * rng.standard_normal(bits.shape, dtype=np.float32)
    return f32_to_bf16_bits(x)


def to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


def to_torch(bits: np.ndarray, device=None):
    """bf16 torch tensor viewing the same bits (torch imported lazily)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t
