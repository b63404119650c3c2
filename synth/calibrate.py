"""Calibrate the centroid scale of the d=128 video workloads.

Bisects the centroid scale ``a`` so that, on 256 random query rows of head (0, 0)
of the 32,760-token workload (seed 0), the median per-query fraction of keys that
holds 90% of the row's softmax mass is 6.2% -- the per-query support the
huashangw.com article reports for Wan2.2 (section on grouped versus per-query
support).  Writes synth/calibration.json.  Input statistics only: plain softmax
rows, nothing of the SparsePR method.

    python -m synth.calibrate
"""
from __future__ import annotations

import json
import math

import numpy as np

from .video import CALIBRATION_FILE, WORKLOADS, _head_rng, bf16_bits_to_f32, f32_to_bf16_bits, head_base, voronoi_centroid_ids

TARGET = 0.062
MASS = 0.90


def support_fraction(a: float, n_rows: int = 256, seed: int = 0) -> float:
    w = WORKLOADS["wan"]
    cid = voronoi_centroid_ids(w.grid, w.n_seeds, w.n_centroids,
                               np.random.default_rng([seed, 0, 0x0B0B]))
    base, _, rng = head_base(w, seed, 0, 0, cid)
    N, d = w.N, w.d
    q = np.float32(a) * base + np.float32(0.5) * rng.standard_normal((N, d), dtype=np.float32)
    k = np.float32(a) * base + np.float32(0.5) * rng.standard_normal((N, d), dtype=np.float32)
    q = bf16_bits_to_f32(f32_to_bf16_bits(q)).astype(np.float64)
    k = bf16_bits_to_f32(f32_to_bf16_bits(k)).astype(np.float64)
    rows = np.random.default_rng([seed, 0xCA1]).choice(N, n_rows, replace=False)
    s = (q[rows] @ k.T) / math.sqrt(d)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    p = -np.sort(-p, axis=1)
    need = (np.cumsum(p, axis=1) < MASS).sum(axis=1) + 1
    return float(np.median(need / N))


def calibrate(lo: float = 0.3, hi: float = 2.0, steps: int = 24) -> float:
    # the support fraction falls as the centroid scale grows
    for _ in range(steps):
        mid = 0.5 * (lo + hi)
        if support_fraction(mid) > TARGET:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


if __name__ == "__main__":
    a = calibrate()
    frac = support_fraction(a)
    with open(CALIBRATION_FILE, "w") as f:
        json.dump({"centroid_scale": a, "median_support_fraction": frac,
                   "target": TARGET, "mass": MASS, "rows": 256, "seed": 0}, f, indent=1)
    print(json.dumps({"centroid_scale": a, "median_support_fraction": frac}))
