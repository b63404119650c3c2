"""Host-side arithmetic of bench.py on CPU: the routed attention's useful and MMA-issued
(query, key) pair counts against a row-by-row enumeration of the kernel's work (units of
up to 256 rows of a query group, 128-row q-tiles, 128-key chunks of the tile's key stream;
frame-causal: the stream of keys of frames <= the frame of the tile's last row, the unit's
last row for its second tile)."""
import numpy as np
import torch

import bench


def _partition(rng, BH, N, Gq, Gk, F=None):
    """A random partition: labels, group-contiguous permutations (ascending token order
    inside a group), offsets and a route with every query group routed somewhere."""
    out = {k: [] for k in ("label_q", "label_k", "perm_q", "perm_k", "qoff", "koff", "route")}
    for _ in range(BH):
        lq = rng.integers(0, Gq, N)
        lk = rng.integers(0, Gk, N)
        route = (rng.random((Gq, Gk)) < 0.3).astype(np.uint8)
        route[np.arange(Gq), rng.integers(0, Gk, Gq)] = 1
        for name, lab, G in (("q", lq, Gq), ("k", lk, Gk)):
            perm = np.argsort(lab, kind="stable")
            off = np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=G))])
            out["label_" + name].append(lab)
            out["perm_" + name].append(perm)
            out[name + "off"].append(off)
        out["route"].append(route)
    return {k: torch.from_numpy(np.stack(v).astype(np.int32 if k != "route" else np.uint8)) for k, v in out.items()}


def _enumerate(part, frames=None):
    lq, lk = part["label_q"].numpy(), part["label_k"].numpy()
    pq = part["perm_q"].numpy()
    qoff, koff, route = part["qoff"].numpy(), part["koff"].numpy(), part["route"].numpy()
    BH, N = lq.shape
    fr = np.zeros(N, np.int64) if frames is None else np.asarray(frames)
    useful = issued = 0
    for bh in range(BH):
        for q in range(N):
            for k in range(N):
                if route[bh, lq[bh, q], lk[bh, k]] and fr[k] <= fr[q]:
                    useful += 1
        for a in range(route.shape[1]):
            def stream_len(row):   # routed keys this query row's frame may see
                f = fr[row]
                return sum(int(route[bh, a, lk[bh, k]]) for k in range(N) if fr[k] <= f)
            for u0 in range(qoff[bh, a], qoff[bh, a + 1], 256):
                rows = min(256, qoff[bh, a + 1] - u0)
                last = stream_len(pq[bh, u0 + rows - 1]) if frames is not None else \
                    sum(int(route[bh, a, lk[bh, k]]) for k in range(N))
                tiles = [last]
                if rows > 128:
                    first = stream_len(pq[bh, u0 + 127]) if frames is not None else last
                    tiles.insert(0, min(first, last))
                issued += sum(128 * 128 * ((t + 127) // 128) for t in tiles)
    return useful, issued


def test_attention_pairs_match_enumeration():
    rng = np.random.default_rng(0)
    part = _partition(rng, BH=2, N=700, Gq=3, Gk=5)
    assert bench.attention_pairs(part) == _enumerate(part)


def test_causal_attention_pairs_match_enumeration():
    rng = np.random.default_rng(1)
    N, F = 720, 4
    frames = np.repeat(np.arange(F), N // F)
    part = _partition(rng, BH=2, N=N, Gq=2, Gk=4, F=F)
    assert bench.attention_pairs(part, frames) == _enumerate(part, frames)


def test_job_figure_is_all_ranks_calls_over_the_slowest_time():
    assert bench.job_ms_per_call(100.0, 10, 1) == 10.0
    assert bench.job_ms_per_call(100.0, 10, 4) == 2.5
