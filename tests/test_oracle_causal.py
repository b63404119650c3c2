"""Pins for the oracle's frame-causal path (the world-model rollout workload:
queries in frame f see the keys of frames <= f, intersected with the route)."""
import numpy as np
import pytest

import oracle as O
from synth import generate, to_f64, workload
from synth.video import frame_index


def _brute_attention(q, k, v, scale, keep):
    out = np.zeros((len(q), v.shape[1]))
    lse = np.full(len(q), -np.inf)
    for i in range(len(q)):
        idx = [j for j in range(len(k)) if keep(i, j)]
        if not idx:
            continue
        s = np.array([scale * float(q[i] @ k[j]) for j in idx])
        m = s.max()
        w = np.exp(s - m)
        out[i] = (w[:, None] * v[idx]).sum(axis=0) / w.sum()
        lse[i] = m + np.log(w.sum())
    return out, lse


@pytest.fixture
def small():
    rng = np.random.default_rng(3)
    n, d = 40, 6
    frames = np.repeat(np.arange(4), 10)
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    lq = rng.integers(0, 3, n)
    lk = rng.integers(0, 4, n)
    return q, k, v, frames, lq, lk


def test_causal_dense_matches_brute_force(small):
    q, k, v, frames, _, _ = small
    o, l = O.attention(q, k, v, 0.4, mask=O.causal_mask(frames))
    ob, lb = _brute_attention(q, k, v, 0.4, lambda i, j: frames[j] <= frames[i])
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(l, lb, atol=1e-12)


def test_causal_sparse_matches_brute_force_and_empty_rows(small):
    q, k, v, frames, lq, lk = small
    route = np.zeros((3, 4), np.uint8)
    route[0, [1, 3]] = 1
    route[1, 2] = 1
    route[2, 0] = 1
    o, l = O.sparse_attention(q, k, v, 0.4, route, lq, lk, frames=frames)
    ob, lb = _brute_attention(q, k, v, 0.4, lambda i, j: route[lq[i], lk[j]] and frames[j] <= frames[i])
    np.testing.assert_allclose(o, ob, atol=1e-12)
    assert np.array_equal(np.isinf(l), np.isinf(lb))
    np.testing.assert_allclose(l[np.isfinite(l)], lb[np.isfinite(lb)], atol=1e-12)
    # a row of frame 0 whose routed group holds keys of later frames only sees nothing
    k0 = np.array([i for i in range(len(q)) if frames[i] == 0 and lq[i] == 1])
    if k0.size and not any(lk[j] == 2 and frames[j] == 0 for j in range(len(k))):
        assert np.all(o[k0] == 0) and np.all(np.isneginf(l[k0]))


def test_visible_counts_and_cost_are_brute_force_pair_counts(small):
    _, _, _, frames, lq, lk = small
    vis_k = O.visible_counts(lk, frames, 4, 4)
    hist_q = O.frame_histogram(lq, frames, 3, 4)
    cost = O.cell_cost(None, None, hist_q, vis_k)
    for a in range(3):
        for g in range(4):
            brute = sum(1 for i in range(len(lq)) for j in range(len(lk))
                        if lq[i] == a and lk[j] == g and frames[j] <= frames[i])
            assert cost[a, g] == brute
    assert (hist_q.sum(axis=0) @ vis_k.sum(axis=0)) == O.causal_mask(frames).sum()


def test_causal_cell_mass_counts_visible_keys_only(small):
    q, k, v, frames, lq, lk = small
    c, n_k = O.group_means(k, lk, 4)
    z = O.query_coords(q, c, 0.4)
    vis_k = O.visible_counts(lk, frames, 4, 4)
    mass = O.cell_mass(z, lq, n_k, 3, frames, vis_k)
    # per query: softmax over groups of z + ln(visible keys of the group), by loops
    p = np.zeros((len(q), 4))
    for i in range(len(q)):
        cnt = [sum(1 for j in range(len(k)) if lk[j] == g and frames[j] <= frames[i]) for g in range(4)]
        lg = np.array([z[i, g] + np.log(cnt[g]) if cnt[g] else -np.inf for g in range(4)])
        e = np.exp(lg - lg.max())
        p[i] = e / e.sum()
    for a in range(3):
        np.testing.assert_allclose(mass[a], p[lq == a].mean(axis=0), atol=1e-13)
    np.testing.assert_allclose(mass.sum(axis=1), 1.0, atol=1e-12)


def test_causal_route_invariants(small):
    q, k, v, frames, lq, lk = small
    c, n_k = O.group_means(k, lk, 4)
    z = O.query_coords(q, c, 0.4)
    vis_k = O.visible_counts(lk, frames, 4, 4)
    hist_q = O.frame_histogram(lq, frames, 3, 4)
    n_q = np.bincount(lq, minlength=3)
    mass = O.cell_mass(z, lq, n_k, 3, frames, vis_k)
    cost = O.cell_cost(n_q, n_k, hist_q, vis_k)
    visible = float(O.causal_mask(frames).sum())
    prev = -1
    for dens in (0.3, 0.5, 0.7, 1.0):
        rr = O.route_select(mass, n_q, n_k, dens, 2, len(q), cost=cost, visible=visible)
        routed = int((cost * rr.route).sum())
        assert routed == rr.routed_pairs
        if dens < 1.0 and rr.alpha > 0:
            assert routed <= rr.budget + 1e-9
        assert abs(rr.budget - (dens * visible - 2 * visible / len(q))) < 1e-9
        for a in range(3):
            if n_q[a]:
                assert rr.route[a].sum() >= 1
        assert routed >= prev
        prev = routed
    assert rr.route[:, n_k > 0].all()   # density 1 routes every non-empty cell


def test_full_density_causal_call_equals_causal_dense():
    w = workload("tiny_causal", H=1, density=1.0)
    qb, kb, vb = generate(w, seed=0)
    q, k, v = to_f64(qb[0, 0]), to_f64(kb[0, 0]), to_f64(vb[0, 0])
    frames = frame_index(w.grid)
    p = O.Params(n_kgroups=w.n_kgroups, n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes,
                 eig_rank=w.eig_rank, sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, density=1.0,
                 ridge_lambda=w.ridge_lambda, seed=0, block=w.block)
    s = p.eff_scale(w.d)
    res = O.sparsepr_head(q, k, v, p, 0, frames=frames)
    od, ld = O.attention(q, k, v, s, mask=O.causal_mask(frames))
    np.testing.assert_allclose(res.o_sparse, od, atol=1e-12)
    np.testing.assert_allclose(res.lse_sparse, ld, atol=1e-12)
    np.testing.assert_allclose(res.o, od, atol=1e-9)      # zero residual: nothing to correct
    assert abs(res.part.route.rho_exec - 1.0 - p.n_probes / w.N) < 1e-12


def test_causal_residual_identity():
    # R = omitted mass x (O_omitted - O_retained) per row, with the causal mask in both parts
    rng = np.random.default_rng(5)
    n, d = 30, 4
    frames = np.repeat(np.arange(3), 10)
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    keep = (rng.random((n, n)) < 0.5) & O.causal_mask(frames)
    keep[np.arange(n), np.arange(n)] = True            # every row keeps its own key
    omit = O.causal_mask(frames) & ~keep
    od, ld = O.attention(q, k, v, 0.3, mask=O.causal_mask(frames))
    orr, lr = O.attention(q, k, v, 0.3, mask=keep)
    oo, lo = O.attention(q, k, v, 0.3, mask=omit)
    m = O.omitted_mass(lr, ld)
    has = np.isfinite(lo)
    r = od - orr
    np.testing.assert_allclose(r[has], (m[has, None] * (oo[has] - orr[has])), atol=1e-12)
    np.testing.assert_allclose(r[~has], 0.0, atol=1e-12)
