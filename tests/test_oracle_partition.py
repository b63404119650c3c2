"""Pins for the oracle's response-coupled partition (metric, eigenpairs, key
coordinates, k-means, group centroids, query coordinates, permutation, tile mask)."""
import itertools

import numpy as np

import oracle as O


def test_metric_brute_force():
    rng = np.random.default_rng(0)
    qs = rng.standard_normal((6, 4))
    m = O.key_metric(qs)
    for a in range(4):
        for b in range(4):
            assert abs(m[a, b] - sum(qs[i, a] * qs[i, b] for i in range(6)) / 6) < 1e-13


def test_sample_queries_are_the_stream_draw():
    idx = O.sample_queries(100, 10, seed=3, bh=2)
    rng = O.SplitMix64(O.stream_state(3, 2, O.STREAM_QUERY_SAMPLE))
    assert list(idx) == O.draw_without_replacement(rng, 100, 10)
    assert len(set(idx)) == 10


def test_eigenpairs_invariants():
    rng = np.random.default_rng(1)
    qs = rng.standard_normal((20, 8))
    m = O.key_metric(qs)
    lam, u = O.top_eigenpairs(m, 8)
    np.testing.assert_allclose(m @ u, u * lam, atol=1e-12)
    np.testing.assert_allclose(u.T @ u, np.eye(8), atol=1e-12)
    assert np.all(np.diff(lam) <= 0)
    # trace = sum of eigenvalues (nothing dropped at full rank)
    assert abs(lam.sum() - np.trace(m)) < 1e-12


def test_key_coords_distance_identity():
    # at full rank, ||y1 - y2||^2 = ||Q_s (k1 - k2)||^2 / M_s: the mean squared
    # logit difference of two keys under the sampled queries (huashangw.com,
    # key-response coordinates)
    rng = np.random.default_rng(2)
    qs = rng.standard_normal((12, 6))
    k = rng.standard_normal((5, 6))
    lam, u = O.top_eigenpairs(O.key_metric(qs), 6)
    y = O.key_coords(k, lam, u)
    for i, j in itertools.combinations(range(5), 2):
        lhs = ((y[i] - y[j]) ** 2).sum()
        rhs = ((qs @ (k[i] - k[j])) ** 2).sum() / 12
        assert abs(lhs - rhs) < 1e-10 * max(1, rhs)
    # eigenvector sign flips leave the coordinates' distances unchanged
    y2 = O.key_coords(k, lam, u * np.array([1, -1, 1, -1, -1, 1]))
    np.testing.assert_allclose(((y2[:, None] - y2[None]) ** 2).sum(-1),
                               ((y[:, None] - y[None]) ** 2).sum(-1), atol=1e-10)


def test_kmeans_assign_ties_and_direct_distance():
    x = np.array([[0.0, 0.0], [1.0, 0.0], [3.0, 0.0]])
    mu = np.array([[0.5, 0.0], [0.5, 0.0], [2.0, 0.0]])
    lab = O.kmeans_assign(x, mu)
    assert list(lab) == [0, 0, 2]          # exact tie 0/1 -> lower index
    x2 = np.array([[1.25, 0.0]])           # equidistant from 0.5 and 2.0
    assert O.kmeans_assign(x2, mu)[0] == 0


def test_kmeans_update_keeps_empty():
    x = np.array([[0.0], [2.0], [10.0]])
    mu = O.kmeans_update(x, np.array([0, 0, 2]), np.array([[0.0], [5.0], [9.0]]))
    np.testing.assert_allclose(mu, [[1.0], [5.0], [10.0]])


def test_kmeans_recovers_planted_clusters():
    rng = np.random.default_rng(3)
    centers = rng.standard_normal((6, 5)) * 20
    truth = rng.integers(0, 6, 300)
    x = centers[truth] + rng.standard_normal((300, 5)) * 0.1
    # seeds drawn until one point of every cluster is seeded
    for seed in range(100):
        init = O.kmeans_init(300, 6, seed, 0, 1)
        if len(set(truth[init])) == 6:
            break
    lab, mu, init2 = O.kmeans(x, 6, 5, seed, 0, 1)
    assert list(init2) == list(init)
    # identical partitions up to renaming
    pairs = set(zip(lab, truth))
    assert len(pairs) == 6 and len({a for a, _ in pairs}) == 6
    # Lloyd fixed point: labels are the argmin of their own means
    mu_f = O.kmeans_update(x, lab, mu)
    assert np.array_equal(O.kmeans_assign(x, mu_f), lab)


def test_kmeans_objective_non_increasing():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((200, 3))
    hist = []
    O.kmeans(x, 7, 8, 11, 0, 1, hist)
    init = O.kmeans_init(200, 7, 11, 0, 1)
    mu = x[init]
    prev = np.inf
    for t, lab in enumerate(hist):
        assert np.array_equal(lab, O.kmeans_assign(x, mu))  # each step is the argmin
        obj = ((x - mu[lab]) ** 2).sum()
        assert obj <= prev + 1e-9
        prev = obj
        mu = O.kmeans_update(x, lab, mu)


def test_kmeans_brute_force_optimum_on_tiny():
    # two well separated blobs of 5 points each: Lloyd from any two distinct
    # seeds in different blobs reaches the exhaustive optimum partition
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal((5, 2)), rng.standard_normal((5, 2)) + 30])
    best, best_lab = np.inf, None
    for bits in itertools.product([0, 1], repeat=10):
        lab = np.array(bits)
        if lab.min() == lab.max():
            continue
        obj = sum(((x[lab == g] - x[lab == g].mean(0)) ** 2).sum() for g in (0, 1))
        if obj < best:
            best, best_lab = obj, lab
    for seed in range(50):
        init = O.kmeans_init(10, 2, seed, 0, 1)
        if (init[0] < 5) != (init[1] < 5):
            lab, _, _ = O.kmeans(x, 2, 4, seed, 0, 1)
            obj = sum(((x[lab == g] - x[lab == g].mean(0)) ** 2).sum() for g in (0, 1))
            assert abs(obj - best) < 1e-9
            assert len(set(zip(lab, best_lab))) == 2


def test_group_means_and_logit_linearity():
    # q . c_g equals q's mean logit over the keys of group g (gist 2.A centroid)
    rng = np.random.default_rng(6)
    k = rng.standard_normal((40, 4))
    lab = rng.integers(0, 5, 40)
    lab[lab == 3] = 4  # group 3 empty
    c, n = O.group_means(k, lab, 5)
    assert n[3] == 0 and np.all(c[3] == 0) and n.sum() == 40
    q = rng.standard_normal((3, 4))
    z = O.query_coords(q, c, 0.5)
    for g in (0, 1, 2, 4):
        np.testing.assert_allclose(z[:, g], 0.5 * (q @ k[lab == g].T).mean(axis=1), atol=1e-12)


def test_query_coords_metric_form():
    # k-means distances in logit-profile space equal the d-space metric form
    # s^2 (q - q')^T C^T C (q - q')
    rng = np.random.default_rng(7)
    c = rng.standard_normal((6, 4))
    q = rng.standard_normal((10, 4))
    z = O.query_coords(q, c, 0.3)
    a = c.T @ c
    for i, j in itertools.combinations(range(10), 2):
        dq = q[i] - q[j]
        assert abs(((z[i] - z[j]) ** 2).sum() - 0.09 * dq @ a @ dq) < 1e-12


def test_group_permutation():
    rng = np.random.default_rng(8)
    lab = rng.integers(0, 6, 50)
    lab[lab == 2] = 5
    perm, off = O.group_permutation(lab, 6)
    assert sorted(perm) == list(range(50))
    assert off[0] == 0 and off[-1] == 50 and off[2] == off[3]
    for g in range(6):
        seg = perm[off[g]:off[g + 1]]
        assert np.all(lab[seg] == g)
        assert np.all(np.diff(seg) > 0)   # stable: ascending original index


def test_block_mask_brute_force():
    rng = np.random.default_rng(9)
    n, blk = 37, 8
    lq = rng.integers(0, 4, n)
    lk = rng.integers(0, 3, n)
    route = (rng.random((4, 3)) < 0.4).astype(np.uint8)
    pq, _ = O.group_permutation(lq, 4)
    pk, _ = O.group_permutation(lk, 3)
    bm = O.block_mask(route, lq, pq, lk, pk, blk)
    t = (n + blk - 1) // blk
    assert bm.shape == (t, t)
    for i in range(t):
        for j in range(t):
            want = any(route[lq[pq[a]], lk[pk[b]]]
                       for a in range(i * blk, min(n, (i + 1) * blk))
                       for b in range(j * blk, min(n, (j + 1) * blk)))
            assert bm[i, j] == want
