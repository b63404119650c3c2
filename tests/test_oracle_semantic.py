"""Pins of the semantic-grouping baseline and of the partition diagnostics
(huashangw.com article: grouping-strategy comparison; per-query versus grouped
support).  CPU only."""
import numpy as np

import oracle as O


def _params(**kw):
    base = dict(n_kgroups=2, n_qgroups=2, n_samples=32, n_probes=8, eig_rank=2, sub_rank=2, kmeans_iters=6,
                density=0.5, ridge_lambda=1e-2, seed=3, block=16)
    base.update(kw)
    return O.Params(**base)


def _same_partition(a, b):
    """Labels a and b split the rows the same way (up to renaming)."""
    pairs = set(zip(a.tolist(), b.tolist()))
    return len(pairs) == len(set(a.tolist())) == len(set(b.tolist()))


def test_semantic_groups_follow_raw_vectors_not_responses():
    """Keys split in two along a direction no query sees (raw vectors far apart,
    responses identical) and in two along a direction the queries do see (small
    raw gap, large response gap).  Raw-vector k-means takes the first split; the
    response-coupled partition takes the second."""
    rng = np.random.default_rng(0)
    n, d = 64, 8
    hidden = np.repeat([0.0, 40.0], n // 2)                 # seen by no query
    seen = np.tile(np.repeat([-1.0, 1.0], n // 4), 2)       # seen by every query
    k = np.zeros((n, d))
    k[:, 0] = seen
    k[:, 1] = hidden
    k += 1e-3 * rng.standard_normal((n, d))
    q = np.zeros((n, d))
    q[:, 0] = 3.0 + 0.1 * rng.standard_normal(n)            # queries look along dim 0 only
    p = _params()
    sem = O.semantic_partition_head(q, k, p, 0)
    cou = O.partition_head(q, k, p, 0)
    assert _same_partition(sem.label_k, (hidden > 0).astype(np.int64))
    assert _same_partition(cou.label_k, (seen > 0).astype(np.int64))
    # both K/V groupings feed the same centroid / route machinery
    np.testing.assert_allclose(sem.centroids[sem.label_k[0]], k[sem.label_k == sem.label_k[0]].mean(axis=0))


def test_semantic_query_groups_are_raw_kmeans_clusters():
    """Queries in two tight raw clusters are grouped by those clusters."""
    rng = np.random.default_rng(1)
    n, d = 48, 6
    centre = np.where(np.arange(n) < 20, -5.0, 5.0)
    q = np.zeros((n, d))
    q[:, 2] = centre
    q += 0.01 * rng.standard_normal((n, d))
    k = rng.standard_normal((n, d))
    sem = O.semantic_partition_head(q, k, _params(), 0)
    assert _same_partition(sem.label_q, (centre > 0).astype(np.int64))
    assert sem.q_offsets[-1] == n and sorted(sem.perm_q.tolist()) == list(range(n))


def test_support_fraction_closed_forms():
    assert O.support_fraction(np.full(10, 0.1)) == 0.9
    assert O.support_fraction([0.5, 0.3, 0.15, 0.05]) == 0.75
    assert O.support_fraction([0.5, 0.3, 0.15, 0.05], mass=0.5) == 0.25
    assert O.support_fraction([0.05, 0.15, 0.5, 0.3], mass=0.8) == 0.5   # order of keys is irrelevant


def test_grouped_support_of_disjoint_and_identical_queries():
    """Two queries each spread evenly over their own 4 of 8 one-hot keys: each needs
    4/8 of the keys for 90%, their pooled distribution needs all 8.  A group of
    identical queries pools to the same distribution."""
    k = np.eye(8)
    big = 60.0
    q = np.zeros((2, 8))
    q[0, :4] = big
    q[1, 4:] = big
    per_q, pooled = O.grouped_support(q, k, 1.0, np.array([0, 0]), [0])
    assert abs(per_q - 0.5) < 1e-12 and abs(pooled - 1.0) < 1e-12
    q_same = np.vstack([q[0], q[0], q[0]])
    per_q, pooled = O.grouped_support(q_same, k, 1.0, np.array([0, 0, 0]), [0])
    assert per_q == pooled == 0.5


def test_affine_explainable_closed_forms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 5))
    b = rng.standard_normal(3)
    B = rng.standard_normal((5, 3))
    e, un = O.affine_explainable(x, b + x @ B)
    assert abs(e - 1.0) < 1e-10 and un < 1e-18
    # a residual orthogonal to span[1, x] is not explained at all
    xa = np.hstack([np.ones((40, 1)), x])
    qmat, _ = np.linalg.qr(xa)
    r = rng.standard_normal((40, 3))
    r -= qmat @ (qmat.T @ r)
    e, un = O.affine_explainable(x, r)
    assert abs(e) < 1e-10 and abs(un - (r ** 2).sum()) < 1e-9 * (r ** 2).sum()
