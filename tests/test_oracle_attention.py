"""Pins for the oracle's dense / masked attention and the residual identity."""
import math

import numpy as np
import pytest

import oracle as O


def _brute(q, k, v, scale, mask=None):
    # direct per-row loops, textbook softmax(scale * q.k) v
    nq, nk = len(q), len(k)
    out = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for i in range(nq):
        logits = []
        for j in range(nk):
            if mask is None or mask[i][j]:
                logits.append((j, scale * sum(q[i][c] * k[j][c] for c in range(q.shape[1]))))
        if not logits:
            continue
        m = max(l for _, l in logits)
        z = sum(math.exp(l - m) for _, l in logits)
        for j, l in logits:
            out[i] += math.exp(l - m) / z * v[j]
        lse[i] = m + math.log(z)
    return out, lse


@pytest.fixture
def small():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((7, 5))
    k = rng.standard_normal((9, 5))
    v = rng.standard_normal((9, 3))
    return q, k, v


def test_dense_matches_brute_force(small):
    q, k, v = small
    o, l = O.attention(q, k, v, 0.37)
    ob, lb = _brute(q, k, v, 0.37)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l, lb, rtol=1e-12)


def test_masked_matches_brute_force_and_empty_rows(small):
    q, k, v = small
    rng = np.random.default_rng(1)
    mask = rng.random((7, 9)) < 0.4
    mask[3] = False  # a row with no key
    o, l = O.attention(q, k, v, 1 / math.sqrt(5), mask=mask, chunk=3)
    ob, lb = _brute(q, k, v, 1 / math.sqrt(5), mask)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-12)
    assert np.all(o[3] == 0) and l[3] == -np.inf
    np.testing.assert_allclose(l[np.isfinite(lb)], lb[np.isfinite(lb)], rtol=1e-12)


def test_full_route_is_dense():
    # density 100% => sparse attention equals dense attention
    rng = np.random.default_rng(2)
    q, k, v = rng.standard_normal((3, 40, 8))
    lq = rng.integers(0, 4, 40)
    lk = rng.integers(0, 5, 40)
    route = np.ones((4, 5), np.uint8)
    o1, l1 = O.sparse_attention(q, k, v, 0.3, route, lq, lk)
    o2, l2 = O.attention(q, k, v, 0.3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_residual_identity():
    # huashangw.com, retained mass vs output error: the residual of a row equals
    # omitted mass x (output over omitted keys - output over retained keys)
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((3, 30, 6))
    lq = rng.integers(0, 3, 30)
    lk = rng.integers(0, 4, 30)
    route = (rng.random((3, 4)) < 0.5).astype(np.uint8)
    route[:, 0] = 1
    o_d, l_d = O.attention(q, k, v, 0.5)
    o_s, l_s = O.sparse_attention(q, k, v, 0.5, route, lq, lk)
    keep = O.pair_mask(route, lq, lk)
    o_om, l_om = O.attention(q, k, v, 0.5, mask=~keep)
    m = O.omitted_mass(l_s, l_d)
    has_om = np.isfinite(l_om)
    r = o_d - o_s
    np.testing.assert_allclose(r[has_om], m[has_om, None] * (o_om - o_s)[has_om], atol=1e-12)
    np.testing.assert_allclose(r[~has_om], 0, atol=1e-12)
    # omitted mass from the partition functions: Z_om / Z
    np.testing.assert_allclose(m[has_om], np.exp(l_om[has_om] - l_d[has_om]), rtol=1e-10)


def test_lse_merge():
    # dense = merge of retained and omitted parts by their partition functions
    rng = np.random.default_rng(4)
    q, k, v = rng.standard_normal((3, 25, 4))
    keep = rng.random((25, 25)) < 0.5
    keep[:, 0] = True
    keep[:, 1] = False
    o_r, l_r = O.attention(q, k, v, 0.8, mask=keep)
    o_o, l_o = O.attention(q, k, v, 0.8, mask=~keep)
    o_d, l_d = O.attention(q, k, v, 0.8)
    lse = np.logaddexp(l_r, l_o)
    np.testing.assert_allclose(lse, l_d, rtol=1e-12)
    merged = (np.exp(l_r - lse)[:, None] * o_r + np.exp(l_o - lse)[:, None] * o_o)
    np.testing.assert_allclose(merged, o_d, atol=1e-12)
