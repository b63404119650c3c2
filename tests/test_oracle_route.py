"""Pins for the oracle's cell-mass estimate and budgeted route.

The selection rule itself is a reading (the pages fix only alpha as the target
retained mass and the cost as the product of group sizes): parity unpinned for
the rule; these tests pin its invariants and its arithmetic."""
import numpy as np
import pytest

import oracle as O


def _case(seed, gq=5, gk=6, n=300):
    rng = np.random.default_rng(seed)
    n_q = rng.multinomial(n, rng.dirichlet(np.ones(gq)))
    n_k = rng.multinomial(n, rng.dirichlet(np.ones(gk)))
    n_k[1] = 0
    mass = rng.dirichlet(np.ones(gk), size=gq)
    mass[:, 1] = 0
    mass /= mass.sum(axis=1, keepdims=True)
    return mass, n_q, n_k, n


def test_cell_mass_exact_for_identical_keys():
    # when all keys of a group are equal to their centroid the estimate
    # n_g exp(s q.c_g) is the exact partition sum of the group
    rng = np.random.default_rng(0)
    centers = rng.standard_normal((4, 5))
    lk = np.array([0] * 3 + [1] * 7 + [3] * 5)         # group 2 empty
    k = centers[lk]
    v = rng.standard_normal((len(k), 2))
    q = rng.standard_normal((6, 5))
    lq = np.array([0, 1, 0, 1, 1, 0])
    c, n_k = O.group_means(k, lk, 4)
    z = O.query_coords(q, c, 0.7)
    mass = O.cell_mass(z, lq, n_k, 2)
    _, lse = O.attention(q, k, v, 0.7)
    for a in range(2):
        for g in range(4):
            sel = lk == g
            if not sel.any():
                assert mass[a, g] == 0
                continue
            _, lg = O.attention(q[lq == a], k, v, 0.7, mask=np.broadcast_to(sel, (int((lq == a).sum()), len(k))))
            np.testing.assert_allclose(mass[a, g], np.exp(lg - lse[lq == a]).mean(), rtol=1e-12)
    np.testing.assert_allclose(mass.sum(axis=1), 1, rtol=1e-12)


def test_cell_mass_uniform_logits_is_size_share():
    z = np.zeros((4, 3))
    m = O.cell_mass(z, np.array([0, 0, 1, 1]), np.array([2, 6, 0]), 3)
    np.testing.assert_allclose(m[0], [0.25, 0.75, 0.0])
    assert np.all(m[2] == 0)   # empty query group


@pytest.mark.parametrize("seed", range(6))
def test_route_budget_and_brute_force_alpha(seed):
    mass, n_q, n_k, n = _case(seed)
    for rho in (0.2, 0.35, 0.6):
        rr = O.route_select(mass, n_q, n_k, rho, 4, n)
        cost = O.cell_cost(n_q, n_k)
        assert rr.routed_pairs == int((cost * rr.route).sum())
        # the probe rows' exact pairs are charged before any cell (gist 2.C)
        assert rr.budget == pytest.approx(rho * n * n - 4 * n, rel=1e-14)
        assert rr.rho_exec == pytest.approx((rr.routed_pairs + 4 * n) / n ** 2)
        # every non-empty query group has at least one cell; nothing on empty groups
        for a in range(len(n_q)):
            assert (rr.route[a].sum() >= 1) == (n_q[a] > 0)
        assert not rr.route[:, n_k == 0].any()
        # brute force over the breakpoints of the cost step function
        rows = [None if n_q[a] == 0 else
                (lambda cand: (cand[np.argsort(-mass[a, cand], kind="stable")]))(np.nonzero(n_k > 0)[0])
                for a in range(len(n_q))]
        bps = {0.0}
        for a, order in enumerate(rows):
            if order is not None:
                bps.update(np.cumsum(mass[a, order]).tolist())

        def sel(alpha):
            r = np.zeros_like(rr.route)
            for a, order in enumerate(rows):
                if order is None:
                    continue
                cm = np.cumsum(mass[a, order])
                hit = np.nonzero(cm >= alpha)[0]
                r[a, order[:max(1, hit[0] + 1 if hit.size else len(order))]] = 1
            return r

        feasible = [b for b in sorted(bps) if b <= 1.0 and (cost * sel(b)).sum() <= rr.budget]
        if feasible:
            assert rr.routed_pairs <= rr.budget
            assert rr.rho_exec <= rho + 1e-12
            np.testing.assert_array_equal(rr.route, sel(max(feasible)))
        else:
            assert rr.alpha == 0.0
            np.testing.assert_array_equal(rr.route, sel(0.0))


def test_route_monotone_and_full():
    mass, n_q, n_k, n = _case(11)
    prev = None
    for rho in np.linspace(0.05, 0.95, 19):
        r = O.route_select(mass, n_q, n_k, float(rho), 2, n).route
        if prev is not None:
            assert np.all(r >= prev)          # nested as the budget grows
        prev = r
    full = O.route_select(mass, n_q, n_k, 1.0, 2, n).route
    np.testing.assert_array_equal(full, np.outer(n_q > 0, n_k > 0).astype(np.uint8))
