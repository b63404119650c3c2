"""Pins for the oracle's probes, residual subspace, ridge fit and correction."""
import numpy as np
import pytest
import scipy.linalg
from sklearn.linear_model import Ridge

import oracle as O


def test_ridge_matches_library_ridge():
    # centred ridge with an unpenalised intercept is exactly sklearn's Ridge
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 20))
    y = rng.standard_normal((64, 5))
    for lam in (1e-3, 1e-2, 3.0):
        w, b = O.ridge_fit(x, y, lam)
        ref = Ridge(alpha=lam, fit_intercept=True, solver="cholesky").fit(x, y)
        np.testing.assert_allclose(w, ref.coef_.T, rtol=1e-8, atol=1e-10)
        np.testing.assert_allclose(b, ref.intercept_, rtol=1e-8, atol=1e-10)


def test_ridge_primal_equals_dual_and_limits():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128))       # more regressors than probes
    y = rng.standard_normal((64, 7))
    lam = 1e-2
    w, b = O.ridge_fit(x, y, lam)
    xc, yc = x - x.mean(0), y - y.mean(0)
    wp = np.linalg.solve(xc.T @ xc + lam * np.eye(128), xc.T @ yc)
    np.testing.assert_allclose(w, wp, rtol=1e-7, atol=1e-9)
    # lam -> infinity: slope vanishes, intercept is the mean
    w_inf, b_inf = O.ridge_fit(x, y, 1e12)
    assert np.abs(w_inf).max() < 1e-9
    np.testing.assert_allclose(b_inf, y.mean(0), atol=1e-9)


def test_ridge_recovers_planted_affine_map():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 10))
    w0 = rng.standard_normal((10, 3))
    b0 = rng.standard_normal(3)
    w, b = O.ridge_fit(x, b0 + x @ w0, 1e-12)
    np.testing.assert_allclose(w, w0, atol=1e-8)
    np.testing.assert_allclose(b, b0, atol=1e-8)


def test_subspace_eckart_young_and_projector():
    rng = np.random.default_rng(3)
    r_p = rng.standard_normal((64, 32)) @ np.diag(np.linspace(3, 0.1, 32))
    v, sig = O.probe_subspace(r_p, 8)
    np.testing.assert_allclose(v.T @ v, np.eye(8), atol=1e-12)
    ev = np.sort(scipy.linalg.eigvalsh(r_p.T @ r_p))[::-1]
    np.testing.assert_allclose(sig ** 2, ev[:8], rtol=1e-9)
    resid = r_p - r_p @ v @ v.T
    np.testing.assert_allclose((resid ** 2).sum(), ev[8:].sum(), rtol=1e-8)
    w_e, u_e = scipy.linalg.eigh(r_p.T @ r_p)
    top = u_e[:, np.argsort(-w_e)[:8]]
    np.testing.assert_allclose(v @ v.T, top @ top.T, atol=1e-9)


def test_subspace_rank_deficient_is_zero_columns():
    rng = np.random.default_rng(4)
    r_p = np.outer(rng.standard_normal(64), rng.standard_normal(16))   # rank 1
    v, sig = O.probe_subspace(r_p, 4)
    assert sig[0] > 0 and np.all(sig[1:] == 0) and np.all(v[:, 1:] == 0)
    v0, s0 = O.probe_subspace(np.zeros((64, 16)), 4)
    assert np.all(v0 == 0) and np.all(s0 == 0)


@pytest.mark.parametrize("fit_input", O.FIT_INPUTS)
def test_correction_exact_for_planted_affine_residual(fit_input):
    # if the residual is exactly an affine map inside the probes' residual span,
    # R = (b + (x V) W) V^T with V the span's basis, the corrected output equals the
    # dense one on every row, whichever input the map takes (P = 64 > d + 1 probes)
    rng = np.random.default_rng(5)
    n, d, r, p = 400, 12, 3, 64
    basis = np.linalg.qr(rng.standard_normal((d, r)))[0]
    b_sub = rng.standard_normal(r)
    w_sub = rng.standard_normal((r, r))
    o_sparse = rng.standard_normal((n, d))
    o_dense = o_sparse + (b_sub + (o_sparse @ basis) @ w_sub) @ basis.T
    pidx = rng.choice(n, p, replace=False)
    fit = O.fit_from_probes(pidx, o_dense[pidx], o_sparse[pidx], np.zeros(p), np.zeros(p), r, 1e-12,
                            fit_input=fit_input)
    np.testing.assert_allclose(fit.vr @ fit.vr.T, basis @ basis.T, atol=1e-9)
    out = O.correct(o_sparse, fit)
    np.testing.assert_allclose(out, o_dense, atol=1e-7)
    np.testing.assert_allclose(fit.bmat, fit.w @ fit.vr.T)
    np.testing.assert_allclose(out[pidx], o_dense[pidx], atol=0)


def test_full_input_recovers_residual_driven_from_outside_the_subspace():
    # R = (b + x M) V^T with M acting on every component of x (gist 2.B: R ~ b + xB,
    # the correction projected on the subspace): the full-input map recovers it exactly
    # on every row; the subspace-input map only sees x V and cannot
    rng = np.random.default_rng(11)
    n, d, r, p = 500, 10, 3, 64
    basis = np.linalg.qr(rng.standard_normal((d, d)))[0]
    v, perp = basis[:, :r], basis[:, r:]
    m = perp @ rng.standard_normal((d - r, r))       # driven only by x's components outside V
    b0 = rng.standard_normal(r)
    o_sparse = rng.standard_normal((n, d))
    o_dense = o_sparse + (b0 + o_sparse @ m) @ v.T
    pidx = rng.choice(n, p, replace=False)
    full = O.fit_from_probes(pidx, o_dense[pidx], o_sparse[pidx], np.zeros(p), np.zeros(p), r, 1e-12,
                             fit_input="full")
    np.testing.assert_allclose(O.correct(o_sparse, full), o_dense, atol=1e-7)
    np.testing.assert_allclose(full.bmat, m @ v.T, atol=1e-8)
    sub = O.fit_from_probes(pidx, o_dense[pidx], o_sparse[pidx], np.zeros(p), np.zeros(p), r, 1e-12,
                            fit_input="subspace")
    rest = np.setdiff1d(np.arange(n), pidx)
    miss = np.linalg.norm(O.correct(o_sparse, sub)[rest] - o_dense[rest])
    assert miss > 0.5 * np.linalg.norm((o_sparse[rest] @ m) @ v.T)


@pytest.mark.parametrize("fit_input", O.FIT_INPUTS)
def test_fit_slope_is_the_primal_ridge_of_its_input(fit_input):
    # the fitted slope equals the primal ridge solution (Xc^T Xc + lam I)^-1 Xc^T Yc of
    # its reading's input (full x, or x V_r mapped back by V_r), Yc = centred R V_r, and
    # the intercept b = ybar - xbar W; this checks the dual solve the oracle uses
    rng = np.random.default_rng(12)
    p, d, r, lam = 64, 24, 6, 0.05
    o_s = rng.standard_normal((p, d))
    o_d = o_s + rng.standard_normal((p, d)) @ np.diag(np.linspace(2, 0.1, d))
    fit = O.fit_from_probes(np.arange(p), o_d, o_s, np.zeros(p), np.zeros(p), r, lam, fit_input=fit_input)
    y = (o_d - o_s) @ fit.vr
    x = o_s if fit_input == "full" else o_s @ fit.vr
    xc, yc = x - x.mean(0), y - y.mean(0)
    wp = np.linalg.solve(xc.T @ xc + lam * np.eye(x.shape[1]), xc.T @ yc)
    w_want = wp if fit_input == "full" else fit.vr @ wp
    np.testing.assert_allclose(fit.w, w_want, rtol=1e-8, atol=1e-10)
    np.testing.assert_allclose(fit.b, y.mean(0) - x.mean(0) @ wp, rtol=1e-8, atol=1e-10)


@pytest.mark.parametrize("fit_input", O.FIT_INPUTS)
def test_correction_lies_in_the_probe_residual_subspace(fit_input):
    # gist 2.B / hs method: whatever the input, the correction of any row falls in the
    # span of the retained singular directions of the probe residuals
    rng = np.random.default_rng(13)
    p, d, r = 64, 16, 4
    o_s = rng.standard_normal((p, d))
    o_d = o_s + rng.standard_normal((p, d))
    fit = O.fit_from_probes(np.arange(p), o_d, o_s, np.zeros(p), np.zeros(p), r, 1e-2, fit_input=fit_input)
    x = rng.standard_normal((50, d))
    corr = fit.b_full + x @ fit.bmat
    np.testing.assert_allclose(corr - corr @ fit.vr @ fit.vr.T, 0, atol=1e-10)


def test_fit_rejects_unknown_input():
    with pytest.raises(ValueError):
        O.fit_from_probes(np.arange(4), np.ones((4, 3)), np.zeros((4, 3)), np.zeros(4), np.zeros(4), 2, 1e-2,
                          fit_input="both")


def test_subspace_input_ignores_sparse_output_outside_the_subspace():
    # fit_input="subspace": the map's input is the sparse output projected on the residual
    # subspace, so adding to x any component orthogonal to V_r changes neither the fit nor
    # the correction
    rng = np.random.default_rng(6)
    n, d, r, p = 300, 10, 3, 48
    basis = np.linalg.qr(rng.standard_normal((d, d)))[0]
    v, perp = basis[:, :r], basis[:, r:]
    o_sparse = rng.standard_normal((n, d))
    o_dense = o_sparse + (rng.standard_normal(r) + (o_sparse @ v) @ rng.standard_normal((r, r))) @ v.T
    o_dense += 1e-3 * rng.standard_normal((n, d)) @ v @ v.T
    pidx = rng.choice(n, p, replace=False)
    fit = O.fit_from_probes(pidx, o_dense[pidx], o_sparse[pidx], np.zeros(p), np.zeros(p), r, 1e-2,
                            fit_input="subspace")
    shift = rng.standard_normal((n, d - r)) @ perp.T
    fit2 = O.fit_from_probes(pidx, o_dense[pidx] + shift[pidx], o_sparse[pidx] + shift[pidx], np.zeros(p),
                             np.zeros(p), r, 1e-2, fit_input="subspace")
    np.testing.assert_allclose(fit2.vr @ fit2.vr.T, fit.vr @ fit.vr.T, atol=1e-9)
    np.testing.assert_allclose(fit2.b_full, fit.b_full, atol=1e-9)
    np.testing.assert_allclose(fit2.bmat, fit.bmat, atol=1e-9)
    np.testing.assert_allclose(shift @ fit.bmat, 0, atol=1e-9)


def test_probe_rows_take_exact_dense_output():
    rng = np.random.default_rng(8)
    o_s = rng.standard_normal((50, 6))
    o_d = o_s + rng.standard_normal((50, 6))      # residual not affine: fit is inexact
    pidx = np.arange(0, 50, 3)
    fit = O.fit_from_probes(pidx, o_d[pidx], o_s[pidx], np.zeros(17), np.zeros(17), 3, 1e-2)
    out = O.correct(o_s, fit)
    np.testing.assert_array_equal(out[pidx], o_d[pidx])
    rest = np.setdiff1d(np.arange(50), pidx)
    np.testing.assert_allclose(out[rest], o_s[rest] + fit.b_full + o_s[rest] @ fit.bmat, atol=1e-12)


def test_zero_residual_leaves_sparse_output():
    rng = np.random.default_rng(6)
    o = rng.standard_normal((100, 8))
    pidx = np.arange(0, 100, 5)
    fit = O.fit_from_probes(pidx, o[pidx], o[pidx], np.zeros(20), np.zeros(20), 4, 1e-2)
    np.testing.assert_array_equal(O.correct(o, fit), o)


@pytest.mark.parametrize("sizes,p", [([10, 10, 10, 10], 64), ([100, 3, 0, 50, 7], 64),
                                     ([2, 1], 64), ([30] * 8, 64), ([9, 9, 9], 10),
                                     ([5, 1, 5, 1, 5], 7)])
def test_probe_allocation(sizes, p):
    sizes = np.array(sizes)
    alloc = O.probe_allocation(sizes, p)
    assert alloc.sum() == min(p, sizes.sum())
    assert np.all(alloc <= sizes) and np.all(alloc >= 0)
    open_ = alloc < sizes
    if open_.any():
        # groups with spare members differ by at most one probe, and no
        # saturated group holds more than an open group's share + 1
        assert alloc[open_].max() - alloc[open_].min() <= 1
        assert np.all(alloc[~open_] <= alloc[open_].max())
    # the leftover probe of the uneven case goes to the larger group first
    if list(sizes) == [9, 9, 9]:
        assert list(alloc) == [4, 3, 3]
    if list(sizes) == [5, 1, 5, 1, 5]:
        assert list(alloc) == [2, 1, 2, 1, 1]


def test_pick_probes_stratified_and_reproducible():
    rng = np.random.default_rng(7)
    lab = rng.integers(0, 8, 1000)
    perm, off = O.group_permutation(lab, 8)
    pidx = O.pick_probes(perm, off, 64, seed=5, bh=3)
    assert len(pidx) == 64 and len(set(pidx)) == 64
    counts = np.bincount(lab[pidx], minlength=8)
    assert list(counts) == list(O.probe_allocation(np.diff(off), 64))
    assert np.array_equal(pidx, O.pick_probes(perm, off, 64, seed=5, bh=3))
    assert not np.array_equal(pidx, O.pick_probes(perm, off, 64, seed=6, bh=3))
    # group order, then the stream's draw order inside each group
    g = O.SplitMix64(O.stream_state(5, 3, O.STREAM_PROBES))
    alloc = O.probe_allocation(np.diff(off), 64)
    want = []
    for a in range(8):
        mem = perm[off[a]:off[a + 1]]
        want += [int(mem[i]) for i in O.draw_without_replacement(g, len(mem), int(alloc[a]))]
    assert list(pidx) == want


def test_weighted_ridge_equals_replicated_rows():
    # integer weights act as replicated probe rows: with weights normalised to mean 1,
    # the weighted fit equals the plain fit on the replicated rows with lam * sum(w) / P
    rng = np.random.default_rng(9)
    x = rng.standard_normal((12, 4))
    y = rng.standard_normal((12, 2))
    rep = rng.integers(1, 4, 12)
    wn = rep * (12 / rep.sum())
    w1, b1 = O.ridge_fit(x, y, 0.3, wn)
    w2, b2 = O.ridge_fit(np.repeat(x, rep, axis=0), np.repeat(y, rep, axis=0), 0.3 * rep.sum() / 12)
    np.testing.assert_allclose(w1, w2, atol=1e-10)
    np.testing.assert_allclose(b1, b2, atol=1e-10)
    # equal weights are the plain fit
    w3, b3 = O.ridge_fit(x, y, 0.3, np.ones(12))
    w4, b4 = O.ridge_fit(x, y, 0.3)
    np.testing.assert_allclose(w3, w4, atol=1e-12)
    np.testing.assert_allclose(b3, b4, atol=1e-12)


def test_probe_weights_are_inverse_inclusion():
    # groups of 10, 3 and 50 tokens with 4 probes: allocation 1, 1, 2 (water-filling)
    qoff = np.array([0, 10, 13, 63])
    alloc = O.probe_allocation(np.diff(qoff), 4)
    w = O.probe_weights(qoff, 4)
    raw = np.concatenate([np.full(a, n / a) for n, a in zip(np.diff(qoff), alloc) if a > 0])
    np.testing.assert_allclose(w, raw * (raw.size / raw.sum()))
    assert abs(w.mean() - 1.0) < 1e-12
    # a probe of the big group stands for more tokens than one of the small group
    assert w[-1] > w[1]
