"""GPU parity: every output of the four C-ABI calls against the CPU oracle.

Integer outputs (sample rows, k-means seeds, labels, permutations, offsets, route,
tile mask, probe rows) are compared bit-exactly, labels with the near-tie
exemption (relative distance gap < 1e-5) after feeding the oracle the device's
fp32 coordinates, one Lloyd step at a time.  Floating-point outputs use the
tolerances O_sparse rel-L2 <= 5e-3 and max-abs <= 2e-2, reconstructed O rel-L2 <=
1e-2 against the oracle's reconstruction; intermediate fp32 quantities use the
tolerances written next to each check.
"""
import numpy as np
import pytest

import oracle as O
from synth import Workload, generate, to_f64, to_torch, workload

from helpers import (O_REL_L2, OS_MAX_ABS, OS_REL_L2, oracle_params, params_dict, rel_l2,
                     teacher_forced_kmeans)

pytestmark = pytest.mark.gpu


def _spr():
    import free_block_sparse_rcp_b200 as spr
    return spr


def _run(pd, qb, kb, vb, device, trace=True):
    import torch
    spr = _spr()
    p = spr.Params.make(**pd)
    Q, K, V = (to_torch(x, device) for x in (qb, kb, vb))
    out = spr.run_call(p, Q, K, V, trace=trace)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
    return p, out


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype.is_floating_point and t.dtype != __import__("torch").float64 \
        else t.detach().cpu().numpy()


def _lse_close(got, ref, tol):
    """LSE parity; a row with no usable key (frame-causal) must be -inf on both sides."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    np.testing.assert_array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    assert np.isfinite(got[fin]).all()
    if fin.any():
        assert np.abs(got[fin] - ref[fin]).max() <= tol * max(1.0, np.abs(ref[fin]).max())


def stage_checks(pd, qb, kb, vb, out, heads, rows=None, check_kmeans=True, frames=None):
    """Per-stage parity of heads `heads` (flattened b*H + h).  rows: number of sampled
    query rows for the attention / reconstruction checks (None = all).  frames: frame of
    each token for a frame-causal call (None = no mask).  pd["partition_mode"] == 1: the
    semantic-grouping baseline (both k-means on the raw rows; no metric or eigen stage)."""
    semantic = pd.get("partition_mode", 0) == 1
    op = oracle_params(pd)
    B, H, N, d = pd["B"], pd["H"], pd["N"], pd["d"]
    s = op.eff_scale(d)
    tr = out["trace"]
    ptr = out["probe_trace"]
    T = pd["kmeans_iters"]
    rng = np.random.default_rng(123)
    for bh in heads:
        b, h = divmod(bh, H)
        q, k, v = to_f64(qb[b, h]), to_f64(kb[b, h]), to_f64(vb[b, h])
        if semantic:
            y_gpu = k   # the key k-means runs on the raw rows
        else:
            y_gpu = _metric_eigen_checks(pd, q, k, tr, bh, N)
        _rest_checks(pd, op, q, k, v, s, tr, ptr, out, bh, b, h, y_gpu, N, T, rng, rows, check_kmeans, frames,
                     semantic)


def _metric_eigen_checks(pd, q, k, tr, bh, N):
    if True:
        # --- a1/a2: sample and metric
        idx = O.sample_queries(N, pd["n_samples"], pd["seed"], bh)
        np.testing.assert_array_equal(_np(tr["sample_idx"][bh]), idx)
        mk = O.key_metric(q[idx])
        mk_gpu = _np(tr["metric"][bh]).astype(np.float64)
        assert np.abs(mk_gpu - mk).max() <= 1e-5 * np.abs(mk).max()
        # --- a3: eigenpairs of the device metric (invariants; sign/rotation free)
        lam_gpu = _np(tr["eigval"][bh]).astype(np.float64)
        u_gpu = _np(tr["eigvec"][bh]).astype(np.float64)
        lam_ref, _ = O.top_eigenpairs(mk_gpu, pd["eig_rank"])
        # the solver runs in fp64 on the fp32 metric; its outputs are rounded to fp32, so the
        # errors are O(sqrt(d) 2^-24) relative to ||M_K|| = lam_ref[0]
        assert np.abs(lam_gpu - lam_ref).max() <= 1e-5 * lam_ref[0]
        assert np.abs(u_gpu.T @ u_gpu - np.eye(pd["eig_rank"])).max() <= 1e-5
        resid = mk_gpu @ u_gpu - u_gpu * lam_gpu
        assert np.abs(resid).max() <= 2e-5 * lam_ref[0]
        # --- a4: key coordinates from the device eigenpairs
        y_gpu = _np(tr["key_coords"][bh]).astype(np.float64)
        y_ref = O.key_coords(k, lam_gpu, u_gpu)
        assert np.abs(y_gpu - y_ref).max() <= 1e-5 * np.abs(y_ref).max()
    return y_gpu


def _rest_checks(pd, op, q, k, v, s, tr, ptr, out, bh, b, h, y_gpu, N, T, rng, rows, check_kmeans, frames,
                 semantic):
    if True:
        # --- a5: key k-means on the device coordinates
        kinit = O.kmeans_init(N, pd["n_kgroups"], pd["seed"], bh, O.STREAM_KEY_KMEANS)
        np.testing.assert_array_equal(_np(tr["key_init"][bh]), kinit)
        lk = _np(out["label_k"][bh]).astype(np.int64)
        if check_kmeans:
            iters = [_np(tr["key_label_iters"][t, bh]).astype(np.int64) for t in range(T)]
            np.testing.assert_array_equal(iters[-1], lk)
            teacher_forced_kmeans(y_gpu, kinit, iters, f"keys head {bh}")
        # --- a10 (keys): permutation and offsets
        pk, ko = O.group_permutation(lk, pd["n_kgroups"])
        np.testing.assert_array_equal(_np(out["perm_k"][bh]), pk)
        np.testing.assert_array_equal(_np(out["koff"][bh]), ko)
        # --- a6: K/V group centroids
        c_ref, n_k = O.group_means(k, lk, pd["n_kgroups"])
        c_gpu = _np(tr["key_centroids"][bh]).astype(np.float64)
        assert np.abs(c_gpu - c_ref).max() <= 1e-5 * max(1.0, np.abs(c_ref).max())
        # --- a7: query coordinates from the device centroids
        z_gpu = _np(tr["query_coords"][bh]).astype(np.float64)
        z_ref = O.query_coords(q, c_gpu, s)
        assert np.abs(z_gpu - z_ref).max() <= 2e-5 * max(1.0, np.abs(z_ref).max())
        zk = q if semantic else z_gpu   # the query k-means runs on the raw rows in the baseline
        # --- a8: query k-means on the device coordinates
        qinit = O.kmeans_init(N, pd["n_qgroups"], pd["seed"], bh, O.STREAM_QUERY_KMEANS)
        np.testing.assert_array_equal(_np(tr["query_init"][bh]), qinit)
        lq = _np(out["label_q"][bh]).astype(np.int64)
        if check_kmeans:
            iters = [_np(tr["query_label_iters"][t, bh]).astype(np.int64) for t in range(T)]
            np.testing.assert_array_equal(iters[-1], lq)
            teacher_forced_kmeans(zk, qinit, iters, f"queries head {bh}")
        pq, qo = O.group_permutation(lq, pd["n_qgroups"])
        np.testing.assert_array_equal(_np(out["perm_q"][bh]), pq)
        np.testing.assert_array_equal(_np(out["qoff"][bh]), qo)
        n_q = np.diff(qo)
        # --- a9: cell mass and route (route bit-exact given the device's fp32 masses)
        m_gpu = _np(tr["cell_mass"][bh]).astype(np.float64)
        if frames is None:
            m_ref = O.cell_mass(z_gpu, lq, n_k, pd["n_qgroups"])
            cost = visible = None
        else:
            nf = int(frames.max()) + 1
            vis_k = O.visible_counts(lk, frames, pd["n_kgroups"], nf)
            hist_q = O.frame_histogram(lq, frames, pd["n_qgroups"], nf)
            m_ref = O.cell_mass(z_gpu, lq, n_k, pd["n_qgroups"], frames, vis_k)
            cost = O.cell_cost(n_q, n_k, hist_q, vis_k)
            visible = float(hist_q.sum(axis=0) @ vis_k.sum(axis=0))
        assert np.abs(m_gpu - m_ref).max() <= 2e-5
        rr = O.route_select(m_gpu, n_q, n_k, op.density, pd["n_probes"], N, cost=cost, visible=visible)
        route = _np(out["route"][bh])
        np.testing.assert_array_equal(route, rr.route)
        assert _np(tr["alpha"])[bh] == rr.alpha
        assert abs(float(_np(out["rho_exec"])[bh]) - rr.rho_exec) <= 1e-6
        bm = O.block_mask(rr.route, lq, pq, lk, pk, pd["block"])
        np.testing.assert_array_equal(_np(out["block_mask"][bh]), bm)
        # --- a11: routed attention (sampled rows, original order)
        sel = np.arange(N) if rows is None or rows >= N else np.sort(rng.choice(N, rows, replace=False))
        o_ref, l_ref = O.sparse_attention(q, k, v, s, rr.route, lq, lk, rows=sel, frames=frames)
        o_gpu = _np(out["o_sparse"][b, h])[sel].astype(np.float64)
        l_gpu = _np(out["lse"][bh])[sel].astype(np.float64)
        assert rel_l2(o_gpu, o_ref) <= OS_REL_L2, rel_l2(o_gpu, o_ref)
        assert np.abs(o_gpu - o_ref).max() <= OS_MAX_ABS
        _lse_close(l_gpu, l_ref, 2e-3)
        # --- a12/a13: probes
        pidx = O.pick_probes(pq, qo, pd["n_probes"], pd["seed"], bh)
        np.testing.assert_array_equal(_np(out["probe_idx"][bh]), pidx)
        od_ref, ld_ref = O.attention(q[pidx], k, v, s,
                                     mask=None if frames is None else O.causal_mask(frames, pidx))
        os_ref, ls_ref = O.sparse_attention(q, k, v, s, rr.route, lq, lk, rows=pidx, frames=frames)
        od_gpu = _np(out["probe_o_dense"][bh]).astype(np.float64)
        os_gpu = _np(ptr["probe_o_sparse"][bh]).astype(np.float64)
        assert rel_l2(od_gpu, od_ref) <= 1e-5 and rel_l2(os_gpu, os_ref) <= 1e-5
        _lse_close(_np(ptr["probe_lse_dense"][bh]), ld_ref, 1e-4)
        _lse_close(_np(ptr["probe_lse_sparse"][bh]), ls_ref, 1e-4)
        # --- a14: the device's residual subspace (from its own probe outputs): singular values
        # against the oracle's, an orthonormal basis of an invariant subspace of R^T R.  The
        # basis itself is not compared: its trailing directions are weak (down to ~3e-4 of
        # the largest at rank 32) and can rotate with the last bits of the inputs.
        r_gpu = od_gpu - os_gpu
        fit_dev = O.fit_from_probes(pidx, od_gpu, os_gpu, ld_ref, ls_ref, pd["sub_rank"], op.ridge_lambda)
        # (the singular values do not depend on the fit's weights)
        sig_gpu = _np(ptr["sigma"][bh]).astype(np.float64)
        s0 = max(fit_dev.sigma[0], 1e-30)
        assert np.abs(sig_gpu - fit_dev.sigma).max() <= 1e-5 * s0 + 1e-9
        b_gpu = _np(out["b_full"][bh]).astype(np.float64)
        vr_gpu = _np(out["Vr"][bh]).astype(np.float64)
        w_gpu = _np(out["W"][bh]).astype(np.float64)
        bm_gpu = _np(out["Bmat"][bh]).astype(np.float64)
        assert np.all(vr_gpu[:, sig_gpu == 0] == 0)
        # v_j = R^T u_j / sigma_j magnifies the error of u_j by sigma_0 / sigma_j, so the basis
        # is checked on the directions above 1e-3 sigma_0 (the weaker ones carry targets below
        # 1e-3 of the largest and barely move the correction)
        # (and above 1e-6 absolute: below that R is the fp32 rounding of the probe outputs)
        keep = sig_gpu > max(1e-3 * s0, 1e-6)
        if keep.any():
            vk = vr_gpu[:, keep]
            assert np.abs(vk.T @ vk - np.eye(vk.shape[1])).max() <= 1e-4
            inv = r_gpu.T @ (r_gpu @ vk) - vk * sig_gpu[keep] ** 2
            assert np.abs(inv).max() <= 1e-5 * s0 ** 2
        # --- a15: the ridge given the device's subspace (exact up to fp32 rounding); its input
        # is the whole sparse output row (fit_input 0) or its projection on V_r (fit_input 1)
        wts = O.probe_weights(qo, pd["n_probes"]) if op.fit_weighted else None
        if op.fit_input == "full":
            w_fit, b_sub = O.ridge_fit(os_gpu, r_gpu @ vr_gpu, op.ridge_lambda, wts)
        else:
            w_sub, b_sub = O.ridge_fit(os_gpu @ vr_gpu, r_gpu @ vr_gpu, op.ridge_lambda, wts)
            w_fit = vr_gpu @ w_sub
        bfull_ref = vr_gpu @ b_sub
        bmat_ref = w_fit @ vr_gpu.T
        np.testing.assert_allclose(bm_gpu, w_gpu @ vr_gpu.T, atol=1e-5 * max(1, np.abs(bm_gpu).max()))
        corr_gpu = b_gpu + o_ref @ bm_gpu
        corr_ref = bfull_ref + o_ref @ bmat_ref
        dc = np.linalg.norm(corr_gpu - corr_ref)
        assert dc <= 1e-4 * np.linalg.norm(o_ref) + 1e-3 * np.linalg.norm(corr_ref), \
            (dc, np.linalg.norm(corr_ref), np.linalg.norm(o_ref))
        # --- a16: reconstruction against the oracle's correction with the device's fit
        o_rows_ref = o_ref + bfull_ref + o_ref @ bmat_ref
        slot = {int(i): j for j, i in enumerate(pidx)}
        for r_, i in enumerate(sel):
            if int(i) in slot:
                o_rows_ref[r_] = od_ref[slot[int(i)]]
        o_rows_gpu = _np(out["o"][b, h])[sel].astype(np.float64)
        assert rel_l2(o_rows_gpu, o_rows_ref) <= O_REL_L2, rel_l2(o_rows_gpu, o_rows_ref)
        if rows is None:
            o_all = _np(out["o"][b, h]).astype(np.float64)
            np.testing.assert_allclose(o_all[pidx], od_ref, atol=1e-2 * max(1, np.abs(od_ref).max()))


CASES = {
    "tiny": dict(name="tiny"),
    "tiny_weighted": dict(name="tiny", fit_weighted=1),
    "mid25_weighted": dict(name="mid", density=0.25, fit_weighted=1),
    "mid15": dict(name="mid", density=0.15),
    "mid25": dict(name="mid", density=0.25),
    "mid40": dict(name="mid", density=0.40),
}


def _ragged_workload():
    # d = 128, N = 1900 (not a multiple of any tile), odd group counts
    return Workload(name="ragged", B=2, H=2, grid=(5, 19, 20), d=128, n_centroids=24, n_seeds=40, block=128,
                    density=0.3, n_kgroups=13, n_qgroups=11, n_samples=128, n_probes=64, eig_rank=32,
                    sub_rank=32, kmeans_iters=6, centroid_scale=1.0)


@pytest.mark.parametrize("case", list(CASES))
def test_stage_parity(gpu, case):
    c = dict(CASES[case])
    w = workload(c.pop("name"))
    pd = params_dict(w, **c)
    heads = range(w.B * w.H)
    if w.name == "mid":
        heads = [0, 5, 11]
    qb, kb, vb = generate(w, seed=0, heads=[divmod(x, w.H) for x in heads])
    _, out = _run(pd, qb, kb, vb, gpu)
    stage_checks(pd, qb, kb, vb, out, heads, rows=None if w.name == "tiny" else 1024)


@pytest.mark.parametrize("weighted", [0, 1])
def test_stage_parity_ragged_d128(gpu, weighted):
    w = _ragged_workload()
    pd = params_dict(w, fit_weighted=weighted)
    qb, kb, vb = generate(w, seed=3)
    _, out = _run(pd, qb, kb, vb, gpu)
    stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None)


def test_tiny_end_to_end_against_oracle(gpu):
    """The oracle's own partition (fp64 coordinates) reaches the same groups, route
    and probes as the device on the 1024-token workload, and the outputs agree."""
    w = workload("tiny")
    pd = params_dict(w)
    op = oracle_params(pd)
    qb, kb, vb = generate(w, seed=0)
    _, out = _run(pd, qb, kb, vb, gpu)
    for h in range(w.H):
        ref = O.sparsepr_head(to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h]), op, h)
        np.testing.assert_array_equal(_np(out["label_k"][h]), ref.part.label_k)
        np.testing.assert_array_equal(_np(out["label_q"][h]), ref.part.label_q)
        np.testing.assert_array_equal(_np(out["route"][h]), ref.part.route.route)
        np.testing.assert_array_equal(_np(out["probe_idx"][h]), ref.fit.probe_idx)
        os_gpu = _np(out["o_sparse"][0, h]).astype(np.float64)
        assert rel_l2(os_gpu, ref.o_sparse) <= OS_REL_L2
        assert np.abs(os_gpu - ref.o_sparse).max() <= OS_MAX_ABS
        assert rel_l2(_np(out["o"][0, h]), ref.o) <= O_REL_L2


def test_dense_attention_matches_oracle(gpu):
    import torch
    spr = _spr()
    for w in (workload("tiny"), _ragged_workload()):
        pd = params_dict(w)
        p = spr.Params.make(**pd)
        qb, kb, vb = generate(w, seed=1)
        Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
        o = torch.empty_like(Q)
        lse = torch.empty(p.BH, p.N, dtype=torch.float32, device=gpu)
        ws = spr.workspace(p, gpu)
        spr.sparsepr_dense_attention(p, Q, K, V, o, lse, ws)
        torch.cuda.synchronize()
        for bh in range(p.BH):
            b, h = divmod(bh, w.H)
            ref, lref = O.attention(to_f64(qb[b, h]), to_f64(kb[b, h]), to_f64(vb[b, h]), 1 / np.sqrt(w.d))
            got = _np(o[b, h]).astype(np.float64)
            assert rel_l2(got, ref) <= OS_REL_L2 and np.abs(got - ref).max() <= OS_MAX_ABS
            assert np.abs(_np(lse[bh]) - lref).max() <= 2e-3 * max(1, np.abs(lref).max())


def test_full_density_is_dense(gpu):
    """density 1 routes every cell: O_sparse = dense attention, zero residual, and the
    correction leaves the sparse output unchanged."""
    w = workload("tiny")
    pd = params_dict(w, density=1.0)
    qb, kb, vb = generate(w, seed=2)
    _, out = _run(pd, qb, kb, vb, gpu)
    for h in range(w.H):
        q, k, v = to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h])
        ref, _ = O.attention(q, k, v, 1 / np.sqrt(w.d))
        os_gpu = _np(out["o_sparse"][0, h]).astype(np.float64)
        assert rel_l2(os_gpu, ref) <= OS_REL_L2
        nk = np.diff(_np(out["koff"][h]))
        nq = np.diff(_np(out["qoff"][h]))
        np.testing.assert_array_equal(_np(out["route"][h]), np.outer(nq > 0, nk > 0).astype(np.uint8))
        assert float(_np(out["rho_exec"])[h]) >= 1.0
        np.testing.assert_array_equal(_np(out["b_full"][h]), 0)
        np.testing.assert_array_equal(_np(out["W"][h]), 0)
        pidx = _np(out["probe_idx"][h])
        rest = np.setdiff1d(np.arange(w.N), pidx)
        np.testing.assert_array_equal(_np(out["o"][0, h])[rest], os_gpu[rest])


@pytest.mark.parametrize("kw", [
    dict(N=37, grid=(1, 1, 37), groups=(5, 4), probes=8, samples=37, density=0.8),
    dict(N=300, grid=(3, 10, 10), groups=(1, 1), probes=20, samples=64, density=0.5),
    dict(N=256, grid=(4, 8, 8), groups=(16, 16), probes=64, samples=64, density=0.5),  # empty clusters likely
    dict(N=1024, grid=(4, 16, 16), groups=(8, 8), probes=64, samples=64, density=64 / 1024 + 1e-3),
])
def test_edge_cases(gpu, kw):
    gk, gq = kw["groups"]
    w = Workload(name="edge", B=1, H=2, grid=kw["grid"], d=64, n_centroids=8, n_seeds=8, block=64,
                 density=kw["density"], n_kgroups=gk, n_qgroups=gq, n_samples=kw["samples"],
                 n_probes=kw["probes"], eig_rank=16, sub_rank=min(16, kw["probes"]), kmeans_iters=4,
                 centroid_scale=1.0)
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=7)
    _, out = _run(pd, qb, kb, vb, gpu)
    stage_checks(pd, qb, kb, vb, out, range(w.H), rows=None)


def test_deterministic(gpu):
    w = workload("tiny")
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=4)
    _, a = _run(pd, qb, kb, vb, gpu, trace=False)
    _, b = _run(pd, qb, kb, vb, gpu, trace=False)
    for key in ("perm_q", "perm_k", "route", "o_sparse", "o", "probe_idx", "W", "Vr", "b_full"):
        assert bool((a[key] == b[key]).all()), key
