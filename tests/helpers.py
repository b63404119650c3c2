"""Shared helpers of the test-suite: workload -> params, and the oracle-side
parity checks (teacher-forced k-means, near-tie exemption)."""
from __future__ import annotations

import numpy as np

import oracle as O
from synth import workload

REL_TIE = 1e-5       # labels may differ only on ties with a relative distance gap below this
OS_REL_L2 = 5e-3     # O_sparse vs oracle
OS_MAX_ABS = 2e-2
O_REL_L2 = 1e-2      # reconstructed O vs oracle


def params_dict(w, **kw):
    d = dict(B=w.B, H=w.H, N=w.N, d=w.d, block=w.block, density=w.density, n_kgroups=w.n_kgroups,
             n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes, eig_rank=w.eig_rank,
             sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, ridge_lambda=w.ridge_lambda, scale=0.0, seed=0)
    d.update(kw)
    return d


def oracle_params(pd: dict) -> O.Params:
    """Oracle params from a C-ABI params dict (density/lambda go through float32 as on
    the device)."""
    return O.Params(n_kgroups=pd["n_kgroups"], n_qgroups=pd["n_qgroups"], n_samples=pd["n_samples"],
                    n_probes=pd["n_probes"], eig_rank=pd["eig_rank"], sub_rank=pd["sub_rank"],
                    kmeans_iters=pd["kmeans_iters"], density=float(np.float32(pd["density"])),
                    ridge_lambda=float(np.float32(pd["ridge_lambda"])), scale=float(np.float32(pd["scale"])),
                    seed=pd["seed"], block=pd["block"], fit_weighted=bool(pd.get("fit_weighted", 0)),
                    fit_input="subspace" if pd.get("fit_input", 0) == 1 else "full")


def check_labels_near_ties(x, mu, got, want, what=""):
    """got may differ from want (the oracle's argmin) only where the two clusters'
    distances are within REL_TIE of each other."""
    bad = np.nonzero(got != want)[0]
    if bad.size == 0:
        return 0
    xb = np.asarray(x, np.float64)[bad]
    dg = ((xb - mu[got[bad]]) ** 2).sum(axis=1)
    dw = ((xb - mu[want[bad]]) ** 2).sum(axis=1)
    gap = (dg - dw) / np.maximum(dw, 1e-300)
    assert np.all(gap <= REL_TIE), f"{what}: {bad.size} label mismatches, worst relative gap {gap.max():.3e}"
    return int(bad.size)


def teacher_forced_kmeans(x, init, label_iters, what=""):
    """Check every GPU assignment step against the oracle's argmin computed from the
    centroids the GPU's previous labels imply (fp64 means of the same fp32 points)."""
    x = np.asarray(x, np.float64)
    mu = x[np.asarray(init)].copy()
    ties = 0
    for t, got in enumerate(label_iters):
        got = np.asarray(got, np.int64)
        want = O.kmeans_assign(x, mu)
        ties += check_labels_near_ties(x, mu, got, want, f"{what} iter {t}")
        mu = O.kmeans_update(x, got, mu)
    return ties


def rel_l2(a, b):
    return O.rel_l2(a, b)
