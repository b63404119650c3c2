"""Write tests/golden/tiny_seed0.txt: the oracle's integer outputs for the
1024-token workload (seed 0).  Calls only oracle/ (and the input generator).

    python tests/golden/make_tiny_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle as O  # noqa: E402
from synth import generate, to_f64, workload  # noqa: E402


def oracle_params(w, **kw):
    p = dict(n_kgroups=w.n_kgroups, n_qgroups=w.n_qgroups, n_samples=w.n_samples,
             n_probes=w.n_probes, eig_rank=w.eig_rank, sub_rank=w.sub_rank,
             kmeans_iters=w.kmeans_iters, density=w.density, ridge_lambda=w.ridge_lambda,
             block=w.block, seed=0)
    p.update(kw)
    return O.Params(**p)


def rows():
    w = workload("tiny")
    qb, kb, vb = generate(w, 0)
    p = oracle_params(w)
    out = []
    for h in range(w.H):
        r = O.sparsepr_head(to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h]), p, h)
        out.append((f"head {h} sample_idx", r.part.sample_idx))
        out.append((f"head {h} label_k", r.part.label_k))
        out.append((f"head {h} label_q", r.part.label_q))
        out.append((f"head {h} route", r.part.route.route.ravel()))
        out.append((f"head {h} probe_idx", r.fit.probe_idx))
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_seed0.txt"), "w") as f:
        f.write("# oracle integer outputs, 1024-token workload, seed 0 "
                "(written by tests/golden/make_tiny_golden.py)\n")
        for name, arr in rows():
            f.write(name + ": " + " ".join(str(int(x)) for x in np.asarray(arr)) + "\n")
