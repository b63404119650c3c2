"""GPU parity of the partition diagnostics the benchmark reports (huashangw.com article:
per-query versus grouped 90%-mass support, and the share of the residual an affine map
of the sparse output explains, in its comparison of grouping strategies): the bench's
device computation on the library's own outputs against the oracle's definitions on the
same partition and outputs, for the coupled partition, the semantic baseline and the
frame-causal call.  Support fractions are counts of keys over N: they agree to within
one key (plus the 5 decimals the bench reports); the explained share and the
unexplained energy to those 5 decimals."""
import numpy as np
import pytest

import bench
import oracle as O
from synth import generate, to_f64, to_torch, workload
from synth.video import frame_index

from helpers import params_dict
from test_gpu_parity import _np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,mode", [("tiny", 0), ("tiny", 1), ("tiny_causal", 0)])
def test_diagnostics_match_oracle(gpu, name, mode):
    import torch
    import free_block_sparse_rcp_b200 as spr
    w = workload(name)
    pd = params_dict(w, partition_mode=mode)
    frames = frame_index(w.grid).astype(np.int64) if w.frame_causal else None
    fid = None if frames is None else torch.from_numpy(frames.astype(np.int32)).to(gpu)
    p = spr.Params.make(**pd, frame_id=fid, n_frames=w.grid[0] if w.frame_causal else 0)
    qb, kb, vb = generate(w, seed=0)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    out = spr.run_call(p, Q, K, V)
    o_dense = torch.empty_like(Q)
    spr.sparsepr_dense_attention(p, Q, K, V, o_dense, None, out["ws"])
    torch.cuda.synchronize()
    heads = tuple(range(w.B * w.H))
    got = bench.partition_diagnostics(out, Q, K, out["o_sparse"], o_dense, p, frames, heads=heads,
                                      groups=pd["n_qgroups"])
    s = p.eff_scale()
    perq_sum = perq_n = pooled_sum = pooled_n = 0.0
    expl, unexpl = [], []
    for bh in heads:
        b, h = divmod(bh, w.H)
        q, k = to_f64(qb[b, h]), to_f64(kb[b, h])
        lq = _np(out["label_q"][bh]).astype(np.int64)
        groups = [a for a in range(pd["n_qgroups"]) if (lq == a).any()]
        pq, pooled = O.grouped_support(q, k, s, lq, groups, 0.9, frames)
        n_rows = sum(int((lq == a).sum()) for a in groups)
        perq_sum += pq * n_rows
        perq_n += n_rows
        pooled_sum += pooled * len(groups)
        pooled_n += len(groups)
        x = _np(out["o_sparse"][b, h]).astype(np.float64)
        r = _np(o_dense[b, h]).astype(np.float64) - x
        e, un = O.affine_explainable(x, r)
        expl.append(e)
        unexpl.append(un / float((r ** 2).sum()))
    one_key = 1.0 / w.N
    assert abs(got["per_query_support"] - perq_sum / perq_n) <= one_key + 1e-5
    assert abs(got["grouped_support"] - pooled_sum / pooled_n) <= one_key + 1e-5
    assert abs(got["affine_explainable"] - float(np.mean(expl))) <= 1e-5
    assert abs(got["unexplained_energy_rel"] - float(np.mean(unexpl))) <= 1e-5
