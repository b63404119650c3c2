"""GPU parity of the semantic-grouping baseline (partition_mode = 1: keys and queries
clustered separately on their raw rows; huashangw.com article, comparison of grouping
strategies) against the oracle, through the C ABI.  The checks after the two k-means
are those of the response-coupled path."""
import numpy as np
import pytest

import oracle as O
from synth import generate, to_f64, workload

from helpers import O_REL_L2, OS_MAX_ABS, OS_REL_L2, oracle_params, params_dict, rel_l2
from test_gpu_parity import _np, _ragged_workload, _run, stage_checks

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["tiny", "mid25"])
def test_semantic_stage_parity(gpu, case):
    w = workload("tiny" if case == "tiny" else "mid")
    pd = params_dict(w, partition_mode=1, **({} if case == "tiny" else dict(density=0.25)))
    heads = range(w.B * w.H) if case == "tiny" else [0, 7]
    qb, kb, vb = generate(w, seed=0, heads=[divmod(x, w.H) for x in heads])
    _, out = _run(pd, qb, kb, vb, gpu)
    stage_checks(pd, qb, kb, vb, out, heads, rows=None if case == "tiny" else 1024)


def test_semantic_stage_parity_ragged_d128(gpu):
    w = _ragged_workload()
    pd = params_dict(w, partition_mode=1)
    qb, kb, vb = generate(w, seed=3)
    _, out = _run(pd, qb, kb, vb, gpu)
    stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None)


def test_semantic_end_to_end_against_oracle(gpu):
    """The oracle's semantic partition (fp64) reaches the same groups and route as the
    device on the 1024-token workload, and the outputs agree."""
    w = workload("tiny")
    pd = params_dict(w, partition_mode=1)
    op = oracle_params(pd)
    qb, kb, vb = generate(w, seed=0)
    _, out = _run(pd, qb, kb, vb, gpu)
    for h in range(w.H):
        q, k, v = to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h])
        part = O.semantic_partition_head(q, k, op, h)
        np.testing.assert_array_equal(_np(out["label_k"][h]), part.label_k)
        np.testing.assert_array_equal(_np(out["label_q"][h]), part.label_q)
        np.testing.assert_array_equal(_np(out["route"][h]), part.route.route)
        s = op.eff_scale(w.d)
        o_s, _ = O.sparse_attention(q, k, v, s, part.route.route, part.label_q, part.label_k)
        fit = O.probe_fit_head(q, k, v, part.label_q, part.label_k, part.route.route, part.perm_q, part.q_offsets,
                               op, h)
        os_gpu = _np(out["o_sparse"][0, h]).astype(np.float64)
        assert rel_l2(os_gpu, o_s) <= OS_REL_L2 and np.abs(os_gpu - o_s).max() <= OS_MAX_ABS
        assert rel_l2(_np(out["o"][0, h]), O.correct(o_s, fit)) <= O_REL_L2
