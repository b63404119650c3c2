"""GPU parity of the frame-causal call (world-model rollout workload: a query of frame f
sees the keys of frames <= f, intersected with the route) against the oracle's
frame-causal path, through the C ABI.

The grouping is the same as without the mask; the cell mass, the cell costs, the
budget, the routed attention, the probe rows and the dense comparator use the mask.
Tolerances are those of the non-causal parity tests; rows left with no usable key
must give O = 0 and LSE = -inf on both sides.
"""
import numpy as np
import pytest

import oracle as O
from synth import Workload, generate, to_f64, to_torch, workload
from synth.video import frame_index

from helpers import O_REL_L2, OS_MAX_ABS, OS_REL_L2, oracle_params, params_dict, rel_l2
from test_gpu_parity import _np, _ragged_workload, stage_checks

pytestmark = pytest.mark.gpu


def _frames(w):
    return frame_index(w.grid).astype(np.int64)


def _run(pd, w, qb, kb, vb, device, frames=None, trace=True):
    import torch
    import free_block_sparse_rcp_b200 as spr
    fr = _frames(w) if frames is None else np.asarray(frames)
    fid = torch.from_numpy(fr.astype(np.int32)).to(device)
    p = spr.Params.make(**pd, frame_id=fid, n_frames=int(w.grid[0]))
    Q, K, V = (to_torch(x, device) for x in (qb, kb, vb))
    out = spr.run_call(p, Q, K, V, trace=trace)
    torch.cuda.synchronize()
    out["frame_tensor"] = fid
    return p, out


def _many_frames():
    # 16 frames of 64 tokens, small groups: rows whose routed groups hold no key of an
    # earlier or equal frame are likely (O = 0, LSE = -inf)
    return Workload(name="frames16", B=1, H=2, grid=(16, 8, 8), d=64, n_centroids=16, n_seeds=16, block=64,
                    density=0.2, n_kgroups=16, n_qgroups=16, n_samples=64, n_probes=64, eig_rank=16,
                    sub_rank=16, kmeans_iters=6, centroid_scale=1.0, frame_causal=True)


@pytest.mark.parametrize("density", [0.25, 0.15, 0.5])
def test_causal_stage_parity_tiny(gpu, density):
    import free_block_sparse_rcp_b200 as spr
    w = workload("tiny_causal")
    pd = params_dict(w, density=density)
    qb, kb, vb = generate(w, seed=0)
    p, out = _run(pd, w, qb, kb, vb, gpu)
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
    stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None, frames=_frames(w))


def test_causal_stage_parity_ragged_d128(gpu):
    import free_block_sparse_rcp_b200 as spr
    w = _ragged_workload()   # 5 frames of 380 tokens, N = 1900, odd group counts
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=3)
    p, out = _run(pd, w, qb, kb, vb, gpu)
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
    stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None, frames=_frames(w))


def test_causal_stage_parity_many_frames(gpu):
    import free_block_sparse_rcp_b200 as spr
    w = _many_frames()
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=5)
    p, out = _run(pd, w, qb, kb, vb, gpu)
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
    stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None, frames=_frames(w))


def test_causal_end_to_end_against_oracle(gpu):
    """The oracle's own frame-causal call (fp64 coordinates) reaches the same groups,
    route and probes as the device, and the outputs agree."""
    w = workload("tiny_causal")
    pd = params_dict(w)
    op = oracle_params(pd)
    fr = _frames(w)
    qb, kb, vb = generate(w, seed=0)
    _, out = _run(pd, w, qb, kb, vb, gpu)
    for h in range(w.H):
        ref = O.sparsepr_head(to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h]), op, h, frames=fr)
        np.testing.assert_array_equal(_np(out["label_k"][h]), ref.part.label_k)
        np.testing.assert_array_equal(_np(out["label_q"][h]), ref.part.label_q)
        np.testing.assert_array_equal(_np(out["route"][h]), ref.part.route.route)
        assert abs(float(_np(out["rho_exec"])[h]) - ref.part.route.rho_exec) <= 1e-6
        np.testing.assert_array_equal(_np(out["probe_idx"][h]), ref.fit.probe_idx)
        os_gpu = _np(out["o_sparse"][0, h]).astype(np.float64)
        assert rel_l2(os_gpu, ref.o_sparse) <= OS_REL_L2
        assert np.abs(os_gpu - ref.o_sparse).max() <= OS_MAX_ABS
        assert rel_l2(_np(out["o"][0, h]), ref.o) <= O_REL_L2


def _dense(spr, p, w, qb, kb, vb, device, fid):
    import torch
    Q, K, V = (to_torch(x, device) for x in (qb, kb, vb))
    o = torch.empty_like(Q)
    lse = torch.empty(p.BH, p.N, dtype=torch.float32, device=device)
    ws = spr.workspace(p, device)
    spr.sparsepr_workspace_clear_error(p, ws)
    spr.sparsepr_dense_attention(p, Q, K, V, o, lse, ws)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, ws) == 0
    return o, lse


def test_causal_dense_attention_matches_oracle(gpu):
    import torch
    import free_block_sparse_rcp_b200 as spr
    for w in (workload("tiny_causal"), _ragged_workload(), _many_frames()):
        pd = params_dict(w)
        fr = _frames(w)
        fid = torch.from_numpy(fr.astype(np.int32)).to(gpu)
        p = spr.Params.make(**pd, frame_id=fid, n_frames=int(w.grid[0]))
        qb, kb, vb = generate(w, seed=1)
        o, lse = _dense(spr, p, w, qb, kb, vb, gpu, fid)
        mask = O.causal_mask(fr)
        for bh in range(p.BH):
            b, h = divmod(bh, w.H)
            ref, lref = O.attention(to_f64(qb[b, h]), to_f64(kb[b, h]), to_f64(vb[b, h]), 1 / np.sqrt(w.d),
                                    mask=mask)
            got = _np(o[b, h]).astype(np.float64)
            assert rel_l2(got, ref) <= OS_REL_L2 and np.abs(got - ref).max() <= OS_MAX_ABS
            assert np.abs(_np(lse[bh]) - lref).max() <= 2e-3 * max(1, np.abs(lref).max())


def test_causal_full_density_is_causal_dense(gpu):
    """density 1 routes every cell: the routed output is the frame-causal dense output."""
    import free_block_sparse_rcp_b200 as spr
    w = workload("tiny_causal")
    pd = params_dict(w, density=1.0)
    qb, kb, vb = generate(w, seed=2)
    p, out = _run(pd, w, qb, kb, vb, gpu)
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
    mask = O.causal_mask(_frames(w))
    for h in range(w.H):
        q, k, v = to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h])
        ref, _ = O.attention(q, k, v, 1 / np.sqrt(w.d), mask=mask)
        os_gpu = _np(out["o_sparse"][0, h]).astype(np.float64)
        assert rel_l2(os_gpu, ref) <= OS_REL_L2
        assert float(_np(out["rho_exec"])[h]) >= 1.0
        np.testing.assert_array_equal(_np(out["W"][h]), 0)


@pytest.mark.parametrize("bad", ["decreasing", "out_of_range"])
def test_causal_invalid_frames_reported(gpu, bad):
    """Frame ids that decrease in token order or leave [0, n_frames) are reported as
    device error 5.  Every kernel clamps the ids it reads, so the call stays in bounds."""
    import free_block_sparse_rcp_b200 as spr
    w = workload("tiny_causal")
    pd = params_dict(w)
    fr = _frames(w).copy()
    if bad == "decreasing":
        fr[100] = 3
    else:
        fr[-1] = 7
    qb, kb, vb = generate(w, seed=0)
    p, out = _run(pd, w, qb, kb, vb, gpu, frames=fr, trace=False)
    assert spr.sparsepr_workspace_error(p, out["ws"]) == 5


def test_causal_deterministic(gpu):
    w = workload("tiny_causal")
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=4)
    _, a = _run(pd, w, qb, kb, vb, gpu, trace=False)
    _, b = _run(pd, w, qb, kb, vb, gpu, trace=False)
    for key in ("perm_q", "perm_k", "route", "o_sparse", "o", "probe_idx", "W", "Vr", "b_full", "rho_exec"):
        assert bool((a[key] == b[key]).all()), key
