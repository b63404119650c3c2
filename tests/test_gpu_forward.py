"""GPU parity of the whole call: the single entry points (sparsepr_forward on device
buffers, sparsepr_forward_host and sparsepr_forward_host_chunked from host buffers)
against the oracle's end-to-end path and against the four-call sequence, head-split
calls against the unsplit call, and both readings of the fit's input.

The pages state the call's interface as Q, K, V and a target density in, the
reconstructed attention output out (ai-feeds.com summary, method: inputs / outputs), and
every step as per head (huashangw.com method walkthrough: 64 probes per head), so a call
over a subset of heads, numbered by head_offset, must give those heads' outputs of the
whole call bit for bit.  Tolerances: reconstructed O rel-L2 <= 1e-2 against the oracle.
"""
import numpy as np
import pytest

import oracle as O
from synth import generate, to_f64, to_torch, workload
from synth.video import frame_index

from helpers import O_REL_L2, oracle_params, params_dict, rel_l2
from test_gpu_parity import _np, _ragged_workload, stage_checks

pytestmark = pytest.mark.gpu


def _spr():
    import free_block_sparse_rcp_b200 as spr
    return spr


def _forward(p, Q, K, V, dev):
    import torch
    spr = _spr()
    ws = spr.workspace(p, dev, forward=True)
    o = torch.empty_like(Q)
    rho = torch.empty(p.BH, dtype=torch.float32, device=dev)
    spr.sparsepr_forward(p, Q, K, V, o, rho, ws)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, ws) == 0
    return o, rho


def _pinned(t):
    import torch
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t.cpu())
    return h


def _oracle_o(pd, qb, kb, vb, frames=None):
    op = oracle_params(pd)
    B, H = pd["B"], pd["H"]
    return {(b, h): O.sparsepr_head(to_f64(qb[b, h]), to_f64(kb[b, h]), to_f64(vb[b, h]), op, b * H + h,
                                    frames=frames).o
            for b in range(B) for h in range(H)}


@pytest.mark.parametrize("name", ["tiny", "tiny_causal"])
def test_forward_matches_oracle(gpu, name):
    import torch
    spr = _spr()
    w = workload(name)
    pd = params_dict(w)
    qb, kb, vb = generate(w, seed=0)
    frames = frame_index(w.grid).astype(np.int64) if w.frame_causal else None
    fid = None if frames is None else torch.from_numpy(frames.astype(np.int32)).to(gpu)
    p = spr.Params.make(**pd, frame_id=fid, n_frames=w.grid[0] if w.frame_causal else 0)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    o, rho = _forward(p, Q, K, V, gpu)
    ref = _oracle_o(pd, qb, kb, vb, frames)
    for (b, h), o_ref in ref.items():
        got = _np(o[b, h]).astype(np.float64)
        assert rel_l2(got, o_ref) <= O_REL_L2, (b, h, rel_l2(got, o_ref))
    assert bool((rho > 0).all()) and bool((rho <= 1).all())


def test_forward_host_matches_oracle(gpu):
    import torch
    spr = _spr()
    w = workload("tiny")
    pd = params_dict(w)
    p = spr.Params.make(**pd)
    qb, kb, vb = generate(w, seed=1)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    Qh, Kh, Vh = (_pinned(t) for t in (Q, K, V))
    Oh = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    qkv = torch.empty((3,) + tuple(Q.shape), dtype=torch.bfloat16, device=gpu)
    o_dev = torch.empty_like(Q)
    ws = spr.workspace(p, gpu, forward=True)
    spr.sparsepr_forward_host(p, Qh, Kh, Vh, Oh, qkv, o_dev, ws)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, ws) == 0
    for (b, h), o_ref in _oracle_o(pd, qb, kb, vb).items():
        assert rel_l2(Oh[b, h].float().numpy().astype(np.float64), o_ref) <= O_REL_L2
    # the same bytes as the device entry point
    o, _ = _forward(p, Q, K, V, gpu)
    assert torch.equal(Oh, o.cpu())


def test_forward_equals_four_calls_bitwise(gpu):
    """sparsepr_forward runs the same kernels as partition -> attend -> probe_fit ->
    reconstruct on separate buffers: the outputs are the same bytes."""
    import torch
    spr = _spr()
    w = _ragged_workload()
    for fit_input in (0, 1):
        pd = params_dict(w, fit_input=fit_input)
        p = spr.Params.make(**pd)
        qb, kb, vb = generate(w, seed=3)
        Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
        four = spr.run_call(p, Q, K, V)
        o, rho = _forward(p, Q, K, V, gpu)
        assert torch.equal(o, four["o"]), fit_input
        assert torch.equal(rho, four["rho_exec"]), fit_input


def _head_chunk_case(gpu, w, n_chunks, seed):
    """Outputs of one call over all heads and of n_chunks calls over consecutive head
    ranges (head_offset = the range's first layer head), through the device entry point
    and through the chunked host pipeline."""
    import torch
    spr = _spr()
    pd = params_dict(w)
    p = spr.Params.make(**pd)
    qb, kb, vb = generate(w, seed=seed)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    o_all, rho_all = _forward(p, Q, K, V, gpu)
    BH, N, d = p.BH, p.N, p.d
    q3, k3, v3 = (t.view(BH, N, d) for t in (Q, K, V))
    per = -(-BH // n_chunks)
    o_split = torch.empty_like(o_all).view(BH, N, d)
    rho_split = torch.empty_like(rho_all)
    for h0 in range(0, BH, per):
        h1 = min(BH, h0 + per)
        pc = spr.Params.make(**dict(pd, B=1, H=h1 - h0, head_offset=h0))
        sl = [t[h0:h1].contiguous().view(1, h1 - h0, N, d) for t in (q3, k3, v3)]
        oc, rc = _forward(pc, *sl, gpu)
        o_split[h0:h1] = oc.view(h1 - h0, N, d)
        rho_split[h0:h1] = rc
    assert torch.equal(o_split.view_as(o_all), o_all)
    assert torch.equal(rho_split, rho_all)
    # the library's own pipeline over the same chunks, from pinned host buffers
    Qh, Kh, Vh = (_pinned(t) for t in (Q, K, V))
    Oh = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    qkv = torch.empty((3,) + tuple(Q.shape), dtype=torch.bfloat16, device=gpu)
    o_dev = torch.empty_like(Q)
    ws = spr.workspace(spr.chunk_params(p, n_chunks), gpu, forward=True)
    s_in, s_out = torch.cuda.Stream(gpu), torch.cuda.Stream(gpu)
    for rep in range(2):   # twice in a row on the same staging buffers
        Oh.fill_(0)
        spr.sparsepr_forward_host_chunked(p, Qh, Kh, Vh, Oh, qkv, o_dev, n_chunks, ws, s_in, s_out)
        torch.cuda.current_stream(gpu).synchronize()
        assert spr.sparsepr_workspace_error(spr.chunk_params(p, n_chunks), ws) == 0
        assert torch.equal(Oh, o_all.cpu()), rep


def test_head_chunks_equal_one_call_tiny(gpu):
    _head_chunk_case(gpu, workload("tiny"), 2, seed=6)


def test_head_chunks_equal_one_call_ragged_batches(gpu):
    # B = 2, H = 2: four chunks of one head, and two chunks that each hold one batch element
    _head_chunk_case(gpu, _ragged_workload(), 4, seed=7)
    _head_chunk_case(gpu, _ragged_workload(), 2, seed=7)


def test_head_chunks_equal_one_call_mid(gpu):
    # 12 heads of 8192 tokens: the k-means runs over many segments per CTA in the unsplit
    # call and over a different CTA layout in each chunk; its sums are per fixed segment
    _head_chunk_case(gpu, workload("mid"), 4, seed=8)


def test_head_offset_draws_the_layer_streams(gpu):
    """A call on one head with head_offset = h draws head h's random streams: its query
    sample, k-means seeds and probe rows are the oracle's for layer head h."""
    import torch
    spr = _spr()
    w = workload("tiny")
    pd = params_dict(w, H=1, head_offset=5, heads_total=8)
    qb, kb, vb = generate(w, seed=2)
    qb, kb, vb = (x[:, :1].copy() for x in (qb, kb, vb))
    p = spr.Params.make(**pd)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    out = spr.run_call(p, Q, K, V, trace=True)
    torch.cuda.synchronize()
    n = w.N
    np.testing.assert_array_equal(_np(out["trace"]["sample_idx"][0]), O.sample_queries(n, pd["n_samples"], 0, 5))
    np.testing.assert_array_equal(_np(out["trace"]["key_init"][0]),
                                  O.kmeans_init(n, pd["n_kgroups"], 0, 5, O.STREAM_KEY_KMEANS))
    np.testing.assert_array_equal(_np(out["trace"]["query_init"][0]),
                                  O.kmeans_init(n, pd["n_qgroups"], 0, 5, O.STREAM_QUERY_KMEANS))
    pq = _np(out["perm_q"][0])
    qo = _np(out["qoff"][0])
    np.testing.assert_array_equal(_np(out["probe_idx"][0]), O.pick_probes(pq, qo, pd["n_probes"], 0, 5))


@pytest.mark.parametrize("fit_input", [0, 1])
def test_fit_readings_stage_parity(gpu, fit_input):
    """Both readings of the affine map's input (0: the whole sparse output row, the
    default; 1: its projection on the probe-residual subspace), stage by stage."""
    import torch
    spr = _spr()
    for w, seed in ((workload("tiny"), 0), (_ragged_workload(), 3)):
        pd = params_dict(w, fit_input=fit_input)
        p = spr.Params.make(**pd)
        qb, kb, vb = generate(w, seed=seed)
        Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
        out = spr.run_call(p, Q, K, V, trace=True)
        torch.cuda.synchronize()
        assert spr.sparsepr_workspace_error(p, out["ws"]) == 0
        stage_checks(pd, qb, kb, vb, out, range(w.B * w.H), rows=None)


@pytest.mark.parametrize("fit_input", [0, 1])
def test_fit_readings_end_to_end_tiny(gpu, fit_input):
    """The oracle's own call with the same reading reconstructs the same O."""
    import torch
    spr = _spr()
    w = workload("tiny")
    pd = params_dict(w, fit_input=fit_input)
    p = spr.Params.make(**pd)
    qb, kb, vb = generate(w, seed=0)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    o, _ = _forward(p, Q, K, V, gpu)
    op = oracle_params(pd)
    for h in range(w.H):
        ref = O.sparsepr_head(to_f64(qb[0, h]), to_f64(kb[0, h]), to_f64(vb[0, h]), op, h)
        assert rel_l2(_np(o[0, h]).astype(np.float64), ref.o) <= O_REL_L2


def test_forward_captured_in_cuda_graph(gpu):
    """The single call captured into a CUDA graph (its probe path then stays on the
    captured stream) replays to the same bytes as the direct call."""
    import torch
    spr = _spr()
    w = _ragged_workload()
    pd = params_dict(w)
    p = spr.Params.make(**pd)
    qb, kb, vb = generate(w, seed=9)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    o_ref, rho_ref = _forward(p, Q, K, V, gpu)
    ws = spr.workspace(p, gpu, forward=True)
    o = torch.empty_like(Q)
    rho = torch.empty(p.BH, dtype=torch.float32, device=gpu)
    side = torch.cuda.Stream(gpu)
    side.wait_stream(torch.cuda.current_stream(gpu))
    with torch.cuda.stream(side):   # warm-up outside the capture
        spr.sparsepr_forward(p, Q, K, V, o, rho, ws)
    torch.cuda.current_stream(gpu).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        spr.sparsepr_forward(p, Q, K, V, o, rho, ws)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, ws) == 0
    assert torch.equal(o, o_ref)
    assert torch.equal(rho, rho_ref)
    del g
