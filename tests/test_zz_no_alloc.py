"""sparsepr_probe_fit_noalloc, the allocation-free variant of the probe + fit call.

Callers that cannot allocate device memory (runtimes with a device memory plan fixed
at start-up, host code where a cudaMalloc, which can synchronize the device, is not
allowed) pass only their inputs and outputs; the variant's scratch is a fixed array
inside the library.  These tests call it through the C ABI and check its outputs
against the workspace entry point's, on two calls in a row (the shared scratch keeps
the previous call's contents), with the tolerances the parity tests use.  The file is
collected last and depends on no other test's state.
"""
import ctypes

import numpy as np
import pytest

from synth import Workload, generate, to_torch, workload

from helpers import O_REL_L2, params_dict


def _ragged():
    return Workload(name="ragged", B=2, H=2, grid=(5, 19, 20), d=128, n_centroids=24, n_seeds=40, block=128,
                    density=0.3, n_kgroups=13, n_qgroups=11, n_samples=128, n_probes=64, eig_rank=32,
                    sub_rank=32, kmeans_iters=6, centroid_scale=1.0)


def _many_heads():
    # 64 heads of 8192 tokens, d = 128: the default four key splits need about 19 MB of
    # scratch, so the variant drops to three splits to fit its 16 MiB array
    return Workload(name="heads64", B=1, H=64, grid=(8, 32, 32), d=128, n_centroids=64, n_seeds=64, block=128,
                    density=0.25, n_kgroups=32, n_qgroups=32, n_samples=128, n_probes=64, eig_rank=32,
                    sub_rank=32, kmeans_iters=5, centroid_scale=1.0)


def _partition_and_reference(spr, p, Q, K, V, gpu):
    """Partition, routed attention, the workspace entry point's probe fit and O."""
    import torch
    ws = spr.workspace(p, gpu)
    part = spr.alloc_partition(p, gpu)
    spr.sparsepr_partition(p, Q, K, part["perm_q"], part["perm_k"], part["label_q"], part["label_k"], part["qoff"],
                           part["koff"], part["route"], part["block_mask"], part["rho_exec"], ws)
    o_sparse = torch.empty_like(Q)
    lse = torch.empty(p.BH, p.N, dtype=torch.float32, device=gpu)
    spr.sparsepr_attend(p, Q, K, V, part["perm_q"], part["perm_k"], part["qoff"], part["koff"], part["route"],
                        o_sparse, lse, ws)
    ref = spr.alloc_probe(p, gpu, with_bmat=True)
    spr.sparsepr_probe_fit(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                           ref["probe_idx"], ref["probe_o_dense"], ref["b_full"], ref["Vr"], ref["W"], ref["Bmat"], ws)
    o_ref = torch.empty_like(Q)
    spr.sparsepr_reconstruct(p, o_sparse, ref["probe_idx"], ref["probe_o_dense"], ref["b_full"], ref["Vr"], ref["W"],
                             o_ref)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, ws) == 0
    return part, o_sparse, ref, o_ref


def _noalloc(spr, p, Q, K, V, part, gpu):
    import torch
    got = spr.alloc_probe(p, gpu, with_bmat=True)
    for t in got.values():
        if t is not None:
            t.fill_(-1 if t.dtype == torch.int32 else float("nan"))
    spr.sparsepr_probe_fit_noalloc(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                                   got["probe_idx"], got["probe_o_dense"], got["b_full"], got["Vr"], got["W"],
                                   got["Bmat"])
    return got


@pytest.mark.gpu
@pytest.mark.parametrize("make", [lambda: workload("tiny"), _ragged, lambda: workload("mid", H=4), _many_heads])
def test_noalloc_matches_workspace_entry_point(gpu, make):
    import torch
    import free_block_sparse_rcp_b200 as spr

    w = make()
    p = spr.Params.make(**params_dict(w))
    qb, kb, vb = generate(w, seed=5)
    Q, K, V = (to_torch(x, gpu) for x in (qb, kb, vb))
    part, o_sparse, ref, o_ref = _partition_and_reference(spr, p, Q, K, V, gpu)
    # another problem of the same shape, whose call leaves its own contents in the shared
    # scratch between the two compared calls
    qo, ko, vo = (to_torch(x, gpu) for x in generate(w, seed=6))
    part_o, _, _, _ = _partition_and_reference(spr, p, qo, ko, vo, gpu)
    for call in range(2):
        if call == 1:
            other = _noalloc(spr, p, qo, ko, vo, part_o, gpu)
            torch.cuda.synchronize()
            assert bool(torch.isfinite(other["W"]).all())
        got = _noalloc(spr, p, Q, K, V, part, gpu)
        o = torch.empty_like(Q)
        spr.sparsepr_reconstruct(p, o_sparse, got["probe_idx"], got["probe_o_dense"], got["b_full"], got["Vr"],
                                 got["W"], o)
        torch.cuda.synchronize()
        assert torch.equal(got["probe_idx"], ref["probe_idx"]), call
        od, od_ref = got["probe_o_dense"].double(), ref["probe_o_dense"].double()
        assert float((od - od_ref).norm() / od_ref.norm()) <= 1e-5, call
        # the fit's effect on the output (a fifth of the reconstruction budget), then O itself
        x = o_sparse.double().reshape(p.BH, p.N, p.d)
        corr = got["b_full"].double()[:, None, :] + x @ got["Bmat"].double()
        corr_ref = ref["b_full"].double()[:, None, :] + x @ ref["Bmat"].double()
        assert float((corr - corr_ref).norm()) <= 2e-3 * float(x.norm()), call
        rel = float((o.double() - o_ref.double()).norm() / o_ref.double().norm())
        assert rel <= O_REL_L2, (call, rel)


def test_noalloc_rejects_before_any_work():
    """Problems larger than the fixed scratch and NULL pointers are refused on the host."""
    import free_block_sparse_rcp_b200 as spr

    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the checks fail first
    big = spr.Params.make(1, 512, 8192, 128, block=128, density=0.25, n_kgroups=64, n_qgroups=64, n_samples=128,
                          n_probes=64, eig_rank=32, sub_rank=32, kmeans_iters=5)
    args = [fake] * 13
    assert spr._lib.sparsepr_probe_fit_noalloc(ctypes.byref(big), *args, None) == 2
    small = spr.Params.make(1, 2, 1024, 64, block=64, density=0.25, n_kgroups=8, n_qgroups=8, n_samples=64,
                            n_probes=64, eig_rank=16, sub_rank=16, kmeans_iters=8)
    nulls = list(args)
    nulls[0] = None
    assert spr._lib.sparsepr_probe_fit_noalloc(ctypes.byref(small), *nulls, None) == 1
    # a Q, K or V off a 16-byte boundary is refused on the host (never dereferenced)
    for i in range(3):
        odd = list(args)
        odd[i] = ctypes.c_void_p((1 << 20) + 8)
        assert spr._lib.sparsepr_probe_fit_noalloc(ctypes.byref(small), *odd, None) == 1
    # frame-causal params need the workspace entry point
    causal = spr.Params.make(1, 2, 1024, 64, block=64, density=0.25, n_kgroups=8, n_qgroups=8, n_samples=64,
                             n_probes=64, eig_rank=16, sub_rank=16, kmeans_iters=8)
    causal.frame_id = 1 << 20
    causal.n_frames = 4
    assert spr._lib.sparsepr_probe_fit_noalloc(ctypes.byref(causal), *args, None) == 2
