"""CPU tests of the C-ABI library: it loads, exports every declared symbol, its
struct layout matches the header, and host-side validation rejects bad arguments
before touching CUDA (no compute call runs here)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparsepr.h")


@pytest.fixture(scope="module")
def spr():
    import __graft_entry__
    __graft_entry__.build()
    import free_block_sparse_rcp_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SPARSEPR_API\s+[\w\s\*]+?\b(sparsepr_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("sparsepr_partition", "sparsepr_attend", "sparsepr_probe_fit", "sparsepr_reconstruct",
                 "sparsepr_workspace_bytes", "sparsepr_dense_attention", "sparsepr_forward"):
        assert need in names


def test_library_exports_every_declared_symbol(spr):
    lib = ctypes.CDLL(spr.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(spr.EXPORTED) == set(declared_functions())


def test_struct_layout_matches_header(spr):
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "sparsepr.h"
#define F(s, m) printf(#m " %zu\n", offsetof(s, m));
int main(void) {
  printf("size %zu\n", sizeof(sparsepr_params));
  F(sparsepr_params, density) F(sparsepr_params, n_kgroups) F(sparsepr_params, kmeans_iters)
  F(sparsepr_params, ridge_lambda) F(sparsepr_params, scale) F(sparsepr_params, seed) F(sparsepr_params, frame_id)
  F(sparsepr_params, n_frames) F(sparsepr_params, partition_mode) F(sparsepr_params, fit_weighted)
  F(sparsepr_params, fit_input) F(sparsepr_params, head_offset) F(sparsepr_params, heads_total)
  printf("ptrace %zu\n", sizeof(sparsepr_partition_trace));
  printf("prtrace %zu\n", sizeof(sparsepr_probe_trace));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "t.c")
        exe = os.path.join(td, "t")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        out = dict(line.split() for line in subprocess.check_output([exe], text=True).splitlines())
    P = spr.Params
    assert int(out["size"]) == ctypes.sizeof(P)
    for f in ("density", "n_kgroups", "kmeans_iters", "ridge_lambda", "scale", "seed", "frame_id", "n_frames",
              "partition_mode", "fit_weighted", "fit_input", "head_offset", "heads_total"):
        assert int(out[f]) == getattr(P, f).offset, f
    assert int(out["ptrace"]) == ctypes.sizeof(spr.PartitionTrace)
    assert int(out["prtrace"]) == ctypes.sizeof(spr.ProbeTrace)


def _params(spr, **kw):
    base = dict(B=1, H=2, N=1024, d=64, block=64, density=0.25, n_kgroups=8, n_qgroups=8, n_samples=64,
                n_probes=64, eig_rank=16, sub_rank=16, kmeans_iters=8)
    base.update(kw)
    return spr.Params.make(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(d=96), 2), (dict(d=32), 2),
    (dict(block=32), 1),
    (dict(density=0.0), 1), (dict(density=1.5), 1), (dict(density=float("nan")), 1),
    (dict(density=0.05), 1),                  # below the probe floor 64/1024
    (dict(n_kgroups=0), 1), (dict(n_qgroups=2000), 1), (dict(n_kgroups=200), 2),
    (dict(n_samples=0), 1), (dict(n_probes=65), 1), (dict(n_probes=0), 1),
    (dict(eig_rank=65), 1), (dict(sub_rank=65), 1), (dict(sub_rank=0), 1),
    (dict(kmeans_iters=0), 1), (dict(ridge_lambda=0.0), 1), (dict(scale=-1.0), 1),
    (dict(N=0), 1), (dict(H=0), 1),
    (dict(N=37, n_kgroups=37, n_qgroups=4, n_samples=37, n_probes=37, sub_rank=16, density=1.0), 0),
    (dict(d=128, eig_rank=32, sub_rank=33), 2),
    (dict(partition_mode=1), 0), (dict(partition_mode=2), 1), (dict(partition_mode=-1), 1),
    (dict(fit_weighted=1), 0), (dict(fit_weighted=2), 1),
    (dict(fit_input=1), 0), (dict(fit_input=2), 1), (dict(fit_input=-1), 1),
    (dict(head_offset=6, heads_total=8), 0), (dict(head_offset=6), 0), (dict(head_offset=-1), 1),
    (dict(head_offset=7, heads_total=8), 1), (dict(heads_total=1), 1), (dict(heads_total=-2), 1),
])
def test_validation(spr, kw, status):
    p = _params(spr, **kw)
    assert spr.sparsepr_validate(p) == status
    assert (spr.sparsepr_workspace_bytes(p) > 0) == (status == 0)


@pytest.mark.parametrize("n_frames,N,status", [(4, 1024, 0), (64, 1024, 0), (0, 1024, 1), (65, 1024, 1),
                                               (4, 70000, 2)])
def test_validation_frames(spr, n_frames, N, status):
    """Frame-causal params: 1..64 frames, N <= 65535 (the pointer is never dereferenced)."""
    p = _params(spr, N=N)
    p.frame_id = 1 << 20
    p.n_frames = n_frames
    assert spr.sparsepr_validate(p) == status
    if status == 0:
        plain = _params(spr, N=N)
        # the causal key streams (one per query group) make the workspace larger
        assert spr.sparsepr_workspace_bytes(p) > spr.sparsepr_workspace_bytes(plain)


def test_calls_reject_before_cuda(spr):
    lib = spr._lib
    p = _params(spr)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    # NULL input
    st = lib.sparsepr_partition(ctypes.byref(p), None, fake, fake, fake, fake, fake, fake, fake, fake, None, fake,
                                None, fake, 1 << 40, None)
    assert st == 1 and b"Q" in lib.sparsepr_last_error()
    # workspace too small / misaligned
    st = lib.sparsepr_partition(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake, None, fake,
                                None, fake, 16, None)
    assert st == 3
    st = lib.sparsepr_attend(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, fake, None,
                             ctypes.c_void_p((1 << 20) + 8), 1 << 40, None)
    assert st == 3
    bad = _params(spr, d=96)
    assert lib.sparsepr_forward(ctypes.byref(bad), fake, fake, fake, fake, None, fake, 1 << 40, None) == 2
    assert lib.sparsepr_reconstruct(ctypes.byref(p), None, fake, fake, fake, fake, fake, fake, None) == 1
    # bf16 token tensors move by TMA: a pointer off a 16-byte boundary is an argument error
    odd = ctypes.c_void_p((1 << 20) + 8)
    st = lib.sparsepr_reconstruct(ctypes.byref(p), fake, fake, fake, fake, fake, fake, odd, None)
    assert st == 1 and b"O" in lib.sparsepr_last_error()
    st = lib.sparsepr_forward(ctypes.byref(p), fake, odd, fake, fake, None, fake, 1 << 40, None)
    assert st == 1 and b"K" in lib.sparsepr_last_error()
    st = lib.sparsepr_dense_attention(ctypes.byref(p), fake, fake, odd, fake, None, None, 0, None)
    assert st == 1 and b"V" in lib.sparsepr_last_error()
    assert lib.sparsepr_status_string(0) == b"ok"


def test_chunked_host_call_rejects_before_cuda(spr):
    lib = spr._lib
    p = _params(spr)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the checks fail first
    odd = ctypes.c_void_p((1 << 20) + 8)
    args = [fake] * 4
    # chunk count out of range, misaligned device staging, workspace too small
    assert lib.sparsepr_forward_host_chunked(ctypes.byref(p), *args, fake, fake, 0, fake, 1 << 40, None, None,
                                             None) == 1
    assert lib.sparsepr_forward_host_chunked(ctypes.byref(p), *args, fake, fake, 3, fake, 1 << 40, None, None,
                                             None) == 1
    assert lib.sparsepr_forward_host_chunked(ctypes.byref(p), *args, odd, fake, 2, fake, 1 << 40, None, None,
                                             None) == 1
    assert lib.sparsepr_forward_host_chunked(ctypes.byref(p), *args, fake, fake, 2, fake, 1024, None, None,
                                             None) == 3
    nul = list(args)
    nul[2] = None
    assert lib.sparsepr_forward_host_chunked(ctypes.byref(p), *nul, fake, fake, 2, fake, 1 << 40, None, None,
                                             None) == 1
    # the workspace of one chunk is enough
    one = spr.chunk_params(p, 2)
    assert one.B == 1 and one.H == 1
    assert spr.sparsepr_forward_workspace_bytes(one) < spr.sparsepr_forward_workspace_bytes(p)


def test_workspace_grows_with_problem(spr):
    a = spr.sparsepr_workspace_bytes(_params(spr))
    b = spr.sparsepr_workspace_bytes(_params(spr, H=4))
    assert b > a > 0
    assert spr.sparsepr_forward_workspace_bytes(_params(spr)) > a
