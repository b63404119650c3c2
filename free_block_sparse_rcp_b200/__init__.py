"""SparsePR per-call sparse attention on B200 (sm_100a): Python binding.

A thin ctypes layer over ``libsparsepr.so`` (the C ABI declared in
``include/sparsepr.h``).  Every function here only marshals torch tensors into
device pointers and the current CUDA stream and raises ``SparsePRError`` on a
non-zero status; all arithmetic runs in the library's CUDA kernels.  There is no
fallback: importing this package without the built library raises ImportError.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparsepr.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python free_block_sparse_rcp_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_ip = ctypes.POINTER(ctypes.c_int)


class Params(ctypes.Structure):
    """Mirror of ``sparsepr_params``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("block", ctypes.c_int), ("density", ctypes.c_float), ("n_kgroups", ctypes.c_int),
                ("n_qgroups", ctypes.c_int), ("n_samples", ctypes.c_int), ("n_probes", ctypes.c_int),
                ("eig_rank", ctypes.c_int), ("sub_rank", ctypes.c_int), ("kmeans_iters", ctypes.c_int),
                ("ridge_lambda", ctypes.c_float), ("scale", ctypes.c_float), ("seed", ctypes.c_ulonglong),
                ("frame_id", _vp), ("n_frames", ctypes.c_int), ("partition_mode", ctypes.c_int),
                ("fit_weighted", ctypes.c_int), ("fit_input", ctypes.c_int), ("head_offset", ctypes.c_int),
                ("heads_total", ctypes.c_int)]

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def tiles(self) -> int:
        return (self.N + self.block - 1) // self.block

    def eff_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_ if k not in ("frame_id", "n_frames")}

    @classmethod
    def make(cls, B, H, N, d, *, block, density, n_kgroups, n_qgroups, n_samples, n_probes, eig_rank,
             sub_rank, kmeans_iters, ridge_lambda=1e-2, scale=0.0, seed=0, frame_id=None, n_frames=0,
             partition_mode=0, fit_weighted=0, fit_input=0, head_offset=0, heads_total=0):
        """frame_id: optional int32 device tensor [N] (frame-causal masking, kept alive by the
        caller for as long as the params are used).  fit_input: 0 = the affine map takes the
        whole sparse output row, 1 = its projection on the residual subspace.  head_offset /
        heads_total: this call's heads within the layer (random streams only)."""
        fid = None if frame_id is None else frame_id.data_ptr()
        return cls(B=B, H=H, N=N, d=d, block=block, density=density, n_kgroups=n_kgroups,
                   n_qgroups=n_qgroups, n_samples=n_samples, n_probes=n_probes, eig_rank=eig_rank,
                   sub_rank=sub_rank, kmeans_iters=kmeans_iters, ridge_lambda=ridge_lambda, scale=scale,
                   seed=seed, frame_id=fid, n_frames=n_frames, partition_mode=partition_mode,
                   fit_weighted=fit_weighted, fit_input=fit_input, head_offset=head_offset,
                   heads_total=heads_total)


class PartitionTrace(ctypes.Structure):
    """Mirror of ``sparsepr_partition_trace`` (NULL fields are skipped)."""
    _fields_ = [(n, _vp) for n in ("sample_idx", "metric", "eigval", "eigvec", "key_coords", "key_init",
                                   "key_label_iters", "key_centroids", "query_coords", "query_init",
                                   "query_label_iters", "cell_mass", "alpha")]


class ProbeTrace(ctypes.Structure):
    """Mirror of ``sparsepr_probe_trace``."""
    _fields_ = [(n, _vp) for n in ("probe_o_sparse", "probe_lse_dense", "probe_lse_sparse", "sigma", "b_sub")]


_P = ctypes.POINTER(Params)
_sig = {
    "sparsepr_workspace_bytes": (ctypes.c_size_t, [_P]),
    "sparsepr_forward_workspace_bytes": (ctypes.c_size_t, [_P]),
    "sparsepr_validate": (ctypes.c_int, [_P]),
    "sparsepr_partition": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          ctypes.POINTER(PartitionTrace), _vp, ctypes.c_size_t, _vp]),
    "sparsepr_attend": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       ctypes.c_size_t, _vp]),
    "sparsepr_probe_fit": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, ctypes.POINTER(ProbeTrace), _vp, ctypes.c_size_t, _vp]),
    "sparsepr_probe_fit_noalloc": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                  _vp, _vp, _vp]),
    "sparsepr_reconstruct": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "sparsepr_forward": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "sparsepr_forward_host": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "sparsepr_forward_host_chunked": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _vp,
                                                     ctypes.c_size_t, _vp, _vp, _vp]),
    "sparsepr_dense_attention": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "sparsepr_workspace_error": (ctypes.c_int, [_P, _vp, _vp]),
    "sparsepr_workspace_clear_error": (ctypes.c_int, [_P, _vp, _vp]),
    "sparsepr_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sparsepr_last_error": (ctypes.c_char_p, []),
    "sparsepr_last_launch_count": (ctypes.c_int, []),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sig)


class SparsePRError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.sparsepr_status_string(status).decode()
        detail = _lib.sparsepr_last_error().decode()
        super().__init__(f"{where}: {msg} ({detail})")


def _check(status: int, where: str):
    if status != 0:
        raise SparsePRError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _trace(cls, d):
    if d is None:
        return None
    tr = cls()
    for k, v in d.items():
        setattr(tr, k, v.data_ptr() if v is not None else None)
    return ctypes.byref(tr)


def last_launch_count() -> int:
    return _lib.sparsepr_last_launch_count()


def sparsepr_validate(p: Params) -> int:
    return _lib.sparsepr_validate(ctypes.byref(p))


def sparsepr_workspace_bytes(p: Params) -> int:
    return _lib.sparsepr_workspace_bytes(ctypes.byref(p))


def sparsepr_forward_workspace_bytes(p: Params) -> int:
    return _lib.sparsepr_forward_workspace_bytes(ctypes.byref(p))


def workspace(p: Params, device, forward: bool = False):
    """A caller-owned workspace tensor of the size the library asks for."""
    import torch
    n = sparsepr_forward_workspace_bytes(p) if forward else sparsepr_workspace_bytes(p)
    if n == 0:
        _check(sparsepr_validate(p), "workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def sparsepr_partition(p, Q, K, perm_q, perm_k, label_q, label_k, qoff, koff, route, block_mask, rho_exec,
                       ws, trace=None):
    _check(_lib.sparsepr_partition(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(perm_q), _ptr(perm_k),
                                   _ptr(label_q), _ptr(label_k), _ptr(qoff), _ptr(koff), _ptr(route),
                                   _ptr(block_mask), _ptr(rho_exec), _trace(PartitionTrace, trace),
                                   _ptr(ws), ws.numel(), _stream(Q)), "sparsepr_partition")


def sparsepr_attend(p, Q, K, V, perm_q, perm_k, qoff, koff, route, O_sparse, lse, ws):
    _check(_lib.sparsepr_attend(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm_q), _ptr(perm_k),
                                _ptr(qoff), _ptr(koff), _ptr(route), _ptr(O_sparse), _ptr(lse), _ptr(ws),
                                ws.numel(), _stream(Q)), "sparsepr_attend")


def sparsepr_probe_fit(p, Q, K, V, label_k, perm_q, qoff, route, probe_idx, probe_o_dense, b_full, Vr, W,
                       Bmat, ws, trace=None):
    _check(_lib.sparsepr_probe_fit(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(label_k), _ptr(perm_q),
                                   _ptr(qoff), _ptr(route), _ptr(probe_idx), _ptr(probe_o_dense),
                                   _ptr(b_full), _ptr(Vr), _ptr(W), _ptr(Bmat), _trace(ProbeTrace, trace),
                                   _ptr(ws), ws.numel(), _stream(Q)), "sparsepr_probe_fit")


def sparsepr_probe_fit_noalloc(p, Q, K, V, label_k, perm_q, qoff, route, probe_idx, probe_o_dense, b_full,
                               Vr, W, Bmat):
    _check(_lib.sparsepr_probe_fit_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(label_k),
                                           _ptr(perm_q), _ptr(qoff), _ptr(route), _ptr(probe_idx),
                                           _ptr(probe_o_dense), _ptr(b_full), _ptr(Vr), _ptr(W), _ptr(Bmat),
                                           _stream(Q)), "sparsepr_probe_fit_noalloc")


def sparsepr_reconstruct(p, O_sparse, probe_idx, probe_o_dense, b_full, Vr, W, O):
    _check(_lib.sparsepr_reconstruct(ctypes.byref(p), _ptr(O_sparse), _ptr(probe_idx), _ptr(probe_o_dense),
                                     _ptr(b_full), _ptr(Vr), _ptr(W), _ptr(O), _stream(O)),
           "sparsepr_reconstruct")


def sparsepr_forward(p, Q, K, V, O, rho_exec, ws):
    _check(_lib.sparsepr_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(rho_exec),
                                 _ptr(ws), ws.numel(), _stream(Q)), "sparsepr_forward")


def sparsepr_forward_host(p, Q_host, K_host, V_host, O_host, qkv_dev, o_dev, ws):
    _check(_lib.sparsepr_forward_host(ctypes.byref(p), _ptr(Q_host), _ptr(K_host), _ptr(V_host),
                                      _ptr(O_host), _ptr(qkv_dev), _ptr(o_dev), _ptr(ws), ws.numel(),
                                      _stream(qkv_dev)), "sparsepr_forward_host")


def sparsepr_forward_host_chunked(p, Q_host, K_host, V_host, O_host, qkv_dev, o_dev, n_chunks, ws,
                                  copy_in_stream=None, copy_out_stream=None):
    """The chunked host pipeline on the current stream of qkv_dev's device; the copy streams
    are torch.cuda.Stream objects (None: the current stream)."""
    def sp(s):
        return None if s is None else ctypes.c_void_p(s.cuda_stream)
    _check(_lib.sparsepr_forward_host_chunked(ctypes.byref(p), _ptr(Q_host), _ptr(K_host), _ptr(V_host),
                                              _ptr(O_host), _ptr(qkv_dev), _ptr(o_dev), int(n_chunks), _ptr(ws),
                                              ws.numel(), _stream(qkv_dev), sp(copy_in_stream),
                                              sp(copy_out_stream)), "sparsepr_forward_host_chunked")


def chunk_params(p: Params, n_chunks: int) -> Params:
    """Params of the largest chunk of sparsepr_forward_host_chunked (for its workspace size)."""
    q = Params.from_buffer_copy(p)
    q.B, q.H = 1, -(-p.BH // n_chunks)
    q.head_offset, q.heads_total = 0, 0
    return q


def sparsepr_dense_attention(p, Q, K, V, O, lse, ws=None):
    _check(_lib.sparsepr_dense_attention(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                         _ptr(ws), 0 if ws is None else ws.numel(), _stream(Q)),
           "sparsepr_dense_attention")


def sparsepr_workspace_error(p, ws) -> int:
    return _lib.sparsepr_workspace_error(ctypes.byref(p), _ptr(ws), _stream(ws))


def sparsepr_workspace_clear_error(p, ws):
    _check(_lib.sparsepr_workspace_clear_error(ctypes.byref(p), _ptr(ws), _stream(ws)),
           "sparsepr_workspace_clear_error")


# ---------------------------------------------------------------------------
# Output allocation helpers (torch.empty only; no arithmetic)
# ---------------------------------------------------------------------------
def alloc_partition(p: Params, device):
    import torch
    BH, N = p.BH, p.N
    i32 = dict(dtype=torch.int32, device=device)
    return dict(perm_q=torch.empty(BH, N, **i32), perm_k=torch.empty(BH, N, **i32),
                label_q=torch.empty(BH, N, **i32), label_k=torch.empty(BH, N, **i32),
                qoff=torch.empty(BH, p.n_qgroups + 1, **i32), koff=torch.empty(BH, p.n_kgroups + 1, **i32),
                route=torch.empty(BH, p.n_qgroups, p.n_kgroups, dtype=torch.uint8, device=device),
                block_mask=torch.empty(BH, p.tiles, p.tiles, dtype=torch.uint8, device=device),
                rho_exec=torch.empty(BH, dtype=torch.float32, device=device))


def alloc_partition_trace(p: Params, device):
    import torch
    BH, N, d, T = p.BH, p.N, p.d, p.kmeans_iters
    f32 = dict(dtype=torch.float32, device=device)
    i32 = dict(dtype=torch.int32, device=device)
    return dict(sample_idx=torch.empty(BH, p.n_samples, **i32), metric=torch.empty(BH, d, d, **f32),
                eigval=torch.empty(BH, p.eig_rank, **f32), eigvec=torch.empty(BH, d, p.eig_rank, **f32),
                key_coords=torch.empty(BH, N, p.eig_rank, **f32), key_init=torch.empty(BH, p.n_kgroups, **i32),
                key_label_iters=torch.empty(T, BH, N, **i32), key_centroids=torch.empty(BH, p.n_kgroups, d, **f32),
                query_coords=torch.empty(BH, N, p.n_kgroups, **f32), query_init=torch.empty(BH, p.n_qgroups, **i32),
                query_label_iters=torch.empty(T, BH, N, **i32),
                cell_mass=torch.empty(BH, p.n_qgroups, p.n_kgroups, **f32),
                alpha=torch.empty(BH, dtype=torch.float64, device=device))


def alloc_probe(p: Params, device, with_bmat: bool = False):
    import torch
    BH, d, P, r = p.BH, p.d, p.n_probes, p.sub_rank
    f32 = dict(dtype=torch.float32, device=device)
    return dict(probe_idx=torch.empty(BH, P, dtype=torch.int32, device=device),
                probe_o_dense=torch.empty(BH, P, d, **f32), b_full=torch.empty(BH, d, **f32),
                Vr=torch.empty(BH, d, r, **f32), W=torch.empty(BH, d, r, **f32),
                Bmat=torch.empty(BH, d, d, **f32) if with_bmat else None)


def alloc_probe_trace(p: Params, device):
    import torch
    BH, d, P, r = p.BH, p.d, p.n_probes, p.sub_rank
    f32 = dict(dtype=torch.float32, device=device)
    return dict(probe_o_sparse=torch.empty(BH, P, d, **f32), probe_lse_dense=torch.empty(BH, P, **f32),
                probe_lse_sparse=torch.empty(BH, P, **f32), sigma=torch.empty(BH, r, **f32),
                b_sub=torch.empty(BH, r, **f32))


def run_call(p: Params, Q, K, V, ws=None, trace=False):
    """The four calls in order on the current stream; returns every output."""
    import torch
    dev = Q.device
    ws = workspace(p, dev) if ws is None else ws
    part = alloc_partition(p, dev)
    ptr = alloc_partition_trace(p, dev) if trace else None
    sparsepr_partition(p, Q, K, part["perm_q"], part["perm_k"], part["label_q"], part["label_k"], part["qoff"],
                       part["koff"], part["route"], part["block_mask"], part["rho_exec"], ws, ptr)
    o_sparse = torch.empty_like(Q)
    lse = torch.empty(p.BH, p.N, dtype=torch.float32, device=dev)
    sparsepr_attend(p, Q, K, V, part["perm_q"], part["perm_k"], part["qoff"], part["koff"], part["route"],
                    o_sparse, lse, ws)
    pr = alloc_probe(p, dev, with_bmat=trace)
    prt = alloc_probe_trace(p, dev) if trace else None
    sparsepr_probe_fit(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                       pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], pr["Bmat"], ws, prt)
    o = torch.empty_like(Q)
    sparsepr_reconstruct(p, o_sparse, pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], o)
    out = dict(part, o_sparse=o_sparse, lse=lse, o=o, ws=ws, **pr)
    if trace:
        out["trace"] = ptr
        out["probe_trace"] = prt
    return out
