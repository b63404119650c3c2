"""Benchmark of the SparsePR per-call sparse-attention path on B200.

One step = one whole attention call (partition -> attend -> probe_fit ->
reconstruct) over the 32,760-token, 40-head, d=128 video-shaped workload at 25%
executed-pair density, inputs resident in HBM.  Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--gpus N > 1 runs under torchrun, one rank per GPU, each rank an independent call
on its own inputs (the heads shard with no data-path collective: weak scaling).
--impl reference times the CPU oracle (the method restated in fp64 numpy) on the
host cores, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "wan"
METRIC = "ms/attention call & executed TFLOP/s (frac of BF16 peak) at 25% density; rel-L2"
UNIT = "ms/call"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return dict(hbm=pk["hbm_gbs"], bf16=pk["bf16_tflops"], bf16_sus=pk.get("bf16_tflops_sustained",
                    pk["bf16_tflops"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _config(w, extra=None):
    c = {"workload": f"{w.name}-shaped video tokens {w.grid[0]}x{w.grid[1]}x{w.grid[2]}",
         "global_batch": w.B, "seq_len": w.N, "heads": w.H, "head_dim": w.d, "density": w.density,
         "k_groups": w.n_kgroups, "q_groups": w.n_qgroups, "probes_per_head": w.n_probes,
         "subspace_rank": w.sub_rank, "kmeans_iters": w.kmeans_iters,
         "parallelism": "independent calls per rank (heads shard, no collective)",
         "l2": "inputs larger than L2 (Q,K,V = 1.0 GB per call), no flush"}
    if extra:
        c.update(extra)
    return c


class ClockSampler:
    """nvidia-smi samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = str(gpu_index)
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # the timed region starts once the sampler is producing lines
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0:
                time.sleep(0.01)
            self.lines.clear()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device=None) -> float:
    """Max of a per-rank scalar (device time) over the process group."""
    if ws <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_call(total_ms_max: float, steps: int, ws: int) -> float:
    """Whole-job figure: every rank runs `steps` independent calls on its own heads, so
    the job completes steps * ws calls in the slowest rank's time."""
    return total_ms_max / (steps * ws)


# ---------------------------------------------------------------------------
def run_cuda(args):
    import datetime
    import numpy as np
    import torch

    ws, rank, local = _dist()
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import __graft_entry__
    __graft_entry__.build()
    import free_block_sparse_rcp_b200 as spr
    from synth import generate, workload

    w = workload(WORKLOAD, H=args.heads) if args.heads else workload(WORKLOAD)
    pd = dict(B=w.B, H=w.H, N=w.N, d=w.d, block=w.block, density=w.density, n_kgroups=w.n_kgroups,
              n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes, eig_rank=w.eig_rank,
              sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, ridge_lambda=w.ridge_lambda, seed=0)
    p = spr.Params.make(**pd)
    qb, kb, vb = generate(w, seed=rank)
    from synth import to_torch
    Q, K, V = (to_torch(x, dev) for x in (qb, kb, vb))
    BH, N, d = p.BH, p.N, p.d
    wsb = spr.workspace(p, dev)
    part = spr.alloc_partition(p, dev)
    pr = spr.alloc_probe(p, dev)
    o_sparse = torch.empty_like(Q)
    lse = torch.empty(BH, N, dtype=torch.float32, device=dev)
    o = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)

    launches = [0]

    def step(ev=None):
        n = 0
        if ev is not None:
            ev[0].record(stream)
        spr.sparsepr_partition(p, Q, K, part["perm_q"], part["perm_k"], part["label_q"], part["label_k"],
                               part["qoff"], part["koff"], part["route"], part["block_mask"], part["rho_exec"], wsb)
        n += spr.last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        spr.sparsepr_attend(p, Q, K, V, part["perm_q"], part["perm_k"], part["qoff"], part["koff"], part["route"],
                            o_sparse, lse, wsb)
        n += spr.last_launch_count()
        if ev is not None:
            ev[2].record(stream)
        spr.sparsepr_probe_fit(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                               pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], None, wsb)
        n += spr.last_launch_count()
        if ev is not None:
            ev[3].record(stream)
        spr.sparsepr_reconstruct(p, o_sparse, pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"],
                                 o)
        n += spr.last_launch_count()
        if ev is not None:
            ev[4].record(stream)
        launches[0] += n

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, wsb) == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    launches[0] = 0
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    stage = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(args.steps)]
    total_ms = sum(evs[i][0].elapsed_time(evs[i][4]) for i in range(args.steps))
    total_ms = max_over_ranks(total_ms, ws, dev)
    ms_per_step = total_ms / args.steps
    value = job_ms_per_call(total_ms, args.steps, ws)
    stage_ms = [statistics.mean(s[j] for s in stage) for j in range(4)]

    # --- algorithmic work of the attention kernel (useful routed pairs)
    nq = torch.diff(part["qoff"].long(), dim=1)
    nk = torch.diff(part["koff"].long(), dim=1)
    routed_pairs = int((nq[:, :, None] * nk[:, None, :] * part["route"].long()).sum().item())
    # MMA-issued pairs: q-tiles of 128 rows x routed key rows padded to 128-key chunks
    ntile = (nq + 127) // 128
    rk = (nk[:, None, :] * part["route"].long()).sum(-1)
    issued_pairs = int((ntile * 128 * ((rk + 127) // 128) * 128).sum().item())
    attn_flops = 4.0 * d * routed_pairs
    attn_ms = stage_ms[1]
    pk = _peaks()
    achieved = attn_flops / (attn_ms * 1e-3) / 1e12
    dense_flops = 4.0 * d * N * N * BH

    # --- dense comparator on the same machinery
    o_dense = torch.empty_like(Q)
    for _ in range(2):
        spr.sparsepr_dense_attention(p, Q, K, V, o_dense, None, wsb)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nd = 3
    e0.record(stream)
    for _ in range(nd):
        spr.sparsepr_dense_attention(p, Q, K, V, o_dense, None, wsb)
    e1.record(stream)
    torch.cuda.synchronize()
    dense_ms = e0.elapsed_time(e1) / nd

    # --- errors against this build's dense output (hard drop, reconstruction)
    def rel(a, b):
        return float((a.float() - b.float()).norm() / b.float().norm())

    err_sparse = rel(o_sparse, o_dense)
    err_recon = rel(o, o_dense)

    # --- end to end through the C ABI from pinned host buffers
    Qh, Kh, Vh = (torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(3))
    Qh.copy_(Q.cpu()); Kh.copy_(K.cpu()); Vh.copy_(V.cpu())
    Oh = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    qkv_dev = torch.empty((3,) + tuple(Q.shape), dtype=torch.bfloat16, device=dev)
    o_dev = torch.empty_like(Q)
    fws = spr.workspace(p, dev, forward=True)
    e2e_steps = max(2, min(args.steps, 5))
    for _ in range(2):
        spr.sparsepr_forward_host(p, Qh, Kh, Vh, Oh, qkv_dev, o_dev, fws)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        spr.sparsepr_forward_host(p, Qh, Kh, Vh, Oh, qkv_dev, o_dev, fws)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_total = max_over_ranks(a0.elapsed_time(a1), ws, dev)
    e2e_value = e2e_total / (e2e_steps * ws)
    bytes_in = 3 * BH * N * d * 2

    traffic = _traffic_record("attend")
    rho = part["rho_exec"].float()
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w),
        "stage_ms": {"partition": round(stage_ms[0], 4), "attend": round(stage_ms[1], 4),
                     "probe_fit": round(stage_ms[2], 4), "reconstruct": round(stage_ms[3], 4)},
        "dense_attention_ms": round(dense_ms, 4),
        "speedup_vs_dense": round(dense_ms / ms_per_step, 3),
        "rho_exec": {"mean": round(float(rho.mean()), 5), "min": round(float(rho.min()), 5),
                     "max": round(float(rho.max()), 5)},
        "attend_tflops_useful": round(achieved, 2),
        "attend_tflops_issued": round(4.0 * d * issued_pairs / (attn_ms * 1e-3) / 1e12, 2),
        "tile_fill": round(routed_pairs / max(1, issued_pairs), 4),
        "dense_equiv_tflops": round(dense_flops / (ms_per_step * 1e-3) / 1e12, 2),
        "dense_kernel_tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 2),
        "rel_l2_vs_dense": {"o_sparse": round(err_sparse, 5), "o_reconstructed": round(err_recon, 5)},
        "roofline": {"kernel": "attend (routed flash attention)", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": pk["bf16_sus"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_sus"], 4),
                     "peak_kind": f"bf16 sustained, {pk['src']}",
                     "frac_of_burst": round(achieved / pk["bf16"], 4),
                     "traffic": traffic, "algorithmic_flops_per_launch": attn_flops},
        "e2e": {"value": round(e2e_value, 4), "unit": UNIT, "h2d_bytes_per_step": bytes_in,
                "d2h_bytes_per_step": BH * N * d * 2},
        "gpu_launches": launches[0],
        "clocks": clk.summary(),
    }
    if rank == 0 and ws == 1 and not args.heads:
        line["cpu_baseline"] = cpu_baseline(args.cpu_budget)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _traffic_record(kernel: str):
    """DRAM traffic per launch from the committed ncu summary, if it was taken on the
    current kernel source (else null)."""
    try:
        import hashlib
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, "free_block_sparse_rcp_b200", "csrc", rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return rec["bytes_per_launch"] if h == rec["source_sha"] else None
    except Exception:
        return None


# ---------------------------------------------------------------------------
def oracle_sample(w, rows_frac=1 / 32, seed=0):
    """One head of the workload through the oracle: full partition, probes and fit,
    routed attention on a row sample; returns (seconds extrapolated to one call,
    seconds actually spent)."""
    import numpy as np
    import oracle as O
    from synth import generate, to_f64
    qb, kb, vb = generate(w, seed=seed, heads=[(0, 0)])
    q, k, v = to_f64(qb[0, 0]), to_f64(kb[0, 0]), to_f64(vb[0, 0])
    p = O.Params(n_kgroups=w.n_kgroups, n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes,
                 eig_rank=w.eig_rank, sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, density=w.density,
                 ridge_lambda=w.ridge_lambda, seed=0, block=w.block)
    s = p.eff_scale(w.d)
    t0 = time.perf_counter()
    part = O.partition_head(q, k, p, 0)
    t1 = time.perf_counter()
    n_rows = max(1, int(w.N * rows_frac))
    rows = np.arange(0, w.N, w.N // n_rows)[:n_rows]
    o_s, _ = O.sparse_attention(q, k, v, s, part.route.route, part.label_q, part.label_k, rows=rows)
    t2 = time.perf_counter()
    fit = O.probe_fit_head(q, k, v, part.label_q, part.label_k, part.route.route, part.perm_q, part.q_offsets, p, 0)
    t3 = time.perf_counter()
    _ = o_s + fit.b_full + (o_s @ fit.w) @ fit.vr.T
    t4 = time.perf_counter()
    per_head = (t1 - t0) + (t2 - t1) * (w.N / len(rows)) + (t3 - t2) + (t4 - t3) * (w.N / len(rows))
    return per_head * w.B * w.H, t4 - t0, len(rows)


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count()


def cpu_baseline(budget_s=30.0):
    from synth import workload
    w = workload(WORKLOAD)
    sec, spent, nrows = oracle_sample(w)
    return {"value": round(sec * 1e3, 1), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"head (0,0) of {w.B * w.H}: full partition, probes and fit; routed attention and "
                      f"correction on {nrows} of {w.N} rows; extrapolated x{w.B * w.H} heads "
                      f"(took {spent:.1f} s)"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    from synth import workload
    w = workload(WORKLOAD)
    for _ in range(args.warmup):
        oracle_sample(workload("tiny"), rows_frac=1.0)   # warms numpy / BLAS; not timed
    vals, spent = [], 0.0
    for _ in range(args.steps):
        v, s, nrows = oracle_sample(w)
        vals.append(v)
        spent += s
    value = statistics.mean(vals) * 1e3
    cores = _cores()
    sample = (f"head (0,0) of {w.B * w.H} per step: full partition, probes and fit; routed attention and "
              f"correction on {nrows} of {w.N} rows; extrapolated to the whole call")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value, 1),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w),
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=30.0)
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (small cases for ncu captures; default: the workload's 40)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
