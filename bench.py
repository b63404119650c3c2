"""Benchmark of the SparsePR per-call sparse-attention path on B200.

One step = one whole attention call (partition -> attend -> probe_fit ->
reconstruct) over the 32,760-token, 40-head, d=128 video-shaped workload at 25%
executed-pair density, inputs resident in HBM.  Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload wan|world]

--workload world times the world-model rollout instead: B=4, H=16, 16 frames of
32x32 tokens, d=128, a frame-causal mask intersected with the route, and one step
= 8 consecutive calls on inputs perturbed by N(0, 0.05^2) per call (a random walk),
each call re-partitioned and re-fitted; the value is ms per call.

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
ROLLOUT_CALLS = 8        # calls per step of the world-model rollout
ROLLOUT_SIGMA = 0.05     # per-call perturbation of Q, K, V
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
    name = (f"world-model rollout, {w.grid[0]}x{w.grid[1]}x{w.grid[2]} video tokens, frame-causal, "
            f"{ROLLOUT_CALLS} perturbed calls per step" if w.frame_causal else
            f"{w.name}-shaped video tokens {w.grid[0]}x{w.grid[1]}x{w.grid[2]}")
    c = {"workload": name,
         "global_batch": w.B, "seq_len": w.N, "heads": w.H, "head_dim": w.d, "density": w.density,
         "k_groups": w.n_kgroups, "q_groups": w.n_qgroups, "probes_per_head": w.n_probes,
         "subspace_rank": w.sub_rank, "kmeans_iters": w.kmeans_iters,
         "parallelism": "independent calls per rank (heads shard, no collective)",
         "l2": f"inputs larger than L2 (Q,K,V = {3 * w.B * w.H * w.N * w.d * 2 / 1e9:.2f} GB per call), no flush"}
    if w.frame_causal:
        c.update({"frames": w.grid[0], "mask": "frame-causal (key frame <= query frame) intersected with the route",
                  "rollout_calls_per_step": ROLLOUT_CALLS,
                  "perturbation": f"N(0, {ROLLOUT_SIGMA}^2) added to Q, K, V before each call (random walk)"})
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

    w = bench_workload(args)
    pd = dict(B=w.B, H=w.H, N=w.N, d=w.d, block=w.block, density=w.density, n_kgroups=w.n_kgroups,
              n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes, eig_rank=w.eig_rank,
              sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, ridge_lambda=w.ridge_lambda, seed=0,
              partition_mode=1 if args.partition == "semantic" else 0, fit_weighted=1 if args.weighted_fit else 0)
    from synth import frame_index, perturb, to_torch
    frames = frame_index(w.grid) if w.frame_causal else None
    fid = torch.from_numpy(frames).to(dev) if w.frame_causal else None
    p = spr.Params.make(**pd, frame_id=fid, n_frames=w.grid[0] if w.frame_causal else 0)
    qb, kb, vb = generate(w, seed=rank)
    # one input triple per call of a step (the rollout perturbs Q, K, V before every call)
    calls = ROLLOUT_CALLS if w.frame_causal else 1
    inputs = []
    for c in range(calls):
        if c > 0:
            qb, kb, vb = (perturb(x, ROLLOUT_SIGMA, 1000 * rank + j, c) for j, x in enumerate((qb, kb, vb)))
        inputs.append(tuple(to_torch(x, dev) for x in (qb, kb, vb)))
    del qb, kb, vb
    Q, K, V = inputs[-1]
    BH, N, d = p.BH, p.N, p.d
    wsb = spr.workspace(p, dev)
    part = spr.alloc_partition(p, dev)
    pr = spr.alloc_probe(p, dev)
    o_sparse = torch.empty_like(Q)
    lse = torch.empty(BH, N, dtype=torch.float32, device=dev)
    o = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)
    # attend and probe_fit depend only on the partition and use disjoint workspace regions:
    # probe_fit runs on a second, higher-priority stream beside the routed attention
    side = torch.cuda.Stream(dev, priority=-1) if args.streams == 2 else None
    fork = [torch.cuda.Event() for _ in range(2)]

    launches = [0]

    def step(evs_step=None):
        for c, (Qc, Kc, Vc) in enumerate(inputs):
            call(Qc, Kc, Vc, None if evs_step is None else evs_step[c])

    def call(Q, K, V, ev=None):
        n = 0
        if ev is not None:
            ev[0].record(stream)
        spr.sparsepr_partition(p, Q, K, part["perm_q"], part["perm_k"], part["label_q"], part["label_k"],
                               part["qoff"], part["koff"], part["route"], part["block_mask"], part["rho_exec"], wsb)
        n += spr.last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        if side is not None:
            fork[0].record(stream)
            side.wait_event(fork[0])
            with torch.cuda.stream(side):
                spr.sparsepr_probe_fit(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                                       pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], None,
                                       wsb)
                n += spr.last_launch_count()
                fork[1].record(side)
        spr.sparsepr_attend(p, Q, K, V, part["perm_q"], part["perm_k"], part["qoff"], part["koff"], part["route"],
                            o_sparse, lse, wsb)
        n += spr.last_launch_count()
        if ev is not None:
            ev[2].record(stream)
        if side is None:
            spr.sparsepr_probe_fit(p, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                                   pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], None, wsb)
            n += spr.last_launch_count()
        else:
            stream.wait_event(fork[1])
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

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(calls)]
           for _ in range(args.steps)]
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
    stage = [[evs[i][c][j].elapsed_time(evs[i][c][j + 1]) for j in range(4)]
             for i in range(args.steps) for c in range(calls)]
    total_ms = sum(evs[i][0][0].elapsed_time(evs[i][calls - 1][4]) for i in range(args.steps))
    total_ms = max_over_ranks(total_ms, ws, dev)
    ms_per_step = total_ms / args.steps
    value = job_ms_per_call(total_ms, args.steps * calls, ws)
    ms_per_call = ms_per_step / calls
    stage_ms = [statistics.mean(s[j] for s in stage) for j in range(4)]

    # --- algorithmic work of the attention kernel of the last call (useful routed pairs)
    routed_pairs, issued_pairs = attention_pairs(part, frames)
    attn_flops = 4.0 * d * routed_pairs
    # the attend stage timed alone (inside the call it shares the GPU with probe_fit)
    Ql, Kl, Vl = inputs[-1]
    ta = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    n_iso = 5
    ta[0].record(stream)
    for _ in range(n_iso):
        spr.sparsepr_attend(p, Ql, Kl, Vl, part["perm_q"], part["perm_k"], part["qoff"], part["koff"],
                            part["route"], o_sparse, lse, wsb)
    ta[1].record(stream)
    torch.cuda.synchronize()
    attn_ms = ta[0].elapsed_time(ta[1]) / n_iso
    pk = _peaks()
    achieved = attn_flops / (attn_ms * 1e-3) / 1e12
    issued_tflops = 4.0 * d * issued_pairs / (attn_ms * 1e-3) / 1e12
    # dense comparator work: every (frame-causal: every visible) pair
    if frames is None:
        dense_pairs = N * N
    else:
        per_frame = np.bincount(frames, minlength=w.grid[0]).astype(np.int64)
        dense_pairs = int((per_frame * np.cumsum(per_frame)).sum())
    dense_flops = 4.0 * d * dense_pairs * BH

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
    # the other reading of the affine map's input, on the same partition and sparse output
    p_alt = spr.Params.make(**dict(pd, fit_input=1 - pd.get("fit_input", 0)), frame_id=fid,
                            n_frames=w.grid[0] if w.frame_causal else 0)
    pr_alt = spr.alloc_probe(p_alt, dev)
    spr.sparsepr_probe_fit(p_alt, Ql, Kl, Vl, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                           pr_alt["probe_idx"], pr_alt["probe_o_dense"], pr_alt["b_full"], pr_alt["Vr"], pr_alt["W"],
                           None, wsb)
    o_alt = torch.empty_like(Q)
    spr.sparsepr_reconstruct(p_alt, o_sparse, pr_alt["probe_idx"], pr_alt["probe_o_dense"], pr_alt["b_full"],
                             pr_alt["Vr"], pr_alt["W"], o_alt)
    torch.cuda.synchronize()
    err_alt = rel(o_alt, o_dense)
    del o_alt, pr_alt
    readings = {0: "whole sparse output", 1: "sparse output projected on the subspace"}
    fit_errors = {readings[pd.get("fit_input", 0)] + " (this run's)": round(err_recon, 5),
                  readings[1 - pd.get("fit_input", 0)]: round(err_alt, 5)}

    # --- the library's single device-buffer entry point (its probe path on a stream of its own)
    fws0 = spr.workspace(p, dev, forward=True)
    o_fwd = torch.empty_like(Q)
    for _ in range(2):
        spr.sparsepr_forward(p, Ql, Kl, Vl, o_fwd, None, fws0)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nf = max(3, min(args.steps, 10))
    f0.record(stream)
    for _ in range(nf):
        spr.sparsepr_forward(p, Ql, Kl, Vl, o_fwd, None, fws0)
    f1.record(stream)
    torch.cuda.synchronize()
    forward_ms = f0.elapsed_time(f1) / nf
    assert spr.sparsepr_workspace_error(p, fws0) == 0
    del fws0, o_fwd

    # --- end to end through the C ABI from pinned host buffers
    Qh, Kh, Vh = (torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(3))
    Qh.copy_(Q.cpu()); Kh.copy_(K.cpu()); Vh.copy_(V.cpu())
    Oh = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    qkv_dev = torch.empty((3,) + tuple(Q.shape), dtype=torch.bfloat16, device=dev)
    o_dev = torch.empty_like(Q)
    fws = spr.workspace(p, dev, forward=True)
    e2e_steps = max(2, min(args.steps, 5))
    timed_launches = launches[0]
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
    e2e_single = e2e_total / (e2e_steps * ws)
    bytes_in = 3 * BH * N * d * 2
    # the same call through the library's pipeline over head chunks: the host-to-device
    # copies of chunk i + 1 and the device-to-host copy of chunk i - 1 run beside the
    # compute of chunk i (one C-ABI call per step; same outputs as the unsplit call)
    del fws
    oh_single = Oh.clone()
    n_chunks = next(c for c in (5, 4, 2, 1) if BH >= c)
    cws = spr.workspace(spr.chunk_params(p, n_chunks), dev, forward=True)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    for _ in range(2):
        spr.sparsepr_forward_host_chunked(p, Qh, Kh, Vh, Oh, qkv_dev, o_dev, n_chunks, cws, s_in, s_out)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(e2e_steps):
        spr.sparsepr_forward_host_chunked(p, Qh, Kh, Vh, Oh, qkv_dev, o_dev, n_chunks, cws, s_in, s_out)
    c1.record(stream)
    torch.cuda.synchronize()
    pipe_ms = c0.elapsed_time(c1) / e2e_steps
    e2e_value = max_over_ranks(pipe_ms, ws, dev) / ws
    e2e_same = bool(torch.equal(Oh, oh_single))
    del qkv_dev, o_dev, cws

    # --- a second seed of the generator (rank r draws seed 2 r + s): one call, its own dense
    seeds = {"0": {"ms_per_call": round(ms_per_call, 4), "o_sparse": round(err_sparse, 5),
                   "o_reconstructed": round(err_recon, 5)}}
    if args.seed1:
        q1, k1, v1 = (to_torch(x, dev) for x in generate(w, seed=2 * rank + 1))
        for _ in range(2):
            call(q1, k1, v1)
        torch.cuda.synchronize()
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        n1 = max(3, min(args.steps, 10))
        s0 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(n1):
            call(q1, k1, v1, ev1)
        torch.cuda.synchronize()
        ms1 = s0.elapsed_time(ev1[4]) / n1
        spr.sparsepr_dense_attention(p, q1, k1, v1, o_dense, None, wsb)
        torch.cuda.synchronize()
        seeds["1"] = {"ms_per_call": round(ms1, 4), "o_sparse": round(rel(o_sparse, o_dense), 5),
                      "o_reconstructed": round(rel(o, o_dense), 5)}
        del q1, k1, v1

    traffic = _traffic_record("attend_causal" if w.frame_causal else "attend")
    rho = part["rho_exec"].float()
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, {"streams": "attend and probe_fit on two streams" if side is not None
                              else "one stream"}),
        "stage_ms": {"partition": round(stage_ms[0], 4), "attend": round(stage_ms[1], 4),
                     ("probe_fit" if side is None else "probe_fit_wait"): round(stage_ms[2], 4),
                     "reconstruct": round(stage_ms[3], 4)},
        "forward_ms": {"value": round(forward_ms, 4),
                       "how": "sparsepr_forward on device buffers: the whole call in one C-ABI call, its probe "
                              "path on a second stream of the call's own"},
        "dense_attention_ms": round(dense_ms, 4),
        "speedup_vs_dense": round(dense_ms / ms_per_call, 3),
        "rho_exec": {"mean": round(float(rho.mean()), 5), "min": round(float(rho.min()), 5),
                     "max": round(float(rho.max()), 5)},
        "attend_ms_alone": round(attn_ms, 4),
        "attend_tflops_useful": round(achieved, 2),
        "attend_tflops_issued": round(issued_tflops, 2),
        "tile_fill": round(routed_pairs / max(1, issued_pairs), 4),
        "dense_equiv_tflops": round(dense_flops / (ms_per_call * 1e-3) / 1e12, 2),
        "dense_kernel_tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 2),
        "rel_l2_vs_dense": {"o_sparse": round(err_sparse, 5), "o_reconstructed": round(err_recon, 5),
                            "o_reconstructed_by_fit_input": fit_errors},
        "roofline": {"kernel": "attend (routed flash attention)", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": pk["bf16"], "unit": "TFLOP/s", "frac": round(achieved / pk["bf16"], 4),
                     "peak_kind": f"bf16 burst, {pk['src']} (the attend stage is timed alone, {n_iso} launches "
                                  f"back to back, {attn_ms * n_iso:.1f} ms)",
                     "frac_issued": round(issued_tflops / pk["bf16"], 4),
                     "frac_of_sustained": round(achieved / pk["bf16_sus"], 4),
                     "traffic": traffic, "algorithmic_flops_per_launch": attn_flops,
                     "algorithmic_unit": "4 d flops per routed (query, key) pair of the call's route"},
        "e2e": {"value": round(e2e_value, 4), "unit": UNIT, "h2d_bytes_per_step": bytes_in,
                "d2h_bytes_per_step": BH * N * d * 2,
                "how": f"pinned host Q, K, V -> device -> O back to pinned host in one C-ABI call, "
                       f"sparsepr_forward_host_chunked: {n_chunks} head chunks (head_offset numbering, so the "
                       f"output is the unsplit call's), copies in / compute / copies out on three streams",
                "single_call_ms": round(e2e_single, 4),
                "single_call_how": "sparsepr_forward_host: copies, call and copy back in sequence on one stream",
                "same_output_as_single_call": e2e_same},
        "seeds": seeds,
        "gpu_launches": timed_launches,
        "clocks": clk.summary(),
    }
    if calls > 1:
        line["ms_per_call"] = round(ms_per_call, 4)
    if args.weighted_fit:
        line["config"]["fit"] = "weighted ridge (probe weights n_a / probes of group a)"
    if args.partition != "coupled":
        line["config"]["partition"] = "semantic-grouping baseline (keys and queries clustered on raw rows)"
    if args.diagnostics:
        line["diagnostics"] = partition_diagnostics(part, Ql, Kl, o_sparse, o_dense, p, frames)
    if rank == 0 and ws == 1 and not args.heads:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0 and ws == 1 and not args.heads and args.others and args.workload == WORKLOAD:
        line["other_workloads"] = {}
        for n in ("world", "long"):
            try:
                line["other_workloads"][n] = other_workload(n, dev, spr, pk)
            except Exception as e:   # reported in the line; the main measurement above stands
                line["other_workloads"][n] = {"error": f"{type(e).__name__}: {e}"[:300]}
                break
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def other_workload(name, dev, spr, pk, steps=2, warmup=2):
    """A compact measurement of another workload of the pages in the same run: ms per call
    (partition -> attend beside probe_fit -> reconstruct, on one stream plus a side stream),
    the attend stage alone with its useful-pair TFLOP/s, this build's dense (frame-causal:
    causal dense) kernel on the same inputs, and both outputs' rel-L2 against it."""
    import numpy as np
    import torch
    from synth import frame_index, generate, perturb, to_torch
    w = bench_workload(argparse.Namespace(workload=name), heads=False)
    pd = dict(B=w.B, H=w.H, N=w.N, d=w.d, block=w.block, density=w.density, n_kgroups=w.n_kgroups,
              n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes, eig_rank=w.eig_rank,
              sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, ridge_lambda=w.ridge_lambda, seed=0)
    frames = frame_index(w.grid) if w.frame_causal else None
    fid = torch.from_numpy(frames).to(dev) if frames is not None else None
    p = spr.Params.make(**pd, frame_id=fid, n_frames=w.grid[0] if frames is not None else 0)
    t_gen = time.perf_counter()
    qb, kb, vb = generate(w, seed=0)
    calls = ROLLOUT_CALLS if w.frame_causal else 1
    inputs = []
    for c in range(calls):
        if c > 0:
            qb, kb, vb = (perturb(x, ROLLOUT_SIGMA, j, c) for j, x in enumerate((qb, kb, vb)))
        inputs.append(tuple(to_torch(x, dev) for x in (qb, kb, vb)))
    del qb, kb, vb
    t_gen = time.perf_counter() - t_gen
    Q, K, V = inputs[-1]
    wsb = spr.workspace(p, dev)
    part = spr.alloc_partition(p, dev)
    pr = spr.alloc_probe(p, dev)
    o_sparse, o = torch.empty_like(Q), torch.empty_like(Q)
    lse = torch.empty(p.BH, p.N, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev, priority=-1)
    fork = [torch.cuda.Event() for _ in range(2)]

    def call(Qc, Kc, Vc):
        spr.sparsepr_partition(p, Qc, Kc, part["perm_q"], part["perm_k"], part["label_q"], part["label_k"],
                               part["qoff"], part["koff"], part["route"], part["block_mask"], part["rho_exec"], wsb)
        fork[0].record(stream)
        side.wait_event(fork[0])
        with torch.cuda.stream(side):
            spr.sparsepr_probe_fit(p, Qc, Kc, Vc, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                                   pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"], pr["W"], None, wsb)
            fork[1].record(side)
        spr.sparsepr_attend(p, Qc, Kc, Vc, part["perm_q"], part["perm_k"], part["qoff"], part["koff"],
                            part["route"], o_sparse, lse, wsb)
        stream.wait_event(fork[1])
        spr.sparsepr_reconstruct(p, o_sparse, pr["probe_idx"], pr["probe_o_dense"], pr["b_full"], pr["Vr"],
                                 pr["W"], o)

    for _ in range(warmup):
        for x in inputs:
            call(*x)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, wsb) == 0
    e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    e[0].record(stream)
    for _ in range(steps):
        for x in inputs:
            call(*x)
    e[1].record(stream)
    for _ in range(3):
        spr.sparsepr_attend(p, Q, K, V, part["perm_q"], part["perm_k"], part["qoff"], part["koff"], part["route"],
                            o_sparse, lse, wsb)
    e[2].record(stream)
    o_dense = torch.empty_like(Q)
    spr.sparsepr_dense_attention(p, Q, K, V, o_dense, None, wsb)
    e[3].record(stream)
    for _ in range(2):
        spr.sparsepr_dense_attention(p, Q, K, V, o_dense, None, wsb)
    e[4].record(stream)
    call(Q, K, V)   # the last call's outputs, for the errors below
    # the other reading of the affine map's input on the same partition and sparse output
    p_alt = spr.Params.make(**dict(pd, fit_input=1), frame_id=fid, n_frames=w.grid[0] if frames is not None else 0)
    pr_alt = spr.alloc_probe(p_alt, dev)
    spr.sparsepr_probe_fit(p_alt, Q, K, V, part["label_k"], part["perm_q"], part["qoff"], part["route"],
                           pr_alt["probe_idx"], pr_alt["probe_o_dense"], pr_alt["b_full"], pr_alt["Vr"], pr_alt["W"],
                           None, wsb)
    o_alt = torch.empty_like(Q)
    spr.sparsepr_reconstruct(p_alt, o_sparse, pr_alt["probe_idx"], pr_alt["probe_o_dense"], pr_alt["b_full"],
                             pr_alt["Vr"], pr_alt["W"], o_alt)
    torch.cuda.synchronize()
    assert spr.sparsepr_workspace_error(p, wsb) == 0
    ms = e[0].elapsed_time(e[1]) / (steps * calls)
    attn_ms = e[1].elapsed_time(e[2]) / 3
    dense_ms = e[3].elapsed_time(e[4]) / 2
    useful, issued = attention_pairs(part, frames)
    rel = lambda a, b: float((a.float() - b.float()).norm() / b.float().norm())
    out = {"config": _config(w), "ms_per_call": round(ms, 4), "calls_timed": steps * calls,
           "attend_ms_alone": round(attn_ms, 4),
           "attend_tflops_useful": round(4.0 * w.d * useful / (attn_ms * 1e-3) / 1e12, 2),
           "attend_frac_useful": round(4.0 * w.d * useful / (attn_ms * 1e-3) / 1e12 / pk["bf16"], 4),
           "tile_fill": round(useful / max(1, issued), 4),
           ("causal_dense_attention_ms" if frames is not None else "dense_attention_ms"): round(dense_ms, 4),
           "speedup_vs_dense": round(dense_ms / ms, 3),
           "rho_exec_mean": round(float(part["rho_exec"].float().mean()), 5),
           "rel_l2_vs_dense": {"o_sparse": round(rel(o_sparse, o_dense), 5), "o_reconstructed": round(rel(o, o_dense), 5),
                               "o_reconstructed, map input projected on the subspace": round(rel(o_alt, o_dense), 5)},
           "input_generation_s": round(t_gen, 1)}
    if w.name == "long":
        out["note"] = "128 K/V and query groups (the kernels' limit), not the ceil(N/256) = 422 of the pages' scale"
    del inputs, Q, K, V, wsb, part, pr, o_sparse, o, o_dense, lse, pr_alt, o_alt
    torch.cuda.empty_cache()
    return out


def bench_workload(args, heads=True):
    """The workload of this run with the command line's overrides."""
    from synth import workload
    over = {}
    if heads and getattr(args, "heads", 0):
        over["H"] = args.heads
    if getattr(args, "density", 0.0):
        over["density"] = args.density
    if getattr(args, "groups", 0):
        over.update(n_kgroups=args.groups, n_qgroups=args.groups)
    elif getattr(args, "workload", WORKLOAD) == "long":
        # the kernels take at most 128 groups; the 108,000-token workload runs at that limit
        over.update(n_kgroups=128, n_qgroups=128)
    return workload(getattr(args, "workload", WORKLOAD), **over)


def partition_diagnostics(part, Q, K, o_sparse, o_dense, p, frames=None, heads=(0, 1), groups=16, mass=0.9):
    """Measurements of the partition on a few heads (torch on the device; reporting only).

    support: the fraction of keys that holds `mass` of a query's softmax, per query and
    for the pooled distribution (mean of the member rows) of each of `groups` query
    groups (the groups' queries would share one key set).  affine: the share of the
    residual O_dense - O_sparse that a least-squares affine map of O_sparse explains over
    all rows, and the unexplained energy relative to the residual energy."""
    import torch
    H, N = p.H, p.N
    s = p.eff_scale()
    out = {"heads": list(heads), "mass": mass, "groups_per_head": groups}
    perq, pooled, expl, unexpl = [], [], [], []
    fr = None if frames is None else torch.as_tensor(frames, device=Q.device).long()
    for bh in heads:
        b, h = divmod(bh, H)
        lq = part["label_q"][bh].long()
        sizes = torch.bincount(lq, minlength=p.n_qgroups)
        cand = torch.nonzero(sizes > 0).flatten()
        pick = cand[torch.linspace(0, cand.numel() - 1, min(groups, cand.numel())).round().long()]
        k = K[b, h].double()
        for a in pick.tolist():
            rows = torch.nonzero(lq == a).flatten()
            logits = s * (Q[b, h, rows].double() @ k.T)
            if fr is not None:
                logits = logits.masked_fill(fr[None, :] > fr[rows][:, None], float("-inf"))
            pr = torch.softmax(logits, dim=1)

            def frac(x):
                srt = torch.sort(x, dim=-1, descending=True).values
                need = (torch.cumsum(srt, dim=-1) < mass * srt.sum(-1, keepdim=True) * (1 - 1e-12)).sum(-1) + 1
                return need.clamp(max=x.shape[-1]).double() / x.shape[-1]
            perq.extend(frac(pr).tolist())
            pooled.append(float(frac(pr.mean(0))))
        x = o_sparse[b, h].double()
        r = o_dense[b, h].double() - x
        xa = torch.cat([torch.ones(N, 1, dtype=x.dtype, device=x.device), x], dim=1)
        coef = torch.linalg.lstsq(xa, r).solution
        un = float(((r - xa @ coef) ** 2).sum())
        tot = float((r ** 2).sum())
        expl.append(1.0 - un / tot)
        unexpl.append(un / tot)
    out["per_query_support"] = round(sum(perq) / len(perq), 5)
    out["grouped_support"] = round(sum(pooled) / len(pooled), 5)
    out["affine_explainable"] = round(sum(expl) / len(expl), 5)
    out["unexplained_energy_rel"] = round(sum(unexpl) / len(unexpl), 5)
    return out


def attention_pairs(part, frames=None):
    """(useful, MMA-issued) query-key pairs of the routed attention of the last call.

    useful: routed pairs (frame-causal: routed pairs whose key frame <= query frame).
    issued: per 256-row unit of a query group, its 128-row q-tiles times the 128-key
    chunks of the key stream each walks: all routed keys of the group, or (frame-causal)
    the routed keys of frames <= the frame of the tile's last row for the unit's first
    tile and of the unit's last row for its second."""
    import numpy as np
    qoff = part["qoff"].long().cpu().numpy()
    koff = part["koff"].long().cpu().numpy()
    route = part["route"].long().cpu().numpy()
    nq, nk = np.diff(qoff, axis=1), np.diff(koff, axis=1)
    if frames is None:
        useful = int((nq[:, :, None] * nk[:, None, :] * route).sum())
        ntile = (nq + 127) // 128
        rk = (nk[:, None, :] * route).sum(-1)
        return useful, int((ntile * 128 * ((rk + 127) // 128) * 128).sum())
    label_q = part["label_q"].long().cpu().numpy()
    label_k = part["label_k"].long().cpu().numpy()
    perm_q = part["perm_q"].long().cpu().numpy()
    fr = np.asarray(frames, np.int64)
    F = int(fr.max()) + 1
    Gq, Gk = route.shape[1], route.shape[2]
    useful = issued = 0
    for bh in range(route.shape[0]):
        hist_q = np.zeros((Gq, F), np.int64)
        np.add.at(hist_q, (label_q[bh], fr), 1)
        vis_k = np.zeros((Gk, F), np.int64)
        np.add.at(vis_k, (label_k[bh], fr), 1)
        vis_k = np.cumsum(vis_k, axis=1)
        useful += int(((hist_q @ vis_k.T) * route[bh]).sum())
        tl = route[bh] @ vis_k                      # [Gq, F] stream prefix per frame
        for a in range(Gq):
            for u0 in range(qoff[bh, a], qoff[bh, a + 1], 256):
                rows = min(256, qoff[bh, a + 1] - u0)
                p_last = int(tl[a, fr[perm_q[bh, u0 + rows - 1]]])
                chunks = (p_last + 127) // 128
                if rows > 128:
                    chunks += (min(int(tl[a, fr[perm_q[bh, u0 + 127]]]), p_last) + 127) // 128
                issued += chunks * 128 * 128
    return useful, issued


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
    from synth import frame_index
    fr = frame_index(w.grid).astype(np.int64) if w.frame_causal else None
    t0 = time.perf_counter()
    part = O.partition_head(q, k, p, 0, frames=fr)
    t1 = time.perf_counter()
    n_rows = max(1, int(w.N * rows_frac))
    rows = np.arange(0, w.N, w.N // n_rows)[:n_rows]
    o_s, _ = O.sparse_attention(q, k, v, s, part.route.route, part.label_q, part.label_k, rows=rows, frames=fr)
    t2 = time.perf_counter()
    fit = O.probe_fit_head(q, k, v, part.label_q, part.label_k, part.route.route, part.perm_q, part.q_offsets, p, 0,
                           frames=fr)
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


def oracle_whole(name: str, threads=None, seed=0):
    """Seconds of the oracle's whole call (every head, every row) on a small workload;
    threads: cap on the BLAS threads (None: as configured)."""
    import contextlib
    import oracle as O
    from synth import generate, to_f64, workload
    w = workload(name)
    qb, kb, vb = generate(w, seed=seed)
    p = O.Params(n_kgroups=w.n_kgroups, n_qgroups=w.n_qgroups, n_samples=w.n_samples, n_probes=w.n_probes,
                 eig_rank=w.eig_rank, sub_rank=w.sub_rank, kmeans_iters=w.kmeans_iters, density=w.density,
                 ridge_lambda=w.ridge_lambda, seed=seed, block=w.block)
    ctx = contextlib.nullcontext()
    if threads is not None:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(threads)
    with ctx:
        t0 = time.perf_counter()
        for b in range(w.B):
            for h in range(w.H):
                O.sparsepr_head(to_f64(qb[b, h]), to_f64(kb[b, h]), to_f64(vb[b, h]), p, b * w.H + h)
        return time.perf_counter() - t0


def cpu_baseline(w):
    sec, spent, nrows = oracle_sample(w)
    whole = {"tiny (1024 tokens x 2 heads)": round(oracle_whole("tiny"), 3),
             "tiny, 1 thread": round(oracle_whole("tiny", threads=1), 3),
             "mid (8192 tokens x 12 heads)": round(oracle_whole("mid"), 2)}
    return {"value": round(sec * 1e3, 1), "unit": UNIT, "cores": _cores(), "kind": "oracle",
            "sample": f"head (0,0) of {w.B * w.H}: full partition, probes and fit; routed attention and "
                      f"correction on {nrows} of {w.N} rows; extrapolated x{w.B * w.H} heads "
                      f"(took {spent:.1f} s)",
            "whole_call_s": whole}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    from synth import workload
    w = bench_workload(args, heads=False)
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
    ap.add_argument("--workload", default=WORKLOAD, choices=["wan", "world", "long"],
                    help="wan: the 32,760-token call (default); world: the frame-causal rollout; "
                         "long: 108,000 tokens x 24 heads with a per-frame drift (128 groups)")
    ap.add_argument("--groups", type=int, default=0, help="override the K/V and query group counts")
    ap.add_argument("--partition", default="coupled", choices=["coupled", "semantic"],
                    help="coupled: the method; semantic: the semantic-grouping baseline of the pages")
    ap.add_argument("--density", type=float, default=0.0, help="override the workload's target density")
    ap.add_argument("--weighted-fit", action="store_true", help="weight the probes of the ridge fit")
    ap.add_argument("--diagnostics", action="store_true",
                    help="add support and affine-explainability measurements of two heads to the line")
    ap.add_argument("--streams", type=int, default=2, choices=[1, 2],
                    help="2: probe_fit beside the routed attention on a second stream (default); 1: in sequence")
    ap.add_argument("--no-seed1", dest="seed1", action="store_false",
                    help="skip the one-call measurement on the generator's second seed")
    ap.add_argument("--no-others", dest="others", action="store_false",
                    help="skip the compact measurements of the rollout and 108,000-token workloads")
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
