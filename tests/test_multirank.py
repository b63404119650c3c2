"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1)."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench._dist()
        # per-rank device times differ; every rank must see the slowest one
        mx = bench.max_over_ranks(10.0 * (rank + 1), w)
        q.put((rank, w, r, lr, mx, bench.job_ms_per_call(mx, 5, w)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, (r0, w, r, lr, mx, v) in enumerate(out):
        assert (r0, w, r, lr) == (rank, 2, rank, rank)
        assert mx == 20.0                      # max over ranks, not the rank's own time
        assert v == pytest.approx(20.0 / (5 * 2))   # 10 calls done in the slowest rank's time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_ms_per_call(50.0, 10, 1) == 5.0


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    called = []
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: called.append(1))

    class A:
        steps, warmup = 2, 3
    bench.run_reference(A())
    assert called == [] and capsys.readouterr().out == ""


def test_attention_pairs_counts_visible_routed_pairs():
    """bench.attention_pairs: the useful pairs are the routed (and, frame-causal,
    visible) token pairs counted one by one; the issued pairs cover them."""
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    import bench
    rng = np.random.default_rng(0)
    BH, N, Gq, Gk, F = 2, 300, 5, 7, 4
    frames = np.repeat(np.arange(F), N // F)
    lq = rng.integers(0, Gq, (BH, N))
    lk = rng.integers(0, Gk, (BH, N))
    route = (rng.random((BH, Gq, Gk)) < 0.4).astype(np.uint8)
    part = {"label_q": torch.from_numpy(lq), "label_k": torch.from_numpy(lk), "route": torch.from_numpy(route),
            "perm_q": torch.from_numpy(np.argsort(lq, axis=1, kind="stable")),
            "qoff": torch.from_numpy(np.stack([np.r_[0, np.cumsum(np.bincount(x, minlength=Gq))] for x in lq])),
            "koff": torch.from_numpy(np.stack([np.r_[0, np.cumsum(np.bincount(x, minlength=Gk))] for x in lk]))}
    for fr in (None, frames):
        useful, issued = bench.attention_pairs(part, fr)
        want = 0
        for bh in range(BH):
            m = route[bh][lq[bh]][:, lk[bh]].astype(bool)
            if fr is not None:
                m &= fr[None, :] <= fr[:, None]
            want += int(m.sum())
        assert useful == want
        assert issued >= useful and issued % (128 * 128) == 0
