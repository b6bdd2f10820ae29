"""Host logic of the N > 1 benchmark path, on CPU with 2 gloo ranks: every rank
gets an independent batch of the same shape, the job time is the max over ranks,
and the whole-job value sums the ranks' work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import datetime

    import numpy as np
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import workloads as W
    r, w, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * r                                # rank 1 is the slow one
        mx = bench.reduce_max(mine, w, device="cpu")
        wl = bench.rank_workload(W.WORKLOADS["mha13b"], r)
        lens = W.context_lens(wl)
        q.put((r, w, local, mx, wl.seed, int(lens.sum()), wl.num_seqs))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, mx0, s0, t0, n0), (r1, w1, l1, mx1, s1, t1, n1) = out
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert mx0 == mx1 == 15.0                               # max over ranks, seen by every rank
    assert s0 != s1 and t0 != t1                            # independent batches ...
    assert n0 == n1                                         # ... of the same shape (weak scaling)


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.reduce_max(3.5, 1) == 3.5
