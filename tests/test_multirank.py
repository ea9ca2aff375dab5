"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own independent problem (distinct seeds, weak scaling);
the job's time is the max over ranks and its throughput counts the tokens of
all ranks.  No GPU is involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import ssd_synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(backend="gloo")
    wl = ssd_synth.BY_NAME[bench.DEFAULT_WORKLOAD]
    ms = 100.0 + 50.0 * r                      # rank 1 is slower
    bench.barrier(w, r)
    m = bench.max_over_ranks(w, ms)
    q.put((r, m, bench.rank_seed(wl, r), bench.job_throughput(wl, w, 10, m)))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    wl = ssd_synth.BY_NAME["mamba2-0.3b-L1M-stream8"]
    assert [r[1] for r in res] == [150.0, 150.0]          # max over ranks on every rank
    assert res[0][2] != res[1][2]                         # independent problems per rank
    expect = wl.tokens * world * 10 / 0.150
    assert all(abs(r[3] - expect) / expect < 1e-12 for r in res)
