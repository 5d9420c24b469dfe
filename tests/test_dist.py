"""Multi-rank host logic of bench.py on CPU with gloo (world size 2): each rank runs its
own copy of the workload (seed = rank), time is the max over ranks, and only rank 0
prints. No data-path collective exists to test."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_init()
    got = bench.max_over_ranks(1.5 + r, w)
    bench.barrier(w)
    ref = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), w, r) if r != 0 else None
    wl = bench.W.WORKLOADS[bench.DECODE_WL].with_(seed=r)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, got, ref, wl.seed))


@pytest.mark.timeout(180)
def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, got, ref, seed in out:
        assert w == 2
        assert got == 2.5                 # max over ranks of 1.5 + rank
        assert seed == r                  # independent inputs per rank
        if r == 1:
            assert ref is None            # only rank 0 runs / prints the reference arm
