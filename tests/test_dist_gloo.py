"""The multi-rank host logic of bench.py on the CPU: two gloo ranks set up the process
group from torchrun-style environment variables, meet at the barrier, and agree on the
max over ranks of their timings (the figure the benchmark reports for N > 1)."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist

    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    vals = bench.max_over_ranks(w, [1.0 + rank, 10.0 - rank, 0.5 * rank], torch.device("cpu"))
    out[rank] = vals
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_over_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 0.5]


def test_single_rank_needs_no_process_group():
    import bench

    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_setup("gloo") == (1, 0, 0)
    assert bench.max_over_ranks(1, [3.0], torch.device("cpu")) == [3.0]
