"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

The path shards over token rows with no data-path collective; the only
cross-rank steps are the barrier around the timed region and the reductions
of the timings (max) and work (sum).  These run here as two CPU processes.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(w)
        t_max = bench.max_over_ranks(10.0 + rank, w, "cpu")
        work = bench.sum_over_ranks(100.0 * (rank + 1), w, "cpu")
        # every rank holds its own batch of the same shape (weak scaling)
        x = torch.arange(12, dtype=torch.float32).reshape(4, 3)
        xr = x if rank == 0 else x.roll(rank, 0).contiguous()
        out[rank] = (t_max, work, float(xr[0, 0]))
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()


def test_two_rank_reductions():
    port = _free_port()
    ctx = mp.get_context("spawn")  # never fork: this process may already run the oracle's OpenMP threads
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][:2] == (11.0, 300.0) and out[1][:2] == (11.0, 300.0)
    assert out[0][2] != out[1][2]  # distinct batches per rank


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.sum_over_ranks(2.0, 1, "cpu") == 2.0
    bench.barrier(1)


def test_workload_table():
    import bench
    layers = bench.workload_layers("esm2_ffn")
    assert [(g.M, g.K, g.N) for _, g, _ in layers] == [(8176, 480, 1920), (8176, 1920, 480)]
    assert bench.gemm_flops(layers[0][1]) == 2.0 * 8176 * 480 * 1920
    with pytest.raises(SystemExit):
        bench.workload_layers("nope")
