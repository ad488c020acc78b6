"""Multi-rank host logic on CPU (gloo, world size 2).

The single system does not shard without a halo exchange (out of scope), so
several GPUs run independent replicas: every rank solves its own seeded system,
the job time is the slowest rank's and the work is the sum over ranks.  One
batch of independent systems does shard: each rank solves a contiguous range
of it, and the results are gathered once afterwards.
"""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    t, w = bench.reduce_over_ranks(10.0 + 5.0 * rank, 2000.0 + rank, "cpu")
    wl = bench.load_workload("c1", rank)
    out[rank] = (t, w, float(wl.b[0][:8].sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_reduce_max_time_and_sum_work():
    world = 2
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0            # slowest rank's time
    assert out[0][1] == out[1][1] == 4001.0          # every rank's iterations
    assert out[0][2] != out[1][2]                    # each replica has its own seeded system


def test_single_rank_passes_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(12.5, 300, "cpu") == (12.5, 300.0)


# ------------------------------------------------ one batch split over ranks ----

def test_shard_ranges_cover_every_system_once():
    sys.path.insert(0, ROOT)
    from differentiable_sparse_linear_csr_b200.sharding import shard_range
    for total in (0, 1, 3, 4, 7, 1024, 1025):
        for world in (1, 2, 3, 4, 8):
            ranges = [shard_range(total, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))       # contiguous, no overlap
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


def _split_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    import numpy as np
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from differentiable_sparse_linear_csr_b200 import workloads as W
    from differentiable_sparse_linear_csr_b200.sharding import gather_shards, shard_range
    from oracle import oracle as O
    w = W.c4_batched(B=5, N=10)                   # the same batch on every rank
    lo, hi = shard_range(w.batch, world, rank)
    # this rank's systems: forward solve, adjoint, value gradient (the oracle stands
    # in for the GPU library on CPU)
    x, _ = O.pcg(w.rowptr, w.colind, w.values[lo:hi], w.b[lo:hi], rtol=1e-10)
    lam, _ = O.cg_adjoint(w.rowptr, w.colind, w.values[lo:hi], x - w.xstar[lo:hi], rtol=1e-10)
    G = O.grad_values(w.rowptr, w.colind, lam, x)
    out[rank] = {k: gather_shards(torch.from_numpy(np.ascontiguousarray(v)), w.batch).numpy()
                 for k, v in (("x", x), ("lam", lam), ("G", G))}
    dist.barrier()
    dist.destroy_process_group()


def test_split_batch_reassembles_the_single_process_batch():
    """Two ranks each solve their shard of one 5-system batch; the gathered
    solutions, adjoints and gradients equal the single-process batch bit for bit
    on both ranks (the systems are independent and each is computed alike)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    from differentiable_sparse_linear_csr_b200 import workloads as W
    from oracle import oracle as O
    world = 2
    out = mp.Manager().dict()
    mp.start_processes(_split_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    w = W.c4_batched(B=5, N=10)
    x, _ = O.pcg(w.rowptr, w.colind, w.values, w.b, rtol=1e-10)
    lam, _ = O.cg_adjoint(w.rowptr, w.colind, w.values, x - w.xstar, rtol=1e-10)
    G = O.grad_values(w.rowptr, w.colind, lam, x)
    for rank in range(world):
        assert np.array_equal(out[rank]["x"], x)
        assert np.array_equal(out[rank]["lam"], lam)
        assert np.array_equal(out[rank]["G"], G)
