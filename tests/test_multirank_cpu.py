"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The single system does not shard without a halo exchange (out of scope), so
several GPUs run independent replicas: every rank solves its own seeded system,
the job time is the slowest rank's and the work is the sum over ranks.
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
