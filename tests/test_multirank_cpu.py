"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

bench.py scales by running one replica of the workload per rank (weak
scaling, no collective on the data path); its only cross-rank steps are a
barrier around the timed region and the maximum of the per-rank step time.
"""
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


def _worker(rank, world, port, results):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        bench.barrier()
        t = bench.reduce_max(1.5 + rank)           # per-rank step time
        results[rank] = t
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_ranks():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    assert dict(results) == {0: 2.5, 1: 2.5}


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.25) == 3.25


def test_weak_scaling_value_counts_all_ranks():
    """value = bytes of every rank / max step time (each rank one replica)."""
    import synthetic as S
    import bench
    w = S.WORKLOADS[bench.WORKLOAD]
    per_rank = bench.LAYERS * (bench.attend_bytes(w, w.ctx) + bench.encode_bytes(w, w.n_kv_heads))
    # 32 layers x (32768 x 8 x 100 B + 32 x 128 x 4 B + 8 x 612 B)
    assert per_rank == 32 * (32768 * 8 * 100 + 32 * 128 * 4 + 8 * 612)
