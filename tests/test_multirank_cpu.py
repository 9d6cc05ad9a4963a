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


# ---- context parallelism: slice bounds and the record exchange (gloo)

def test_slice_bounds_partition_the_context():
    from compressed_decode_attention_b200.context_parallel import slice_bounds
    for n in (0, 1, 63, 64, 65, 1000, 32768):
        for world in (1, 2, 3, 8):
            spans = [slice_bounds(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, _) in zip(spans, spans[1:]):
                assert b == c and a <= b
            assert all(a % 64 == 0 or a == n for a, _ in spans)


def _cp_worker(rank, world, port, results):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    from compressed_decode_attention_b200 import context_parallel as cp
    from oracle import attention
    import test_oracle_attention as ta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(21)                 # the same cache on every rank
        B, Hkv, cap, d, seed, gqa = 2, 2, 200, 128, 3, 2
        arrs = ta._cache(B, Hkv, cap, d, 4, 2, seed, rng)
        q = rng.standard_normal((B, Hkv * gqa, d)) * 2
        ctx = np.array([200, 70])
        a, b = cp.slice_bounds(cap, world, rank)
        loc = cp.local_ctx_lens(ctx, a, b)
        part = [x[:, :, a:b] for x in arrs]
        rec, _ = attention.attend_partial(q, *part, loc, gqa, 4, 2, seed, 0.02)
        mine = torch.from_numpy(rec)
        gathered = torch.empty((world,) + mine.shape, dtype=mine.dtype)
        cp.gather_records(mine, gathered)
        got = attention.combine(gathered.numpy(), seed)
        want, _ = attention.attend(q, *arrs, ctx, gqa, 4, 2, seed, 0.02)
        results[rank] = float(np.abs(got - want).max())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange_matches_one_pass(world):
    """Every rank holds one slice; after the all-gather of the records each
    rank's merge equals the one-pass attention over the whole context."""
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_cp_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    assert len(results) == world
    assert max(results.values()) < 1e-12
