"""Multi-process plumbing on CPU: world_size-2 gloo process groups (no GPU).

The decode path shards whole agents over ranks with no data-path collective;
what needs checking is the host logic: every agent on exactly one rank, the
slowest rank's time as the job time, and whole-job throughput aggregation."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from quantized_kv_cache_dequantize_b200 import dist as kdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    r, w, _ = kdist.init_from_env(timeout_s=30)
    t = kdist.max_over_ranks(1.0 + r * 2.5)          # rank 1 is the slow one
    kdist.barrier()
    agents = kdist.shard_agents(10, r, w)
    q.put((r, w, t, agents))
    kdist.shutdown()


def test_two_rank_gloo_max_and_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 3.5 for r in res)             # both ranks see the max
    assigned = res[0][3] + res[1][3]
    assert sorted(assigned) == list(range(10))        # each agent exactly once


@pytest.mark.parametrize("n,world", [(10, 1), (10, 3), (7, 8), (64, 8)])
def test_shard_agents_partition(n, world):
    parts = [kdist.shard_agents(n, r, world) for r in range(world)]
    flat = [a for p in parts for a in p]
    assert sorted(flat) == list(range(n))
    sizes = [len(p) for p in parts]
    assert max(sizes) - min(sizes) <= 1


def test_single_process_identity_and_aggregate():
    assert kdist.max_over_ranks(2.0) == 2.0
    assert kdist.aggregate_throughput(100.0, 4, 2.0) == 200.0
