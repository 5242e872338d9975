"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks.

The path shards by (sequence, head) with no exchange step, so the only
collectives are the barrier and the max over ranks of the timings."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.dist_env()
        seed = bench.rank_seed(1, r)
        bench.barrier(None)
        t = bench.reduce_max(10.0 + r, torch.device("cpu"))
        q.put((r, lr, w, seed, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_distinct_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    assert all(x[2] == world for x in res)
    assert res[0][3] != res[1][3]                 # independent batches per rank
    assert all(x[4] == 11.0 for x in res)         # the max over ranks reaches every rank


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.dist_env()[2] >= 1


def test_alg_bytes_and_flops_match_the_stated_per_unit_figures():
    import bench
    # per (token, head) at dk = dv = 128, bf16: 1,540 B and 132,437 flop
    assert bench.alg_bytes_prefill(1, 0, 128, 128, 2, False, False) == 1540
    assert bench.alg_flops_prefill(1, 128, 128) == 132437
    # prefill workload: 262,144 token-heads + 64 final states
    assert bench.alg_bytes_prefill(262144, 64, 128, 128, 2, False, True) == 407896064
    # decode: per (sequence, head, step)
    assert bench.alg_bytes_decode(1, 128, 128, 2) == 132612
