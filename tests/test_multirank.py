"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, each with its own timing,
agree on the job time (the max over ranks) after a barrier.  Decode batches shard with
no data-path collective, so this max and the barrier are the only communication."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier(world)
    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    job = bench.max_over_ranks(local_ms, world)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, job))


def test_two_gloo_ranks_take_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_byte_model_matches_the_per_token_formula():
    import bench
    from sparse_attention_long_03_b200 import workloads as W
    cfg = W.CONFIGS["decode_128k"]
    lens = [100000, 70000]
    m = bench.algorithmic_bytes(cfg, lens)
    # 132*L + 2,646,788 bytes per query token: keys 132*L, indexer query 8452,
    # gathered rows 2048*1152, q 147456, out 131072, LSE 512
    assert m["total"] == sum(132 * L + 2646788 for L in lens)
    assert m["gather"] == 2 * 2048 * 1152
