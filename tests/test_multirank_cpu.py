"""The replica (weak-scaling) logic of bench.py on two gloo ranks on CPU:
each rank gets its own token batch, and the timing reduction is the max over
ranks that every rank sees."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys

    import torch.distributed as dist

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle
        from combine_ep_get_10_b200 import workloads as W

        seed = bench.rank_seed(2, rank)
        inp = W.make_inputs(2, seed=seed, T=64)
        L = oracle.tc_layout(inp["topk_idx"], 256, 8)
        local_ms = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(local_ms, world)
        q.put((rank, seed, inp["topk_idx"].tobytes(), int(L["expert_offsets"][-1]), got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_reduction():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] != res[1][1]  # distinct seeds
    assert res[0][2] != res[1][2]  # distinct token batches
    assert all(r[3] == 64 * 8 for r in res)  # every pair valid in workload 2
    assert all(r[4] == 15.0 for r in res)  # both ranks see the max
