"""The cross-GPU exchange (combine_ep_get_10_b200/ep_exchange.py) with its
CUDA compute steps, on a one-rank NCCL group (the runs here have one GPU):
per-rank dispatch, counts exchange, NCCL all-to-all-v of the rows and their
top-k entries, the local experts through layout -> dispatch -> combine, the
reverse exchange and the rank-level combine.  With one rank every token's
experts sit in that rank, so the result equals the oracle's per-expert
combine of bf16(x * (e + 1)) expert outputs, rounded to bf16 once as the
partial row and once more (exactly) after the sum over the one rank.  The
multi-rank protocol is covered on CPU processes (test_ep_exchange_cpu.py)."""
import socket

import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_exchange_on_one_rank_matches_the_oracle():
    import torch.distributed as dist

    from combine_ep_get_10_b200.ep_exchange import ExpertParallel

    inp = W.make_inputs(2, T=512)
    c = inp["cfg"]
    E, H = c["E"], 1024
    x = np.ascontiguousarray(inp["x"][:, :H])
    idx, w = inp["topk_idx"], inp["topk_weights"]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        ep = ExpertParallel(E)

        def experts(rows, offsets):
            out = torch.empty_like(rows)
            off = offsets.tolist()
            for e in range(E):
                if off[e + 1] > off[e]:
                    out[off[e]:off[e + 1]] = (rows[off[e]:off[e + 1]].float() * (e + 1)).to(torch.bfloat16)
            return out

        recv = ep.dispatch(to_dev(x, bf16=True), to_dev(idx), to_dev(w))
        assert recv.recv_counts == [int((idx >= 0).any(axis=1).sum())]
        y = ep.experts(recv, experts)
        out = ep.combine(y, recv, torch.bfloat16)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    L = oracle.tc_layout(idx, E, 1)
    yf = oracle.tc_dispatch(x, idx, E, L)["recv"]
    for e in range(E):
        a, b = int(L["expert_offsets"][e]), int(L["expert_offsets"][e + 1])
        if b > a:
            yf[a:b] = oracle.f32_to_bf16((oracle.bf16_to_f32(yf[a:b]) * np.float32(e + 1)).astype(np.float32))
    ref = oracle.tc_combine(yf, idx, E, L, w, out_dtype=oracle.BF16)
    assert np.array_equal(host(out), ref)


def _two_rank_worker(rank, world, port, q):
    import os
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from combine_ep_get_10_b200.ep_exchange import ExpertParallel
        from test_ep_exchange_cpu import E, _inputs

        ep = ExpertParallel(E)  # the CUDA compute steps
        x, idx, w = _inputs(rank, world)
        recv = ep.dispatch(to_dev(x, bf16=True), to_dev(idx), to_dev(w))
        first = rank * (E // world)

        def experts(rows, offsets):
            out = torch.empty_like(rows)
            off = offsets.tolist()
            for j in range(len(off) - 1):
                if off[j + 1] > off[j]:
                    out[off[j]:off[j + 1]] = (rows[off[j]:off[j + 1]].float() * (first + j + 1)).to(torch.bfloat16)
            return out

        y = ep.experts(recv, experts)
        out = ep.combine(y, recv, torch.bfloat16)
        torch.cuda.synchronize()
        q.put((rank, "ok", host(out)))
        dist.barrier()
    except BaseException:
        import traceback

        q.put((rank, "error", traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_ranks_sharing_the_gpu(world):
    """2 or 4 processes on the one GPU, each a rank of a gloo group (rows
    staged through host memory): the CUDA compute steps of every rank and the
    protocol between them give each rank the single-process oracle's
    two-level result bit for bit.  No kernel waits on another process."""
    import torch.multiprocessing as mp

    from test_ep_exchange_cpu import _reference

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_two_rank_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            item = q.get(timeout=300)
            assert item[1] == "ok", "rank %d failed:\n%s" % (item[0], item[2])
            res[item[0]] = item[2]
    finally:
        for p in procs:
            p.join(timeout=120 if len(res) == world else 5)
            if p.exitcode is None:
                p.kill()
    ref = _reference(oracle, world)
    for r in range(world):
        assert np.array_equal(res[r], ref[r]["two_bf16"]), r
