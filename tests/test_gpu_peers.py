"""The per-rank path over peer memory (ep_peer_publish_counts,
ep_dispatch_peers, ep_combine_peers; combine_ep_get_10_b200/ep_exchange.py
PeerExpertParallel) against the oracle's two-level composition.

The runs here have one GPU, so the ranks are emulated two ways, and neither
has a kernel that waits for another rank:
  * in one process: W sets of buffers on the one GPU, each rank's tables
    pointing at all of them, and the ranks' kernels launched one after the
    other on one stream, phase by phase (publish all, dispatch all, experts
    all, combine all);
  * in W processes sharing the GPU: buffers from ep_peer_alloc mapped into
    the other processes with ep_peer_open (CUDA IPC), a gloo group for the
    handles and the barriers between the phases.

Reference (the oracle, in one process from all ranks' inputs): per source
rank i, the oracle's rank layout and per-rank dispatch give the rows it
sends to each rank j; rank j receives source 0's rows first, each source's
rows in token order; rank j's experts turn each received row into one bf16
partial row (the oracle's layout -> dispatch -> expert -> combine over its
E/W local experts, expert e mapping x to bf16(x * (e + 1))); the oracle's
rank combine sums a token's partial rows over its ranks in ascending order.
Received rows, their entries and source tokens, and both output precisions
are compared bit for bit."""
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


def rank_inputs(rank, world, T, H, E, K=8, seed=9100):
    """Rank `rank`'s batch of the prefill routing recipe (sigmoid router with
    bias, top-K of E) at T tokens and H channels; every fourth token keeps
    its experts inside one rank, so single-rank and multi-rank tokens occur."""
    inp = W.make_inputs(2, seed=seed + rank, T=T)
    x = np.ascontiguousarray(inp["x"][:, :H])
    idx = np.ascontiguousarray(inp["topk_idx"][:, :K])
    w = np.ascontiguousarray(inp["topk_weights"][:, :K])
    el = E // world
    idx = idx % E
    for t in range(0, T, 4):
        idx[t] = idx[t] % el + (t % world) * el
    return x, idx, w


def expert_rows_oracle(rows_bits, offsets, first_expert):
    out = np.empty_like(rows_bits)
    for j in range(len(offsets) - 1):
        a, b = int(offsets[j]), int(offsets[j + 1])
        if b > a:
            f = oracle.bf16_to_f32(rows_bits[a:b]) * np.float32(first_expert + j + 1)
            out[a:b] = oracle.f32_to_bf16(f.astype(np.float32))
    return out


def expert_fn_for(first_expert):
    def fn(rows, offsets):
        out = torch.empty_like(rows)
        off = offsets.tolist()
        for j in range(len(off) - 1):
            if off[j + 1] > off[j]:
                out[off[j]:off[j + 1]] = (rows[off[j]:off[j + 1]].float() * (first_expert + j + 1)).to(torch.bfloat16)
        return out
    return fn


def two_level_reference(inputs, E, world):
    """Per rank r: what it receives (rows, entries, source tokens, counts
    per source) and its two-level outputs (bf16 and fp32)."""
    el = E // world
    sent = []
    for x, idx, w in inputs:
        L = oracle.tc_layout(idx, E, world)
        RL = oracle.rank_layout(L["is_token_in_rank"])
        D = oracle.rank_dispatch(x, idx, E, world, RL, topk_weights=w, want_src=True)
        sent.append((RL, D))
    ref = []
    for r in range(world):
        blocks = []
        for i in range(world):
            RL, D = sent[i]
            a, b = int(RL["rank_offsets"][r]), int(RL["rank_offsets"][r + 1])
            blocks.append((D["recv"][a:b], D["recv_topk_idx"][a:b], D["recv_topk_weights"][a:b],
                           D["recv_src"][a:b]))
        ref.append(dict(x=np.concatenate([b[0] for b in blocks]), idx=np.concatenate([b[1] for b in blocks]),
                        w=np.concatenate([b[2] for b in blocks]), src=np.concatenate([b[3] for b in blocks]),
                        counts=[len(b[0]) for b in blocks]))
    for i, (x, idx, w) in enumerate(inputs):
        RL, D = sent[i]
        back = np.empty_like(D["recv"])
        offs = RL["rank_offsets"]
        for r in range(world):
            a, b = int(offs[r]), int(offs[r + 1])
            if b == a:
                continue
            ridx = D["recv_topk_idx"][a:b]
            LL = oracle.tc_layout(ridx, el, 1)
            rows = oracle.tc_dispatch(D["recv"][a:b], ridx, el, LL)["recv"]
            yr = expert_rows_oracle(rows, LL["expert_offsets"], r * el)
            back[a:b] = oracle.tc_combine(yr, ridx, el, LL, D["recv_topk_weights"][a:b], out_dtype=oracle.BF16)
        ref[i]["out_bf16"] = oracle.rank_combine(back, RL, out_dtype=oracle.BF16)
        ref[i]["out_f32"] = oracle.rank_combine(back, RL, out_dtype=oracle.FP32)
    return ref


class LocalRanks:
    """W ranks' buffers on the one GPU and each rank's tables over all of
    them (the single-process emulation).  Unwritten memory holds patterns:
    NaN rows, index -7, weight NaN, source -9, counts -1."""

    def __init__(self, world, capacity, H, K, guard=0):
        self.world, self.capacity, self.H, self.K = world, capacity, H, K
        rows = capacity + guard
        d = "cuda"
        self.recv_x = [torch.full((rows, H), float("nan"), dtype=torch.bfloat16, device=d) for _ in range(world)]
        self.y = [torch.full((rows, H), float("nan"), dtype=torch.bfloat16, device=d) for _ in range(world)]
        self.idx = [torch.full((rows, K), -7, dtype=torch.int64, device=d) for _ in range(world)]
        self.w = [torch.full((rows, K), float("nan"), dtype=torch.float32, device=d) for _ in range(world)]
        self.src = [torch.full((rows,), -9, dtype=torch.int32, device=d) for _ in range(world)]
        self.counts = [torch.full((world, world), -1, dtype=torch.int32, device=d) for _ in range(world)]

        def table(ts):
            return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device=d)

        tabs = [table(self.recv_x), table(self.y), table(self.counts), table(self.idx), table(self.w),
                table(self.src)]
        self.peers = [B.Peers(r, capacity, tabs[0], tabs[1], tabs[2], recv_topk_idx=tabs[3], recv_topk_weights=tabs[4],
                              recv_src=tabs[5]) for r in range(world)]


def run_local(inputs, E, world, capacity, guard=0):
    """One step of every emulated rank, phase by phase on one stream."""
    H, K = inputs[0][0].shape[1], inputs[0][1].shape[1]
    L = LocalRanks(world, capacity, H, K, guard)
    state = []
    for r, (x, idx, w) in enumerate(inputs):
        xd, idd, wd = to_dev(x, bf16=True), to_dev(idx), to_dev(w)
        routing = B.Routing.topk(idd, E, world)
        layout = B.Layout(routing)
        B.ep_get_layout(routing, layout)
        rl = B.RankLayout(routing)
        B.ep_get_rank_layout(routing, layout, rl)
        B.ep_peer_publish_counts(routing, layout, L.peers[r])
        state.append((xd, idd, wd, routing, layout, rl))
    for r, (xd, idd, wd, routing, layout, rl) in enumerate(state):
        B.ep_dispatch_peers(xd, routing, layout, rl, L.peers[r], topk_weights=wd)
    torch.cuda.synchronize()
    return L, state


def finish_local(L, state, E, world, received):
    """Experts on every rank (partial rows into its y buffer), then every
    rank's combine in both precisions."""
    from combine_ep_get_10_b200.ep_exchange import CudaRowOps

    ops = CudaRowOps()
    el = E // world
    for r in range(world):
        n = received[r]
        ops.local_experts(L.recv_x[r][:n], L.idx[r][:n], L.w[r][:n], el, expert_fn_for(r * el), out=L.y[r][:n])
    outs = []
    for r, (xd, idd, wd, routing, layout, rl) in enumerate(state):
        ob = torch.empty((routing.T, L.H), dtype=torch.bfloat16, device="cuda")
        of = torch.empty((routing.T, L.H), dtype=torch.float32, device="cuda")
        B.ep_combine_peers(routing, layout, rl, L.peers[r], ob)
        B.ep_combine_peers(routing, layout, rl, L.peers[r], of)
        outs.append((ob, of))
    torch.cuda.synchronize()
    return outs


def check_step(L, state, inputs, E, world):
    ref = two_level_reference(inputs, E, world)
    full = np.array([host(L.counts[0])[i] for i in range(world)])
    for r in range(world):
        # every rank holds every rank's counts
        assert np.array_equal(host(L.counts[r]), full), r
        assert full[:, r].tolist() == ref[r]["counts"], r
    received = [int(full[:, r].sum()) for r in range(world)]
    for r in range(world):
        n = received[r]
        assert np.array_equal(host(L.recv_x[r][:n]), ref[r]["x"]), r
        assert np.array_equal(host(L.idx[r][:n]), ref[r]["idx"]), r
        assert np.array_equal(host(L.w[r][:n]).view(np.uint32), ref[r]["w"].view(np.uint32)), r
        assert np.array_equal(host(L.src[r][:n]), ref[r]["src"]), r
        # rows past the received ones are untouched
        assert np.isnan(L.recv_x[r][n:].float().cpu().numpy()).all(), r
        assert (host(L.idx[r][n:]) == -7).all() and (host(L.src[r][n:]) == -9).all(), r
    outs = finish_local(L, state, E, world, received)
    for r in range(world):
        ob, of = outs[r]
        assert np.array_equal(host(ob), ref[r]["out_bf16"]), r
        assert np.array_equal(host(of).view(np.uint32), ref[r]["out_f32"].view(np.uint32)), r
        assert B.ep_get_device_error(state[r][4]) == 0, r


@pytest.mark.parametrize("world", [2, 4, 8])
def test_peer_path_emulated_ranks_match_the_oracle(world):
    """Uneven batches (40 + 24 r tokens on rank r, H = 256, 256 experts, top-8)."""
    E = 256
    inputs = [rank_inputs(r, world, 40 + 24 * r, 256, E) for r in range(world)]
    capacity = sum(len(x) for x, _, _ in inputs)
    L, state = run_local(inputs, E, world, capacity)
    check_step(L, state, inputs, E, world)


def test_peer_path_prefill_rows_in_two_chunks():
    """Rows of 7168 channels (14 KB, one bulk copy per (token, rank)) and
    rows of 9000 channels (18 KB: two chunks per row), 4 ranks."""
    E, world = 256, 4
    for H, T in ((7168, 256), (9000, 96)):
        inputs = [rank_inputs(r, world, T + 16 * r, H, E, seed=9300) for r in range(world)]
        capacity = sum(len(x) for x, _, _ in inputs)
        L, state = run_local(inputs, E, world, capacity)
        check_step(L, state, inputs, E, world)


def test_peer_path_edge_cases():
    """A rank with no tokens, a rank that receives nothing (its experts are
    never picked), tokens with every entry -1, and 32 ranks."""
    E, world, H = 64, 4, 64
    inputs = []
    for r in range(world):
        T = 0 if r == 1 else 30
        x, idx, w = rank_inputs(r, world, max(T, 1), H, E, K=4, seed=9500)
        x, idx, w = x[:T], idx[:T], w[:T]
        idx = np.where(idx // (E // world) == 2, idx - E // world, idx)  # nothing for rank 2
        if T:
            idx[3] = -1
        inputs.append((np.ascontiguousarray(x), np.ascontiguousarray(idx), np.ascontiguousarray(w)))
    capacity = sum(len(x) for x, _, _ in inputs) + 5
    L, state = run_local(inputs, E, world, capacity)
    check_step(L, state, inputs, E, world)
    E, world = 256, 32
    inputs = [rank_inputs(r, world, 20 + r, 32, E, K=6, seed=9700) for r in range(world)]
    capacity = sum(len(x) for x, _, _ in inputs)
    L, state = run_local(inputs, E, world, capacity)
    check_step(L, state, inputs, E, world)


def test_peer_dispatch_beyond_capacity_is_flagged_and_stays_in_bounds():
    """Receive buffers smaller than what arrives: the rows that would land
    at or past `capacity` are skipped (the 64 guard rows behind each buffer
    stay untouched) and the sources flag EP_DEVERR_OVERFLOW."""
    E, world, H = 64, 2, 64
    inputs = [rank_inputs(r, world, 100, H, E, K=4, seed=9900) for r in range(world)]
    L, state = run_local(inputs, E, world, capacity=60, guard=64)
    flags = [B.ep_get_device_error(s[4], clear=False) for s in state]
    assert all(f & B.EP_DEVERR_OVERFLOW for f in flags), flags
    for r in range(world):
        assert np.isnan(L.recv_x[r][60:].float().cpu().numpy()).all(), r
        assert (host(L.idx[r][60:]) == -7).all() and (host(L.src[r][60:]) == -9).all(), r


def test_peer_path_at_the_bench_configuration():
    """Full size, as bench.py times the peer path: the prefill workload
    (4096 x 7168, top-8 of 256, 8 ranks), this process as rank 4 of 8 ranks
    that all hold its routing.  Every rank's block of received rows, entries
    and source tokens equals the oracle's per-rank dispatch rows for that
    rank, at rows 4 * count .. 5 * count of its buffer (rows around it
    untouched); with each rank's received rows as its partial rows, the
    combine equals the oracle's rank combine of the same rows, bit for bit
    on all outputs."""
    inp = W.make_inputs(2)
    cfg = inp["cfg"]
    T, H, E, R, K = cfg["T"], cfg["H"], cfg["E"], cfg["R"], cfg["K"]
    x_np, idx_np, w_np = inp["x"], inp["topk_idx"], inp["topk_weights"]
    L = oracle.tc_layout(idx_np, E, R)
    RL = oracle.rank_layout(L["is_token_in_rank"])
    D = oracle.rank_dispatch(x_np, idx_np, E, R, RL, topk_weights=w_np, want_src=True)
    want_out = oracle.rank_combine(D["recv"], RL, out_dtype=oracle.BF16)

    x, w = to_dev(x_np, bf16=True), to_dev(w_np)
    rt = B.Routing.topk(to_dev(idx_np), E, R)
    lay = B.Layout(rt)
    B.ep_get_layout(rt, lay)
    rl = B.RankLayout(rt)
    B.ep_get_rank_layout(rt, lay, rl)
    counts = host(lay.num_tokens_per_rank).astype(np.int64)
    me = R // 2
    capacity = int((me + 1) * counts.max())
    Lr = LocalRanks(R, capacity, H, K)
    for j in range(R):
        Lr.counts[j].copy_(lay.num_tokens_per_rank.repeat(R, 1))
    B.ep_dispatch_peers(x, rt, lay, rl, Lr.peers[me], topk_weights=w)
    torch.cuda.synchronize()
    offs = RL["rank_offsets"]
    for j in range(R):
        a, n = me * int(counts[j]), int(counts[j])
        blk = slice(int(offs[j]), int(offs[j + 1]))
        assert np.array_equal(host(Lr.recv_x[j][a:a + n]), D["recv"][blk]), j
        assert np.array_equal(host(Lr.idx[j][a:a + n]), D["recv_topk_idx"][blk]), j
        assert np.array_equal(host(Lr.w[j][a:a + n]).view(np.uint32), D["recv_topk_weights"][blk].view(np.uint32)), j
        assert np.array_equal(host(Lr.src[j][a:a + n]), D["recv_src"][blk]), j
        assert torch.isnan(Lr.recv_x[j][a - 1].float()).all() and (host(Lr.src[j][a + n:]) == -9).all(), j
        Lr.y[j][a:a + n].copy_(Lr.recv_x[j][a:a + n])
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    B.ep_combine_peers(rt, lay, rl, Lr.peers[me], out)
    assert np.array_equal(host(out), want_out)
    assert B.ep_get_device_error(lay) == 0


def test_peer_calls_check_their_tables():
    E, world = 64, 2
    x, idx, w = rank_inputs(0, world, 16, 64, E, K=4)
    routing = B.Routing.topk(to_dev(idx), E, world)
    layout = B.Layout(routing)
    rl = B.RankLayout(routing)
    L = LocalRanks(world, 32, 64, 4)
    bad_rank = B.Peers(2, 32, L.peers[0].tables["recv_x"], L.peers[0].tables["y"], L.peers[0].tables["rank_counts"])
    for peers in (bad_rank,):
        with pytest.raises(B.EPError):
            B.ep_dispatch_peers(to_dev(x, bf16=True), routing, layout, rl, peers)
        with pytest.raises(B.EPError):
            B.ep_combine_peers(routing, layout, rl, peers, torch.empty((16, 64), dtype=torch.bfloat16, device="cuda"))
        with pytest.raises(B.EPError):
            B.ep_peer_publish_counts(routing, layout, peers)
    # weights asked for without topk_weights
    with pytest.raises(B.EPError):
        B.ep_dispatch_peers(to_dev(x, bf16=True), routing, layout, rl, L.peers[0])


def test_peer_exchange_on_one_rank_nccl_matches_the_oracle():
    """PeerExpertParallel on a one-rank NCCL group (the barrier between the
    phases is NCCL's): its own block only, every token's experts local."""
    import torch.distributed as dist

    from combine_ep_get_10_b200.ep_exchange import PeerExpertParallel

    E, H = 256, 1024
    inputs = [rank_inputs(0, 1, 512, H, E)]
    x, idx, w = inputs[0]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        ep = PeerExpertParallel(E, H, idx.shape[1], capacity=len(x))
        recv = ep.dispatch(to_dev(x, bf16=True), to_dev(idx), to_dev(w))
        y = ep.experts(recv, expert_fn_for(0))
        ob = ep.combine(y, recv, torch.bfloat16)
        got = (host(recv.x).copy(), host(recv.src).copy(), recv.recv_counts, host(ob).copy())
        ep.close()
    finally:
        dist.destroy_process_group()
    ref = two_level_reference(inputs, E, 1)[0]
    assert got[2] == ref["counts"]
    assert np.array_equal(got[0], ref["x"]) and np.array_equal(got[1], ref["src"])
    assert np.array_equal(got[3], ref["out_bf16"])


def _ipc_worker(rank, world, port, q):
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
    ep = None
    try:
        from combine_ep_get_10_b200.ep_exchange import PeerExpertParallel
        from test_gpu_peers import E_IPC, H_IPC, expert_fn_for, ipc_inputs

        inputs = ipc_inputs(world)
        capacity = sum(len(x) for x, _, _ in inputs)
        x, idx, w = inputs[rank]
        ep = PeerExpertParallel(E_IPC, H_IPC, idx.shape[1], capacity)
        el = E_IPC // world
        results = []
        for step in range(2):  # the second step reuses every buffer
            recv = ep.dispatch(to_dev(x, bf16=True), to_dev(idx), to_dev(w))
            got_recv = (host(recv.x).copy(), host(recv.topk_idx).copy(), host(recv.src).copy(), recv.recv_counts)
            y = ep.experts(recv, expert_fn_for(rank * el))
            ob = ep.combine(y, recv, torch.bfloat16)
            of = ep.combine(y, recv, torch.float32)
            torch.cuda.synchronize()
            results.append((got_recv, host(ob).copy(), host(of).copy()))
        ep.close()
        ep = None
        q.put((rank, "ok", results))
        dist.barrier()
    except BaseException:
        import traceback

        q.put((rank, "error", traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


E_IPC, H_IPC = 256, 512


def ipc_inputs(world):
    return [rank_inputs(r, world, 48 + 20 * r, H_IPC, E_IPC, seed=9800) for r in range(world)]


@pytest.mark.parametrize("world", [2, 4])
def test_peer_exchange_processes_sharing_the_gpu(world):
    """W processes on the one GPU, each a rank of PeerExpertParallel: its
    block from ep_peer_alloc, the others' blocks mapped by ep_peer_open, the
    dispatch storing into and the combine reading from them.  Two steps; both
    give every rank the oracle's received rows and two-level results bit for
    bit.  No kernel waits on another process: the phases are separated by
    stream synchronisation and a gloo barrier."""
    import torch.multiprocessing as mp

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
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
    ref = two_level_reference(ipc_inputs(world), E_IPC, world)
    for r in range(world):
        for step in range(2):
            (rx, ridx, rsrc, counts), ob, of = res[r][step]
            assert counts == ref[r]["counts"], (r, step)
            assert np.array_equal(rx, ref[r]["x"]), (r, step)
            assert np.array_equal(ridx, ref[r]["idx"]), (r, step)
            assert np.array_equal(rsrc, ref[r]["src"]), (r, step)
            assert np.array_equal(ob, ref[r]["out_bf16"]), (r, step)
            assert np.array_equal(of.view(np.uint32), ref[r]["out_f32"].view(np.uint32)), (r, step)
