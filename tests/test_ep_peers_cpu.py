"""The peer-memory exchange protocol (combine_ep_get_10_b200/ep_exchange.py
PeerExpertParallel) on 2 and 4 gloo ranks on CPU.

The CUDA kernels need a GPU, so the memory and compute steps come from a
stand-in (``FilePeerOps``): each rank's block is a file mapped into every
process (its path plays the IPC handle), the layouts come from the CPU
oracle, and the counts publish, the dispatch placement and the combine
gather are restated here in plain Python from the rule the exchange defines
(rank j's rows: source 0's first, each source's rows in token order; source
i's block at sum over i' < i of counts[i', j]).  What is under test is the
protocol of PeerExpertParallel itself: the block layout every rank must
agree on, the handle exchange and mapping, the phase order with its
barriers, the counts read, the partial rows in the rank's own block, and
close / free.  Each rank's received rows and results are compared bit for
bit with the single-process oracle composition of test_ep_exchange_cpu."""
import mmap
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


_NP = {torch.bfloat16: np.int16, torch.int32: np.int32, torch.int64: np.int64, torch.float32: np.float32}


class FilePeerOps:
    """Blocks as mapped files; addresses are (block number << 40) + offset."""

    SHIFT = 40

    def __init__(self, oracle, directory):
        self.o = oracle
        self.dir = directory
        self.maps = {}  # block number -> (mmap, path, owned)
        self.next = 1

    def _map(self, path, owned):
        fd = os.open(path, os.O_RDWR)
        try:
            mm = mmap.mmap(fd, os.fstat(fd).st_size)
        finally:
            os.close(fd)
        n = self.next
        self.next += 1
        self.maps[n] = (mm, path, owned)
        return n << self.SHIFT

    def alloc(self, nbytes):
        fd, path = tempfile.mkstemp(dir=self.dir)
        os.ftruncate(fd, nbytes)
        os.close(fd)
        return self._map(path, True), path.encode()

    def open(self, handle):
        return self._map(handle.decode(), False)

    @staticmethod
    def _unmap(mm):
        try:
            mm.close()
        except BufferError:  # tensors over it still alive: unmapped when they go
            pass

    def close(self, base):
        self._unmap(self.maps.pop(base >> self.SHIFT)[0])

    def free(self, base):
        mm, path, _ = self.maps.pop(base >> self.SHIFT)
        self._unmap(mm)
        os.unlink(path)

    def view(self, addr, shape, dtype):
        mm = self.maps[addr >> self.SHIFT][0]
        off = addr & ((1 << self.SHIFT) - 1)
        a = np.frombuffer(mm, dtype=_NP[dtype], count=int(np.prod(shape)), offset=off).reshape(shape)
        t = torch.from_numpy(a)
        return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t

    def peers(self, rank, capacity, tables):
        return dict(rank=rank, capacity=capacity, tables=tables)

    def sync(self):
        pass

    # compute steps
    def layout(self, topk_idx, num_experts, world):
        idx = topk_idx.numpy()
        L = self.o.tc_layout(idx, num_experts, world)
        RL = self.o.rank_layout(L["is_token_in_rank"])
        return dict(idx=idx, E=num_experts, W=world, L=L, RL=RL)

    def _bases(self, h, p):
        """Row of this rank's block start minus its rank_offsets, per rank."""
        W, me = h["W"], p["rank"]
        counts = self.view(p["tables"]["rank_counts"][me], (W, W), torch.int32).numpy()
        return [int(counts[:me, j].sum()) - int(h["RL"]["rank_offsets"][j]) for j in range(W)]

    def publish(self, h, p):
        W, me = h["W"], p["rank"]
        for j in range(W):
            m = self.view(p["tables"]["rank_counts"][j], (W, W), torch.int32)
            m[me] = torch.from_numpy(np.asarray(h["L"]["num_tokens_per_rank"], dtype=np.int32))

    def dispatch(self, x, topk_weights, h, p):
        W, E, me, C = h["W"], h["E"], p["rank"], p["capacity"]
        idx, w, rank_row = h["idx"], topk_weights.numpy(), h["RL"]["rank_row"]
        K, H, el = idx.shape[1], x.shape[1], E // W
        base = self._bases(h, p)
        tabs = p["tables"]
        for t in range(idx.shape[0]):
            for j in range(W):
                if rank_row[t, j] < 0:
                    continue
                row = base[j] + int(rank_row[t, j])
                assert 0 <= row < C
                self.view(tabs["recv_x"][j], (C, H), torch.bfloat16)[row] = x[t]
                local = [(e - j * el) if 0 <= e < E and e // el == j else -1 for e in idx[t].tolist()]
                self.view(tabs["recv_topk_idx"][j], (C, K), torch.int64)[row] = torch.tensor(local)
                self.view(tabs["recv_topk_weights"][j], (C, K), torch.float32)[row] = torch.from_numpy(
                    np.where(np.array(local) >= 0, w[t], np.float32(0)).astype(np.float32))
                self.view(tabs["recv_src"][j], (C,), torch.int32)[row] = t

    def local_experts(self, x, topk_idx, topk_weights, local_experts, expert_fn, out):
        from test_ep_exchange_cpu import OracleRowOps

        out.copy_(OracleRowOps(self.o, 0, local_experts).local_experts(x, topk_idx, topk_weights, local_experts,
                                                                      expert_fn))
        return out

    def combine(self, h, p, hidden, out_dtype):
        from test_ep_exchange_cpu import _bits_to_t, _t_to_bits

        o, W, C = self.o, h["W"], p["capacity"]
        base = self._bases(h, p)
        rank_row = h["RL"]["rank_row"]
        back = np.zeros((int(h["RL"]["rank_offsets"][W]), hidden), np.uint16)
        for t in range(rank_row.shape[0]):
            for j in range(W):
                if rank_row[t, j] >= 0:
                    yj = self.view(p["tables"]["y"][j], (C, hidden), torch.bfloat16)
                    back[rank_row[t, j]] = _t_to_bits(yj[base[j] + int(rank_row[t, j])])
        code = o.BF16 if out_dtype == torch.bfloat16 else o.FP32
        out = o.rank_combine(back, h["RL"], out_dtype=code)
        return _bits_to_t(out) if code == o.BF16 else torch.from_numpy(out)


def _worker(rank, world, port, directory, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle
        from combine_ep_get_10_b200.ep_exchange import PeerExpertParallel
        from test_ep_exchange_cpu import E, H, _bits_to_t, _expert_rows, _inputs, _t_to_bits, tokens_of

        oracle.build()
        capacity = sum(tokens_of(i) for i in range(world))
        x, idx, w = _inputs(rank, world)
        ep = PeerExpertParallel(E, H, idx.shape[1], capacity, ops=FilePeerOps(oracle, directory))
        first = rank * (E // world)
        recv = ep.dispatch(_bits_to_t(x), torch.from_numpy(idx), torch.from_numpy(w))
        got = (_t_to_bits(recv.x).copy(), recv.topk_idx.numpy().copy(), recv.src.numpy().copy(), recv.recv_counts)
        y = ep.experts(recv, lambda rows, offs: _expert_rows(oracle, rows, offs, first))
        out_bf16 = ep.combine(y, recv, torch.bfloat16)
        out_f32 = ep.combine(y, recv, torch.float32)
        ep.close()
        q.put((rank, "ok", got, _t_to_bits(out_bf16).copy(), out_f32.numpy().copy()))
        dist.barrier()
    except BaseException:
        import traceback

        q.put((rank, "error", traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_peer_exchange_protocol_matches_the_single_process_oracle(world, oracle_mod, tmp_path):
    from test_ep_exchange_cpu import _reference

    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path), q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            item = q.get(timeout=300)
            assert item[1] == "ok", "rank %d failed:\n%s" % (item[0], item[2])
            res[item[0]] = item[2:]
    finally:
        for p in procs:
            p.join(timeout=120 if len(res) == world else 5)
            if p.exitcode is None:
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    assert os.listdir(tmp_path) == []  # every block freed
    ref = _reference(oracle_mod, world)
    for r in range(world):
        (rx, ridx, rsrc, counts), out_bf16, out_f32 = res[r]
        assert counts == [ref[i]["counts"][r] for i in range(world)]
        want = np.concatenate([ref[i]["send"][sum(ref[i]["counts"][:r]):sum(ref[i]["counts"][:r + 1])]
                               for i in range(world)])
        want_idx = np.concatenate([ref[i]["send_idx"][sum(ref[i]["counts"][:r]):sum(ref[i]["counts"][:r + 1])]
                                   for i in range(world)])
        assert np.array_equal(rx, want)
        assert np.array_equal(ridx, want_idx)
        assert ((rsrc >= 0) & (rsrc < 48 + 20 * (world - 1))).all()
        assert np.array_equal(out_bf16, ref[r]["two_bf16"])
        assert np.array_equal(out_f32.view(np.uint32), ref[r]["two_f32"].view(np.uint32))


def _leaving_worker(rank, world, port, directory, kind, q):
    """Rank 1 leaves between steps (after the exchange is set up, before the
    step's first collective); rank 0 then runs a step."""
    import sys
    import time
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=5))
    import oracle
    from combine_ep_get_10_b200.ep_exchange import ExpertParallel, PeerExpertParallel
    from test_ep_exchange_cpu import E, H, OracleRowOps, _bits_to_t, _inputs, tokens_of

    oracle.build()
    x, idx, w = _inputs(rank, world)
    if kind == "peer":
        ep = PeerExpertParallel(E, H, idx.shape[1], sum(tokens_of(i) for i in range(world)),
                                ops=FilePeerOps(oracle, directory))
    else:
        ep = ExpertParallel(E, ops=OracleRowOps(oracle, rank, E // world))
        dist.barrier()
    if rank == 1:
        q.put((rank, "left", 0.0))
        q.close()
        q.join_thread()
        os._exit(0)  # no destroy_process_group: the rank is simply gone
    t0 = time.time()
    try:
        ep.dispatch(_bits_to_t(x), torch.from_numpy(idx), torch.from_numpy(w))
        q.put((rank, "no error", time.time() - t0))
    except Exception as e:  # the collective fails: the peer is gone or the timeout ran out
        q.put((rank, "raised " + type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()
    os._exit(0)


@pytest.mark.parametrize("kind", ["peer", "alltoall"])
def test_a_rank_that_leaves_fails_the_next_step_instead_of_hanging(kind, tmp_path):
    """Failure detection on the host: with a short process-group timeout,
    the remaining rank's next collective of the step (the barrier after the
    counts publish, or the counts all-to-all) raises instead of waiting."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, str(tmp_path), kind, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(2):
            rank, what, secs = q.get(timeout=120)
            res[rank] = (what, secs)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.exitcode is None:
                p.kill()
    assert res[1][0] == "left"
    assert res[0][0].startswith("raised"), res[0]
    assert res[0][1] < 60.0, res[0]
