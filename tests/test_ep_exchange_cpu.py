"""Expert parallelism across processes: the exchange protocol of
combine_ep_get_10_b200/ep_exchange.py on 2 and 4 gloo ranks on CPU.

Each rank holds its own token batch (the prefill routing recipe at a small
size: 256 experts, top-8, sigmoid router with bias; 48 + 20 r tokens on rank
r, so the counts differ in both directions), and rank r owns experts
[r*E/W, (r+1)*E/W).  The compute steps run in the CPU oracle (the CUDA
kernels need a GPU); what is under test is the protocol: the counts exchange,
the receive-buffer sizes, the all-to-all-v of rows and their top-k entries,
the order rows arrive in, the reverse exchange and the rank-level combine on
the returned rows.  The experts are row-wise: expert e maps a row x to
bf16(x * (e + 1)).

Each rank's output is checked against two references computed in one
process from all ranks' inputs:
  * the same two-level sum with no exchange (per-rank partial rows from the
    oracle's per-rank dispatch and local combine, then the oracle's rank
    combine): equal bit for bit;
  * the oracle's flat per-expert combine (one fmaf chain over the token's k
    in ascending order): equal bit for bit on tokens whose experts all lie in
    one rank, and within the bound that the bf16 rounding of the per-rank
    partials and the fp32 additions over ranks allow on the others.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, H = 256, 128


def tokens_of(rank):
    """Uneven batches: rank r holds 48 + 20 r tokens."""
    return 48 + 20 * rank


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(rank, world):
    """Rank `rank`'s batch; every fourth token keeps its experts inside one
    rank (ids folded into rank t % W's range: duplicates may appear, which
    the layout allows), so that single-rank and multi-rank tokens both occur."""
    from combine_ep_get_10_b200 import workloads as W

    T = tokens_of(rank)
    inp = W.make_inputs(2, seed=7000 + rank, T=T)
    x = np.ascontiguousarray(inp["x"][:, :H])
    idx = inp["topk_idx"].copy()
    el = E // world
    for t in range(0, T, 4):
        idx[t] = idx[t] % el + (t % world) * el
    return x, idx, inp["topk_weights"]


def _bits_to_t(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _t_to_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _expert_rows(oracle, rows_bits, offsets, first_expert):
    """bf16(x * (e + 1)) for the rows of each local expert (rows grouped by
    local expert j at [offsets[j], offsets[j+1]), e = first_expert + j)."""
    out = np.empty_like(rows_bits)
    for j in range(len(offsets) - 1):
        a, b = int(offsets[j]), int(offsets[j + 1])
        if b > a:
            f = oracle.bf16_to_f32(rows_bits[a:b]) * np.float32(first_expert + j + 1)
            out[a:b] = oracle.f32_to_bf16(f.astype(np.float32))
    return out


class OracleRowOps:
    """The exchange's compute steps on CPU tensors, in the CPU oracle."""

    def __init__(self, oracle, rank, local_experts):
        self.o = oracle
        self.rank = rank
        self.local = local_experts

    def rank_rows(self, x, topk_idx, topk_weights, num_experts, world):
        from combine_ep_get_10_b200.ep_exchange import SendRows

        o = self.o
        idx, w = topk_idx.numpy(), topk_weights.numpy()
        L = o.tc_layout(idx, num_experts, world)
        RL = o.rank_layout(L["is_token_in_rank"])
        D = o.rank_dispatch(_t_to_bits(x), idx, num_experts, world, RL, topk_weights=w)
        counts = np.diff(RL["rank_offsets"]).tolist()
        return SendRows(_bits_to_t(D["recv"]), torch.from_numpy(D["recv_topk_idx"]),
                        torch.from_numpy(D["recv_topk_weights"]), counts, RL)

    def local_experts(self, x, topk_idx, topk_weights, local_experts, expert_fn):
        o = self.o
        idx = topk_idx.numpy()
        L = o.tc_layout(idx, local_experts, 1)
        rows = o.tc_dispatch(_t_to_bits(x), idx, local_experts, L)["recv"]
        y_rows = expert_fn(rows, L["expert_offsets"])
        y = o.tc_combine(y_rows, idx, local_experts, L, topk_weights.numpy(), out_dtype=o.BF16)
        return _bits_to_t(y)

    def combine_ranks(self, back, handle, out_dtype):
        o = self.o
        code = o.BF16 if out_dtype == torch.bfloat16 else o.FP32
        out = o.rank_combine(_t_to_bits(back), handle, out_dtype=code)
        return _bits_to_t(out) if code == o.BF16 else torch.from_numpy(out)


def _worker(rank, world, port, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        _run(rank, world, q)
    except BaseException:
        import traceback

        q.put((rank, "error", traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def _run(rank, world, q):
    import torch.distributed as dist

    import oracle
    from combine_ep_get_10_b200.ep_exchange import ExpertParallel

    oracle.build()
    ep = ExpertParallel(E, ops=OracleRowOps(oracle, rank, E // world))
    x, idx, w = _inputs(rank, world)
    recv = ep.dispatch(_bits_to_t(x), torch.from_numpy(idx), torch.from_numpy(w))
    first = rank * (E // world)
    y = ep.experts(recv, lambda rows, offs: _expert_rows(oracle, rows, offs, first))
    out_bf16 = ep.combine(y, recv, torch.bfloat16)
    out_f32 = ep.combine(y, recv, torch.float32)
    q.put((rank, recv.recv_counts, recv.send.counts, _t_to_bits(recv.x).copy(), recv.topk_idx.numpy().copy(),
           _t_to_bits(out_bf16).copy(), out_f32.numpy().copy()))
    dist.barrier()


def _reference(oracle, world):
    """Per rank (source), in one process: the rows it sends, the partial rows
    its destinations return (no exchange), the two-level result, and the flat
    per-expert combine."""
    el = E // world
    ref = {}
    for i in range(world):
        x, idx, w = _inputs(i, world)
        L = oracle.tc_layout(idx, E, world)
        RL = oracle.rank_layout(L["is_token_in_rank"])
        D = oracle.rank_dispatch(x, idx, E, world, RL, topk_weights=w)
        back = np.empty_like(D["recv"])
        offs = RL["rank_offsets"]
        for r in range(world):
            a, b = int(offs[r]), int(offs[r + 1])
            if b == a:
                continue
            ridx = D["recv_topk_idx"][a:b]
            LL = oracle.tc_layout(ridx, el, 1)
            rows = oracle.tc_dispatch(D["recv"][a:b], ridx, el, LL)["recv"]
            yr = _expert_rows(oracle, rows, LL["expert_offsets"], r * el)
            back[a:b] = oracle.tc_combine(yr, ridx, el, LL, D["recv_topk_weights"][a:b], out_dtype=oracle.BF16)
        two_bf16 = oracle.rank_combine(back, RL, out_dtype=oracle.BF16)
        two_f32 = oracle.rank_combine(back, RL, out_dtype=oracle.FP32)
        # flat: every (t, k) pair's expert output as its own dispatched row
        LF = oracle.tc_layout(idx, E, world)
        yf = oracle.tc_dispatch(x, idx, E, LF)["recv"]
        for e in range(E):
            a, b = int(LF["expert_offsets"][e]), int(LF["expert_offsets"][e + 1])
            if b > a:
                yf[a:b] = oracle.f32_to_bf16((oracle.bf16_to_f32(yf[a:b]) * np.float32(e + 1)).astype(np.float32))
        flat = oracle.tc_combine(yf, idx, E, LF, w, out_dtype=oracle.FP32)
        flat_bf16 = oracle.tc_combine(yf, idx, E, LF, w, out_dtype=oracle.BF16)
        # |w * y| summed per token, for the tolerance of multi-rank tokens
        T = tokens_of(i)
        mag = np.zeros((T, H), np.float64)
        for t in range(T):
            for k in range(idx.shape[1]):
                e = int(idx[t, k])
                if e >= 0:
                    row = int(LF["expert_offsets"][e] + LF["slot"][t, k])
                    mag[t] += abs(float(w[t, k])) * np.abs(oracle.bf16_to_f32(yf[row]).astype(np.float64))
        ranks_of = [{int(e) // el for e in idx[t] if e >= 0} for t in range(T)]
        ref[i] = dict(send=D["recv"], send_idx=D["recv_topk_idx"], counts=np.diff(offs).tolist(), two_bf16=two_bf16,
                      two_f32=two_f32, flat=flat, flat_bf16=flat_bf16, mag=mag, ranks_of=ranks_of)
    return ref


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_matches_the_single_process_oracle(world, oracle_mod):
    oracle = oracle_mod
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            item = q.get(timeout=300)
            assert item[1] != "error", "rank %d failed:\n%s" % (item[0], item[2])
            res[item[0]] = item[1:]
    finally:
        for p in procs:
            p.join(timeout=120 if len(res) == world else 5)
            if p.exitcode is None:
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    ref = _reference(oracle, world)
    for r in range(world):
        recv_counts, send_counts, rx, ridx, out_bf16, out_f32 = res[r]
        # the counts exchange: what rank r receives from i is what i sends to r
        assert send_counts == ref[r]["counts"]
        assert recv_counts == [ref[i]["counts"][r] for i in range(world)]
        # received rows: source 0's block for rank r first, each in token order
        want = np.concatenate([ref[i]["send"][sum(ref[i]["counts"][:r]):sum(ref[i]["counts"][:r + 1])]
                               for i in range(world)])
        want_idx = np.concatenate([ref[i]["send_idx"][sum(ref[i]["counts"][:r]):sum(ref[i]["counts"][:r + 1])]
                                   for i in range(world)])
        assert np.array_equal(rx, want)
        assert np.array_equal(ridx, want_idx)
        assert ((ridx == -1) | ((ridx >= 0) & (ridx < E // world))).all()
        # the two-level result, bit for bit
        assert np.array_equal(out_bf16, ref[r]["two_bf16"])
        assert np.array_equal(out_f32.view(np.uint32), ref[r]["two_f32"].view(np.uint32))
        # against the flat per-expert combine
        one = np.array([len(s) <= 1 for s in ref[r]["ranks_of"]])
        assert one.any() and (~one).any()
        assert np.array_equal(out_bf16[one], ref[r]["flat_bf16"][one])
        got = out_f32.astype(np.float64)
        flat = ref[r]["flat"].astype(np.float64)
        # each partial rounds to bf16 once (unit roundoff 2^-8: 8 significant
        # bits), the additions over ranks and both fmaf chains add fp32
        # roundings (2^-24 each)
        bound = (2.0 ** -8 + (8 + world) * 2.0 ** -24) * ref[r]["mag"] + 1e-30
        assert (np.abs(got - flat) <= bound).all()
