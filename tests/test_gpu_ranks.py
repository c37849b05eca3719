"""GPU parity of the per-rank (deduplicated) path -- DeepEP-Ascend README,
"API Overview": normal-mode dispatch to expert ranks with the received
tokens' top-k information, and the combine that reduces what the ranks send
back -- against the CPU oracle: rank layout, received rows, top-k entries
and source tokens bit for bit; the rank combine within the combine
tolerance (and, the order being the same, expected bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import assert_combine_close, exact_fraction, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _layouts(idx, E, R):
    routing = B.Routing.topk(to_dev(np.ascontiguousarray(idx, np.int64)), E, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    rl = B.RankLayout(routing)
    B.ep_get_rank_layout(routing, lay, rl)
    return routing, lay, rl


def _check_rank_layout(rl, ref):
    assert np.array_equal(host(rl.rank_offsets), ref["rank_offsets"]), "rank_offsets"
    assert np.array_equal(host(rl.rank_row), ref["rank_row"]), "rank_row"


CASES = [
    # T, E, R, K, p_neg, dup, p_bad, seed
    (0, 8, 2, 2, 0.0, False, 0.0, 1),
    (1, 4, 1, 4, 0.0, False, 0.0, 2),
    (45, 12, 3, 36, 0.2, True, 0.02, 3),  # K > 32, duplicates, bad ids
    (3000, 64, 32, 6, 0.3, False, 0.0, 4),  # R = 32, three 1024-token tiles
    (1500, 16, 16, 1, 0.5, False, 0.0, 5),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_E%d_R%d_K%d" % c[:4])
def test_rank_path_small(case):
    T, E, R, K, p_neg, dup, p_bad, seed = case
    r = _rng(seed)
    idx = W.random_topk(r, T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad)
    H = 136
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    w = r.random((T, K)).astype(np.float32)
    ref_l = oracle.tc_layout(idx, E, R)
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    routing, lay, rl = _layouts(idx, E, R)
    _check_rank_layout(rl, ref_rl)
    rows = int(ref_rl["rank_offsets"][-1])
    if T == 0:
        assert rows == 0
        recv = torch.zeros((1, H), dtype=torch.bfloat16, device="cuda")
        B.ep_dispatch_ranks(torch.zeros((1, H), dtype=torch.bfloat16, device="cuda"), routing, lay, rl, recv,
                            num_recv_rows=0)
        assert B.ep_get_device_error(lay) == 0
        return
    ref = oracle.rank_dispatch(x, idx, E, R, ref_rl, w, want_src=True)
    recv = torch.zeros((rows, H), dtype=torch.bfloat16, device="cuda")
    ridx = torch.full((rows, K), -7, dtype=torch.int64, device="cuda")
    rw = torch.full((rows, K), -7.0, dtype=torch.float32, device="cuda")
    src = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    B.ep_dispatch_ranks(to_dev(x, bf16=True), routing, lay, rl, recv, topk_weights=to_dev(w), recv_topk_idx=ridx,
                        recv_topk_weights=rw, recv_src=src)
    flags = B.ep_get_device_error(lay)
    assert bool(flags & B.EP_DEVERR_BAD_INDEX) == (p_bad > 0)
    assert not flags & B.EP_DEVERR_OVERFLOW
    assert np.array_equal(host(recv), ref["recv"])
    assert np.array_equal(host(ridx), ref["recv_topk_idx"])
    assert np.array_equal(host(rw).view(np.uint32), ref["recv_topk_weights"].view(np.uint32))
    assert np.array_equal(host(src), ref["recv_src"])
    y = W.to_bf16_bits(r.standard_normal((rows, H)).astype(np.float32))
    yd = to_dev(y, bf16=True)
    for dt, tdt in ((W.FP32, torch.float32), (W.BF16, torch.bfloat16)):
        out = torch.empty((T, H), dtype=tdt, device="cuda")
        B.ep_combine_ranks(yd, routing, lay, rl, out)
        want = oracle.rank_combine(y, ref_rl, out_dtype=dt)
        got = host(out)
        assert_combine_close(got, want, bf16=(dt == W.BF16), what="rank combine")
        assert exact_fraction(got, want) == 1.0  # same order, same roundings
    assert B.ep_get_device_error(lay) == 0


@pytest.mark.parametrize("wl", [1, 2, 5])
def test_rank_path_workloads(wl):
    """Workloads 1, 2 (4096 x 7168, 256 experts in 8 ranks, top-8) and 5
    (16384 tokens, skewed, 10% -1): the full rank layout, all received rows'
    top-k entries and sources, and sampled rows / tokens of the payloads."""
    inp = W.make_inputs(wl)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    T, H, E, R, K = c["T"], c["H"], c["E"], c["R"], c["K"]
    ref_l = oracle.tc_layout(idx, E, R)
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    routing, lay, rl = _layouts(idx, E, R)
    _check_rank_layout(rl, ref_rl)
    rows = int(ref_rl["rank_offsets"][-1])
    assert rows < int(((idx >= 0)).sum())  # deduplication saves rows
    recv = torch.empty((rows, H), dtype=torch.bfloat16, device="cuda")
    ridx = torch.empty((rows, K), dtype=torch.int64, device="cuda")
    rw = torch.empty((rows, K), dtype=torch.float32, device="cuda")
    src = torch.empty((rows,), dtype=torch.int32, device="cuda")
    B.ep_dispatch_ranks(to_dev(x, bf16=True), routing, lay, rl, recv, topk_weights=to_dev(w), recv_topk_idx=ridx,
                        recv_topk_weights=rw, recv_src=src)
    assert B.ep_get_device_error(lay) == 0
    # top-k entries and sources of every row, from the oracle on the metadata
    # (an 8-channel payload keeps the oracle call cheap)
    ref_meta = oracle.rank_dispatch(x[:, :8], idx, E, R, ref_rl, w, want_src=True)
    g_src = host(src)
    assert np.array_equal(g_src, ref_meta["recv_src"])
    assert np.array_equal(host(ridx), ref_meta["recv_topk_idx"])
    assert np.array_equal(host(rw).view(np.uint32), ref_meta["recv_topk_weights"].view(np.uint32))
    # payload rows: a sample, each against its source row
    sample = np.sort(_rng(7).choice(rows, size=min(rows, 512), replace=False))
    g_rows = host(recv[torch.from_numpy(sample).cuda()])
    assert np.array_equal(g_rows, x[g_src[sample]])
    # combine over the received rows: sampled tokens, against the oracle on
    # just the rows those tokens read (rank_row renumbered into that subset)
    tokens = np.sort(_rng(8).choice(T, size=min(T, 96), replace=False))
    rr = ref_rl["rank_row"][tokens]
    used = np.unique(rr[rr >= 0])
    sub = dict(rank_row=np.where(rr >= 0, np.searchsorted(used, rr), -1).astype(np.int32))
    y_sub = host(recv[torch.from_numpy(used).cuda()])
    for dt, tdt in ((W.FP32, torch.float32), (W.BF16, torch.bfloat16)):
        out = torch.empty((T, H), dtype=tdt, device="cuda")
        B.ep_combine_ranks(recv, routing, lay, rl, out)
        want = oracle.rank_combine(y_sub, sub, out_dtype=dt)
        got = host(out[torch.from_numpy(tokens).cuda()])
        assert_combine_close(got, want, bf16=(dt == W.BF16), what="rank combine wl%d" % wl)
        assert exact_fraction(got, want) == 1.0
    assert B.ep_get_device_error(lay) == 0


def test_rank_dispatch_overflow_is_flagged():
    r = _rng(11)
    T, E, R, K, H = 200, 16, 4, 4, 64
    idx = W.random_topk(r, T, E, K)
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    ref_l = oracle.tc_layout(idx, E, R)
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    rows = int(ref_rl["rank_offsets"][-1])
    cut = rows // 2
    routing, lay, rl = _layouts(idx, E, R)
    recv = torch.zeros((rows, H), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch_ranks(to_dev(x, bf16=True), routing, lay, rl, recv, num_recv_rows=cut)
    assert B.ep_get_device_error(lay) & B.EP_DEVERR_OVERFLOW
    ref = oracle.rank_dispatch(x, idx, E, R, ref_rl)
    g = host(recv)
    assert np.array_equal(g[:cut], ref["recv"][:cut]) and (g[cut:] == 0).all()
    out = torch.empty((T, H), dtype=torch.float32, device="cuda")
    B.ep_combine_ranks(recv, routing, lay, rl, out, num_y_rows=cut)
    assert B.ep_get_device_error(lay) & B.EP_DEVERR_OVERFLOW


@pytest.mark.parametrize("wl", [2, 5])
def test_layout_dispatch_ranks_one_call_equals_the_three_calls(wl):
    """ep_layout_dispatch_ranks: the layout, the rank layout and the per-rank
    dispatch in one call (the rows are loaded while the rank layout runs)
    writes the same layouts, rows, entries and sources as the three calls,
    bit for bit, on the full prefill and skewed workloads."""
    inp = W.make_inputs(wl)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    T, H, E, R, K = c["T"], c["H"], c["E"], c["R"], c["K"]
    xd, wd = to_dev(x, bf16=True), to_dev(w)
    routing, lay, rl = _layouts(idx, E, R)
    rows = int(host(rl.rank_offsets)[-1])
    outs = []
    for one_call in (False, True):
        recv = torch.full((rows, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        ridx = torch.full((rows, K), -7, dtype=torch.int64, device="cuda")
        rw = torch.full((rows, K), float("nan"), dtype=torch.float32, device="cuda")
        src = torch.full((rows,), -9, dtype=torch.int32, device="cuda")
        if one_call:
            lay = B.Layout(routing, report_num_valid=True)
            rl = B.RankLayout(routing)
            B.ep_layout_dispatch_ranks(xd, routing, lay, rl, recv, topk_weights=wd, recv_topk_idx=ridx,
                                       recv_topk_weights=rw, recv_src=src)
            assert lay.num_valid == int((idx >= 0).sum())  # num_valid_host, as ep_get_layout reports it
        else:
            B.ep_dispatch_ranks(xd, routing, lay, rl, recv, topk_weights=wd, recv_topk_idx=ridx, recv_topk_weights=rw,
                                recv_src=src)
        assert B.ep_get_device_error(lay) == 0
        outs.append((host(rl.rank_offsets), host(rl.rank_row), host(lay.slot), host(recv), host(ridx),
                     host(rw).view(np.uint32), host(src)))
    for a, b in zip(*outs):
        assert np.array_equal(a, b)
    ref_rl = oracle.rank_layout(oracle.tc_layout(idx, E, R)["is_token_in_rank"])
    _check_rank_layout(rl, ref_rl)
    assert np.array_equal(outs[1][3], x[outs[1][6]])  # every received row is its source token's row
