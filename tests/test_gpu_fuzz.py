"""Seeded random shapes through every entry point, against the CPU oracle:
token counts, expert / rank / top-k counts, hidden sizes (ragged against the
kernels' tiles), -1 and duplicate ids, padded overflow, every quantised
format, the per-rank path, the per-rank path over peer memory and expert
choice.  Deterministic (fixed seeds)."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import assert_combine_close, host, to_dev

pytestmark = pytest.mark.gpu

QUANT = [W.FP8_E4M3, W.INT8_PER_TOKEN, W.FP8_E4M3_PER_TOKEN, W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def _shape(seed):
    r = np.random.Generator(np.random.PCG64(1000 + seed))
    R = int(r.choice([1, 2, 3, 4, 8, 16, 32]))
    E = R * int(r.integers(1, 12))
    K = int(r.integers(1, min(E, 12) + 1)) if r.random() < 0.9 else int(r.integers(33, 48))
    T = int(r.choice([0, 1, 7, 63, 64, 65, 129, 500, 1500, 3000]))
    H = 128 * int(r.integers(1, 9)) + int(r.choice([0, 0, 32, 64, 96]))
    return r, T, E, R, K, H


@pytest.mark.parametrize("seed", range(24))
def test_token_choice_random_shapes(seed):
    r, T, E, R, K, H = _shape(seed)
    dup = bool(r.random() < 0.3) or K > E  # more slots than experts need repeats
    idx = W.random_topk(r, T, E, K, p_neg=float(r.choice([0.0, 0.1, 0.5])), allow_dup=dup, p_bad=0.0)
    x = W.to_bf16_bits((r.standard_normal((T, H)) * 10.0 ** r.uniform(-2, 2)).astype(np.float32))
    w = r.standard_normal((T, K)).astype(np.float32)
    ref_l = oracle.tc_layout(idx, E, R)
    routing = B.Routing.topk(to_dev(np.ascontiguousarray(idx, np.int64)), E, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    assert np.array_equal(host(lay.slot), ref_l["slot"])
    assert np.array_equal(host(lay.expert_offsets), ref_l["expert_offsets"])
    assert np.array_equal(host(lay.num_tokens_per_rank), ref_l["num_tokens_per_rank"])
    if T == 0:
        return
    xd, wd = to_dev(x, bf16=True), to_dev(w)
    n = int(ref_l["expert_offsets"][-1])
    # bf16 compact dispatch + fp32 / bf16 combine
    recv = torch.zeros((max(n, 1), H), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch(xd, routing, lay, recv, num_recv_rows=n)
    ref_d = oracle.tc_dispatch(x, idx, E, ref_l)
    assert np.array_equal(host(recv)[:n], ref_d["recv"])
    for dt, tdt in ((W.FP32, torch.float32), (W.BF16, torch.bfloat16)):
        out = torch.full((T, H), float("nan"), dtype=tdt, device="cuda")
        B.ep_combine(recv, routing, lay, wd, out, num_y_rows=n)
        ref_c = oracle.tc_combine(ref_d["recv"], idx, E, ref_l, w, out_dtype=dt)
        assert_combine_close(host(out), ref_c, dt == W.BF16, "combine seed %d" % seed)
    # one quantised format, padded with a small max_tokens (overflow likely)
    dt = QUANT[seed % len(QUANT)]
    group = 128 if dt == W.FP8_E4M3 else (32 if dt in (W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1) else 8)
    if H % group == 0:
        mt = int(r.integers(1, 12))
        rows = E * mt
        codes = torch.full((rows, oracle.row_code_bytes(dt, H)), 0xAB, dtype=torch.uint8, device="cuda")
        sc = torch.full((rows, oracle.row_scale_bytes(dt, H)), 0x5A, dtype=torch.uint8, device="cuda")
        B.ep_dispatch(xd, routing, lay, codes, mode=B.EP_LAYOUT_PADDED, max_tokens_per_expert=mt, recv_scales=sc,
                      out_dtype=dt)
        ref_q = oracle.tc_dispatch(x, idx, E, ref_l, mode=W.PADDED, max_tokens=mt, out_dtype=dt)
        valid = np.zeros(rows, bool)
        for e in range(E):
            valid[e * mt:e * mt + min(int(ref_l["num_tokens_per_expert"][e]), mt)] = True
        rc = np.ascontiguousarray(ref_q["recv"]).view(np.uint8).reshape(rows, -1)
        rs = np.ascontiguousarray(ref_q["recv_scales"]).view(np.uint8).reshape(rows, -1)
        assert np.array_equal(host(codes)[valid], rc[valid]) and np.array_equal(host(sc)[valid], rs[valid])
    # per rank
    rl = B.RankLayout(routing)
    B.ep_get_rank_layout(routing, lay, rl)
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    assert np.array_equal(host(rl.rank_row), ref_rl["rank_row"])
    nr = int(ref_rl["rank_offsets"][-1])
    if nr:
        rrecv = torch.empty((nr, H), dtype=torch.bfloat16, device="cuda")
        B.ep_dispatch_ranks(xd, routing, lay, rl, rrecv)
        assert np.array_equal(host(rrecv), oracle.rank_dispatch(x, idx, E, R, ref_rl)["recv"])
        rout = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
        B.ep_combine_ranks(rrecv, routing, lay, rl, rout)
        assert_combine_close(host(rout), oracle.rank_combine(host(rrecv), ref_rl, out_dtype=W.FP32), False, "ranks")
    assert B.ep_get_device_error(lay) & ~B.EP_DEVERR_OVERFLOW == 0


@pytest.mark.parametrize("seed", range(12))
def test_expert_choice_random_shapes(seed):
    r = np.random.Generator(np.random.PCG64(2000 + seed))
    R = int(r.choice([1, 2, 4, 8]))
    E = R * int(r.integers(1, 10))
    C = int(r.integers(1, 200))
    T = int(r.choice([1, 5, 100, 2000, 9000]))
    H = 8 * int(r.integers(1, 80))
    ti = W.random_token_indices(r, T, E, C, p_neg=float(r.choice([0.0, 0.2])))
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    ew = r.standard_normal((E, C)).astype(np.float32)
    ref_l = oracle.ec_layout(ti, T, R)
    routing = B.Routing.expert_choice(to_dev(ti), T, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    n = int(ref_l["token_offsets"][-1])
    assert np.array_equal(host(lay.token_offsets), ref_l["token_offsets"])
    assert np.array_equal(host(lay.token_slots)[:n], ref_l["token_slots"][:n])
    recv = torch.zeros((E * C, H), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch_expert_choice(to_dev(x, bf16=True), routing, lay, recv)
    ref_d = oracle.ec_dispatch(x, ti)
    assert np.array_equal(host(recv), ref_d)
    out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.ep_combine_expert_choice(recv, routing, lay, to_dev(ew), out)
    assert_combine_close(host(out), oracle.ec_combine(ref_d, ref_l, ew, T, out_dtype=W.BF16), True, "ec")
    assert B.ep_get_device_error(lay) == 0


@pytest.mark.parametrize("seed", range(12))
def test_peer_path_random_shapes(seed):
    """The per-rank path over peer memory with its ranks emulated on the one
    GPU (tests/test_gpu_peers.py): random rank counts (1..32), uneven token
    batches per rank (some empty), -1 and duplicate ids, hidden sizes from 8
    to 8800 (rows of two bulk chunks past 16 KB), capacity with or without
    slack; received rows, entries, source tokens and both output precisions
    bit for bit against the oracle's two-level composition."""
    from test_gpu_peers import check_step, run_local

    r = np.random.Generator(np.random.PCG64(5000 + seed))
    world = int(r.choice([1, 2, 3, 4, 8, 16, 32]))
    E = world * int(r.integers(1, 9))
    K = int(r.integers(1, min(E, 10) + 1))
    H = 8 * int(r.integers(1030, 1126) if seed % 4 == 3 else r.integers(1, 1101))  # every 4th: two chunks
    inputs = []
    for _ in range(world):
        T = int(r.choice([0, 1, 5, 33, 100, 257]))
        idx = W.random_topk(r, T, E, K, p_neg=float(r.choice([0.0, 0.2])), allow_dup=bool(r.random() < 0.3),
                            p_bad=0.0)
        x = W.to_bf16_bits((r.standard_normal((T, H)) * 10.0 ** r.uniform(-2, 2)).astype(np.float32))
        w = r.standard_normal((T, K)).astype(np.float32)
        inputs.append((np.ascontiguousarray(x), np.ascontiguousarray(idx, np.int64), np.ascontiguousarray(w)))
    capacity = sum(len(x) for x, _, _ in inputs) + int(r.choice([0, 3]))
    L, state = run_local(inputs, E, world, capacity)
    check_step(L, state, inputs, E, world)
