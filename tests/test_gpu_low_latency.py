"""GPU parity of the fused low-latency dispatch (DeepEP-Ascend README, API
Overview: low_latency_dispatch, which needs no separate layout call): one
launch must give exactly what ep_get_layout followed by a padded ep_dispatch
gives -- layout outputs, received rows (bf16 or any quantised format),
scales, sources, weights and device error bits -- checked against the CPU
oracle.  Batches beyond the fused limits take the two-call path."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu

FORMATS = [W.BF16, W.FP8_E4M3, W.INT8_PER_TOKEN, W.FP8_E4M3_PER_TOKEN, W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _run(x, idx, w, E, R, mt, dt):
    T, H = x.shape
    K = idx.shape[1]
    rows = E * mt
    ref_l = oracle.tc_layout(idx, E, R)
    ref = oracle.tc_dispatch(x, idx, E, ref_l, mode=W.PADDED, max_tokens=mt, out_dtype=dt, topk_weights=w,
                             want_src=True, want_weights=True)
    routing = B.Routing.topk(to_dev(np.ascontiguousarray(idx, np.int64)), E, R)
    lay = B.Layout(routing)
    # poison the layout outputs so that stale values cannot pass
    for tns in (lay.num_tokens_per_expert, lay.expert_offsets, lay.num_tokens_per_rank, lay.slot):
        tns.fill_(-77)
    lay.is_token_in_rank.fill_(9)
    if dt == W.BF16:
        recv = torch.full((rows, H), -3.0, dtype=torch.bfloat16, device="cuda")
        sc = None
    else:
        recv = torch.full((rows, oracle.row_code_bytes(dt, H)), 0xAB, dtype=torch.uint8, device="cuda")
        sc = torch.full((rows, oracle.row_scale_bytes(dt, H)), 0x5A, dtype=torch.uint8, device="cuda")
    src = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    rw = torch.zeros(rows, dtype=torch.float32, device="cuda")
    B.ep_dispatch_low_latency(to_dev(x, bf16=True), routing, lay, recv, max_tokens_per_expert=mt, out_dtype=dt,
                              topk_weights=to_dev(w), recv_scales=sc, recv_src=src, recv_weights=rw)
    flags = B.ep_get_device_error(lay)
    assert np.array_equal(host(lay.slot), ref_l["slot"]), "slot"
    assert np.array_equal(host(lay.num_tokens_per_expert), ref_l["num_tokens_per_expert"]), "counts"
    assert np.array_equal(host(lay.expert_offsets), ref_l["expert_offsets"]), "offsets"
    assert np.array_equal(host(lay.num_tokens_per_rank), ref_l["num_tokens_per_rank"]), "rank counts"
    assert np.array_equal(host(lay.is_token_in_rank), ref_l["is_token_in_rank"]), "in rank"
    counts = ref_l["num_tokens_per_expert"]
    valid = np.zeros(rows, bool)
    for e in range(E):
        valid[e * mt:e * mt + min(int(counts[e]), mt)] = True
    g = host(recv)
    if dt == W.BF16:
        assert np.array_equal(g[valid], ref["recv"][valid])
    else:
        gc = g.view(np.uint8).reshape(rows, -1)
        rc = np.ascontiguousarray(ref["recv"]).view(np.uint8).reshape(rows, -1)
        gs = host(sc).reshape(rows, -1)
        rs = np.ascontiguousarray(ref["recv_scales"]).view(np.uint8).reshape(rows, -1)
        assert np.array_equal(gc[valid], rc[valid]) and np.array_equal(gs[valid], rs[valid])
        assert (gc[~valid] == 0xAB).all() and (gs[~valid] == 0x5A).all()
    assert np.array_equal(host(src), ref["recv_src"]) and np.array_equal(host(rw), ref["recv_weights"])
    return flags, ref


@pytest.mark.parametrize("dt", FORMATS)
def test_low_latency_decode_workload(dt):
    """The decode workload: 128 tokens, hidden 7168, 256 experts in 8 ranks,
    top-8, 128-row padded buffers per expert."""
    inp = W.make_inputs(3)
    c = inp["cfg"]
    flags, _ = _run(inp["x"], inp["topk_idx"], inp["topk_weights"], c["E"], c["R"], c["max_tokens"], dt)
    assert flags == 0


@pytest.mark.parametrize("case", [
    # T, E, R, K, H, mt, p_neg, dup, p_bad, seed
    (1, 4, 1, 4, 128, 4, 0.0, False, 0.0, 1),
    (45, 12, 3, 32, 384, 5, 0.2, True, 0.02, 2),   # K = 32, duplicates, bad ids, overflow
    (256, 1024, 32, 8, 256, 3, 0.1, False, 0.0, 3),  # E = 1024, R = 32
    (1024, 64, 8, 8, 128, 200, 0.0, False, 0.0, 4),  # T*K = 8192: the largest fused batch
    (1100, 64, 8, 8, 128, 200, 0.0, False, 0.0, 5),  # beyond: the two-call path
    (20, 8, 2, 40, 128, 40, 0.3, True, 0.0, 6),      # K > 32: the two-call path
], ids=lambda c: "T%d_E%d_R%d_K%d" % c[:4])
def test_low_latency_edges(case):
    T, E, R, K, H, mt, p_neg, dup, p_bad, seed = case
    r = _rng(seed)
    idx = W.random_topk(r, T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad)
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    w = r.random((T, K)).astype(np.float32)
    for dt in (W.BF16, W.MXFP8_E4M3):
        flags, ref = _run(x, idx, w, E, R, mt, dt)
        assert bool(flags & B.EP_DEVERR_BAD_INDEX) == (p_bad > 0)
        assert bool(flags & B.EP_DEVERR_OVERFLOW) == (ref["overflow_count"] > 0)
