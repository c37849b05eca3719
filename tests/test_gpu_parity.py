"""GPU parity: the CUDA library (called through its C ABI via the ctypes
binding) against the CPU oracle on the same seeded inputs.

Layout, indices, counts, offsets, CSR, dispatched bf16 rows and FP8
codes/scales must match bit for bit; combine must be within rtol 1e-5 /
atol 1e-6 (fp32 out) or 1 bf16 ulp (bf16 out).  Inputs come from
combine_ep_get_10_b200.workloads; expected values come from oracle/ only.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import assert_combine_close, exact_fraction, host, to_dev

pytestmark = pytest.mark.gpu

_INPUTS = {}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()
    yield
    _INPUTS.clear()


def inputs(cfg, T=None):
    key = (cfg, T)
    if key not in _INPUTS:
        _INPUTS[key] = W.make_inputs(cfg, T=T)
    return _INPUTS[key]


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def nan_filled(shape, dtype):
    """An output buffer holding NaN bit patterns, so that a row the kernel
    fails to write (or writes for the wrong token) cannot match the oracle."""
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


# ---------------------------------------------------------------- helpers
def gpu_tc_layout(idx_np, E, R, stream=None):
    idx = to_dev(np.ascontiguousarray(idx_np, np.int64))
    routing = B.Routing.topk(idx, E, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay, stream=stream)
    flags = B.ep_get_device_error(lay, stream=stream)
    return routing, lay, flags


def check_tc_layout(lay, ref):
    assert np.array_equal(host(lay.slot), ref["slot"]), "slot"
    assert np.array_equal(host(lay.num_tokens_per_expert), ref["num_tokens_per_expert"]), "counts"
    assert np.array_equal(host(lay.expert_offsets), ref["expert_offsets"]), "offsets"
    assert np.array_equal(host(lay.num_tokens_per_rank), ref["num_tokens_per_rank"]), "rank counts"
    assert np.array_equal(host(lay.is_token_in_rank), ref["is_token_in_rank"]), "is_token_in_rank"


def gpu_ec_layout(ti_np, T, R):
    ti = to_dev(np.ascontiguousarray(ti_np, np.int32))
    routing = B.Routing.expert_choice(ti, T, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    flags = B.ep_get_device_error(lay)
    return routing, lay, flags


def check_ec_layout(lay, ref):
    n = int(ref["token_offsets"][-1])
    assert np.array_equal(host(lay.token_offsets), ref["token_offsets"]), "token_offsets"
    assert np.array_equal(host(lay.token_slots)[:n], ref["token_slots"][:n]), "token_slots"
    assert np.array_equal(host(lay.num_tokens_per_expert), ref["num_tokens_per_expert"]), "counts"
    assert np.array_equal(host(lay.num_tokens_per_rank), ref["num_tokens_per_rank"]), "rank counts"
    assert np.array_equal(host(lay.is_token_in_rank), ref["is_token_in_rank"]), "is_token_in_rank"


# ----------------------------------------------------------- token-choice layout
@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_tc_layout_workloads(cfg):
    inp = inputs(cfg)
    c = inp["cfg"]
    ref = oracle.tc_layout(inp["topk_idx"], c["E"], c["R"])
    _, lay, flags = gpu_tc_layout(inp["topk_idx"], c["E"], c["R"])
    check_tc_layout(lay, ref)
    assert flags == 0


TC_EDGE = [
    # T, E, R, K, p_neg, dup, p_bad, seed
    (100000, 256, 8, 8, 0.05, False, 0.0, 1),   # many tokens: full 16-CTA cluster, several steps per warp
    (777, 64, 32, 40, 0.3, True, 0.01, 2),      # K > 32, R = 32, duplicates, bad ids
    (5000, 1024, 16, 8, 0.1, True, 0.0, 3),     # E at the layout limit
    (3000, 1, 1, 4, 0.2, True, 0.0, 4),         # one expert: every pair in one segment
    (2000, 16, 4, 3, 1.0, False, 0.0, 5),       # nothing routed
    (0, 8, 2, 2, 0.0, False, 0.0, 6),           # no tokens
    (1, 4, 1, 1, 0.0, False, 0.0, 7),
    (33, 7, 7, 5, 0.1, True, 0.2, 8),           # bad ids flagged, treated as -1
    (4097, 256, 8, 8, 0.0, False, 0.0, 9),      # ragged last CTA
]


@pytest.mark.parametrize("case", TC_EDGE, ids=[str(c[:4]) for c in TC_EDGE])
def test_tc_layout_edges(case):
    T, E, R, K, p_neg, dup, p_bad, seed = case
    idx = W.random_topk(rng(seed), T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad).reshape(T, K)
    ref = oracle.tc_layout(idx, E, R)
    _, lay, flags = gpu_tc_layout(idx, E, R)
    check_tc_layout(lay, ref)
    assert bool(flags & B.EP_DEVERR_BAD_INDEX) == (ref["bad_index_count"] > 0)


def test_tc_layout_deterministic_and_on_side_stream():
    inp = inputs(2)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _, lay1, _ = gpu_tc_layout(inp["topk_idx"], 256, 8, stream=s)
        _, lay2, _ = gpu_tc_layout(inp["topk_idx"], 256, 8, stream=s)
    s.synchronize()
    assert torch.equal(lay1.slot, lay2.slot) and torch.equal(lay1.expert_offsets, lay2.expert_offsets)


# --------------------------------------------------------- token-choice dispatch
@pytest.mark.parametrize("cfg", [1, 2, 5])
def test_tc_dispatch_bf16_compact(cfg):
    inp = inputs(cfg)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, c["E"], c["R"])
    want_extra = cfg != 5
    ref = oracle.tc_dispatch(x, idx, c["E"], ref_l, topk_weights=w, want_src=want_extra, want_weights=want_extra)
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    n = int(ref_l["expert_offsets"][-1])
    xd = to_dev(x, bf16=True)
    recv = torch.empty((n, c["H"]), dtype=torch.bfloat16, device="cuda")
    src = torch.full((n,), -1, dtype=torch.int32, device="cuda") if want_extra else None
    rw = torch.zeros(n, dtype=torch.float32, device="cuda") if want_extra else None
    B.ep_dispatch(xd, routing, lay, recv, topk_weights=to_dev(w), recv_src=src, recv_weights=rw)
    assert B.ep_get_device_error(lay) == 0
    assert np.array_equal(host(recv), ref["recv"])
    if want_extra:
        assert np.array_equal(host(src), ref["recv_src"]) and np.array_equal(host(rw), ref["recv_weights"])


def test_tc_dispatch_fp8_padded_decode():
    inp = inputs(3)
    c = inp["cfg"]
    E, H, mt = c["E"], c["H"], c["max_tokens"]
    x, idx = inp["x"], inp["topk_idx"]
    ref_l = oracle.tc_layout(idx, E, c["R"])
    ref = oracle.tc_dispatch(x, idx, E, ref_l, mode=W.PADDED, max_tokens=mt, out_dtype=W.FP8_E4M3)
    routing, lay, _ = gpu_tc_layout(idx, E, c["R"])
    recv = torch.full((E * mt, H), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((E * mt, H // 128), -1.0, dtype=torch.float32, device="cuda")
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, recv, mode=B.EP_LAYOUT_PADDED, max_tokens_per_expert=mt,
                  recv_scales=scales)
    assert B.ep_get_device_error(lay) == 0
    counts = ref_l["num_tokens_per_expert"]
    got, gs = host(recv), host(scales)
    valid = np.zeros(E * mt, bool)
    for e in range(E):
        valid[e * mt:e * mt + counts[e]] = True
    assert np.array_equal(got[valid], ref["recv"][valid])
    assert np.array_equal(gs[valid].view(np.uint32), ref["recv_scales"][valid].view(np.uint32))
    assert (got[~valid] == 0xAB).all() and (gs[~valid] == -1.0).all()  # padding rows untouched


@pytest.mark.parametrize("mode,mt,dtype", [(W.PADDED, 3, W.BF16), (W.PADDED, 5, W.FP8_E4M3), (W.COMPACT, 0, W.FP8_E4M3)])
def test_tc_dispatch_small_edges(mode, mt, dtype):
    """Padded overflow (flagged, skipped), duplicates, -1, K > 32, FP8 compact,
    a ragged two-chunk row (H = 8264 -> 16528-byte rows), and special values."""
    r = rng(77)
    T, E, R, K = 45, 12, 3, 36
    H = 8264 if dtype == W.BF16 else 384
    idx = W.random_topk(r, T, E, K, p_neg=0.2, allow_dup=True, p_bad=0.02)
    xf = r.standard_normal((T, H)).astype(np.float32) * np.float32(3.0)
    xf[0, :128] = 0.0  # an all-zero group
    xf[1, 128:256] *= np.float32(1e-38)  # tiny group: 448/amax overflows fp32
    xf[2, 5] = -0.0
    x = W.to_bf16_bits(xf)
    w = r.random((T, K)).astype(np.float32)
    ref_l = oracle.tc_layout(idx, E, R)
    rows = E * mt if mode == W.PADDED else int(ref_l["expert_offsets"][-1])
    ref = oracle.tc_dispatch(x, idx, E, ref_l, mode=mode, max_tokens=mt, out_dtype=dtype, topk_weights=w,
                             want_src=True, want_weights=True)
    routing, lay, flags = gpu_tc_layout(idx, E, R)
    assert flags & B.EP_DEVERR_BAD_INDEX
    if dtype == W.BF16:
        recv = torch.zeros((rows, H), dtype=torch.bfloat16, device="cuda")
        scales = None
    else:
        recv = torch.zeros((rows, H), dtype=torch.uint8, device="cuda")
        scales = torch.zeros((rows, H // 128), dtype=torch.float32, device="cuda")
    src = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    rw = torch.zeros(rows, dtype=torch.float32, device="cuda")
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, recv, mode=mode, max_tokens_per_expert=mt,
                  topk_weights=to_dev(w), recv_scales=scales, recv_src=src, recv_weights=rw)
    flags = B.ep_get_device_error(lay)
    assert bool(flags & B.EP_DEVERR_OVERFLOW) == (ref["overflow_count"] > 0)
    assert np.array_equal(host(recv), ref["recv"])
    if scales is not None:
        assert np.array_equal(host(scales).view(np.uint32), ref["recv_scales"].view(np.uint32))
    assert np.array_equal(host(src), ref["recv_src"]) and np.array_equal(host(rw), ref["recv_weights"])


def test_fp8_cast_matches_oracle_codec_on_a_sweep():
    """Device FP8 cast against the oracle codec over many bf16 inputs and
    scales: every bf16 exponent range, and groups whose amax is any bf16."""
    r = rng(91)
    T, H = 512, 1024
    mag = np.float32(2.0) ** r.integers(-40, 40, size=(T, H // 128, 1)).astype(np.float32)
    xf = (r.standard_normal((T, H // 128, 128)).astype(np.float32) * mag).reshape(T, H)
    x = W.to_bf16_bits(xf)
    idx = np.arange(T, dtype=np.int64).reshape(T, 1) % 4
    ref_l = oracle.tc_layout(idx, 4, 1)
    ref = oracle.tc_dispatch(x, idx, 4, ref_l, out_dtype=W.FP8_E4M3)
    routing, lay, _ = gpu_tc_layout(idx, 4, 1)
    recv = torch.zeros((T, H), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((T, H // 128), dtype=torch.float32, device="cuda")
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, recv, recv_scales=scales)
    assert np.array_equal(host(recv), ref["recv"])
    assert np.array_equal(host(scales).view(np.uint32), ref["recv_scales"].view(np.uint32))


# ---------------------------------------------------------- token-choice combine
def _combine_both(y_np, routing, lay, w_np, T, H, mode=W.COMPACT, mt=0, num_rows=None):
    yd = to_dev(y_np, bf16=True)
    wd = to_dev(w_np)
    outs = {}
    for dt in (W.FP32, W.BF16):
        out = nan_filled((T, H), torch.float32 if dt == W.FP32 else torch.bfloat16)
        B.ep_combine(yd, routing, lay, wd, out, mode=mode, max_tokens_per_expert=mt, num_y_rows=num_rows)
        outs[dt] = host(out)
    return outs


def test_tc_combine_tiny_closed_form_workload():
    """Workload 1: expert outputs are the dispatched rows times (e+1)."""
    inp = inputs(1)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, 8, 2)
    recv = oracle.tc_dispatch(x, idx, 8, ref_l)["recv"]
    e_of_row = np.searchsorted(ref_l["expert_offsets"], np.arange(recv.shape[0]), side="right") - 1
    y = W.to_bf16_bits(oracle.bf16_to_f32(recv) * (e_of_row[:, None] + 1).astype(np.float32))
    routing, lay, _ = gpu_tc_layout(idx, 8, 2)
    outs = _combine_both(y, routing, lay, w, 128, 256)
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        ref = oracle.tc_combine(y, idx, 8, ref_l, w, out_dtype=dt)
        assert_combine_close(outs[dt], ref, bf, "workload 1")
        assert exact_fraction(outs[dt], ref) == 1.0


def test_tc_combine_prefill_workload():
    inp = inputs(2)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, c["E"], c["R"])
    y = oracle.tc_dispatch(x, idx, c["E"], ref_l)["recv"]
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    outs = _combine_both(y, routing, lay, w, c["T"], c["H"])
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        ref = oracle.tc_combine(y, idx, c["E"], ref_l, w, out_dtype=dt)
        assert_combine_close(outs[dt], ref, bf, "workload 2")
        assert exact_fraction(outs[dt], ref) == 1.0


def test_tc_pipeline_prefill_gpu_end_to_end():
    """layout -> dispatch -> combine entirely on the GPU (the benchmarked
    step), against the oracle's own layout -> dispatch -> combine."""
    inp = inputs(2)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, c["E"], c["R"])
    ref_y = oracle.tc_dispatch(x, idx, c["E"], ref_l)["recv"]
    ref = oracle.tc_combine(ref_y, idx, c["E"], ref_l, w, out_dtype=W.BF16)
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    n = c["T"] * c["K"]
    recv = torch.empty((n, c["H"]), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((c["T"], c["H"]), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, recv)
    B.ep_combine(recv, routing, lay, to_dev(w), out)
    assert B.ep_get_device_error(lay) == 0
    assert_combine_close(host(out), ref, True, "pipeline")


def test_tc_dispatch_combine_in_token_chunks():
    """Dispatch and combine called on token sub-ranges (offset views of the
    routing, layout, x, weights and out) give the same bytes as one call."""
    inp = inputs(2)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, c["E"], c["R"])
    ref_y = oracle.tc_dispatch(x, idx, c["E"], ref_l)["recv"]
    ref = oracle.tc_combine(ref_y, idx, c["E"], ref_l, w, out_dtype=W.BF16)
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    n = c["T"] * c["K"]
    xd, wd = to_dev(x, bf16=True), to_dev(w)
    recv = torch.empty((n, c["H"]), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((c["T"], c["H"]), dtype=torch.bfloat16, device="cuda")
    bounds = [0, 1, 1000, 1000, 2555, 4096]  # includes an empty and a one-token chunk
    for t0, t1 in zip(bounds[:-1], bounds[1:]):
        r = routing.tokens(t0, t1)
        v = B.layout_tokens(lay, routing, t0, t1)
        B.ep_dispatch(xd[t0:t1], r, v, recv, num_recv_rows=n)
    for t0, t1 in zip(bounds[:-1], bounds[1:]):
        r = routing.tokens(t0, t1)
        v = B.layout_tokens(lay, routing, t0, t1)
        B.ep_combine(recv, r, v, wd[t0:t1], out[t0:t1], num_y_rows=n)
    assert B.ep_get_device_error(lay) == 0
    assert np.array_equal(host(recv), ref_y)
    assert np.array_equal(host(out), ref)


def test_tc_combine_decode_padded():
    inp = inputs(3)
    c = inp["cfg"]
    E, H, mt = c["E"], c["H"], c["max_tokens"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, E, c["R"])
    y = oracle.tc_dispatch(x, idx, E, ref_l, mode=W.PADDED, max_tokens=mt)["recv"]
    routing, lay, _ = gpu_tc_layout(idx, E, c["R"])
    outs = _combine_both(y, routing, lay, w, c["T"], H, mode=W.PADDED, mt=mt)
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        ref = oracle.tc_combine(y, idx, E, ref_l, w, mode=W.PADDED, max_tokens=mt, out_dtype=dt)
        assert_combine_close(outs[dt], ref, bf, "workload 3")


def test_tc_combine_skewed_sampled():
    """Workload 5 at full size; the oracle computes a sample of tokens."""
    inp = inputs(5)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref_l = oracle.tc_layout(idx, c["E"], c["R"])
    y = oracle.tc_dispatch(x, idx, c["E"], ref_l)["recv"]
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    yd = to_dev(y, bf16=True)
    out = torch.empty((c["T"], c["H"]), dtype=torch.bfloat16, device="cuda")
    B.ep_combine(yd, routing, lay, to_dev(w), out)
    tokens = np.sort(rng(5).choice(c["T"], 1500, replace=False)).astype(np.int32)
    tokens = np.concatenate([tokens, np.nonzero((idx < 0).all(axis=1))[0].astype(np.int32)])
    ref = oracle.tc_combine(y, idx, c["E"], ref_l, w, out_dtype=W.BF16, tokens=tokens)
    got = host(out)[tokens]
    assert_combine_close(got, ref, True, "workload 5")
    assert exact_fraction(got, ref) == 1.0


def test_tc_combine_edges():
    """K > 32, duplicates, -1 slots, tokens with nothing routed, padded
    overflow rows skipped, a ragged segment (H = 200)."""
    r = rng(55)
    T, E, R, K, H, mt = 70, 10, 5, 37, 200, 40
    idx = W.random_topk(r, T, E, K, p_neg=0.3, allow_dup=True)
    idx[3] = -1
    w = r.standard_normal((T, K)).astype(np.float32)
    ref_l = oracle.tc_layout(idx, E, R)
    routing, lay, _ = gpu_tc_layout(idx, E, R)
    for mode in (W.COMPACT, W.PADDED):
        rows = E * mt if mode == W.PADDED else int(ref_l["expert_offsets"][-1])
        y = W.to_bf16_bits(r.standard_normal((rows, H)).astype(np.float32))
        outs = _combine_both(y, routing, lay, w, T, H, mode=mode, mt=mt)
        for dt, bf in ((W.FP32, False), (W.BF16, True)):
            ref = oracle.tc_combine(y, idx, E, ref_l, w, mode=mode, max_tokens=mt, out_dtype=dt)
            assert_combine_close(outs[dt], ref, bf, "edges")
            assert exact_fraction(outs[dt], ref) == 1.0
            assert (outs[dt][3] == 0).all()
    assert B.ep_get_device_error(lay) & B.EP_DEVERR_OVERFLOW  # padded rows past 40 were skipped


# ------------------------------------------------------------------ expert choice
@pytest.mark.parametrize("R", [1, 8])
def test_ec_workload(R):
    inp = inputs(4)
    c = inp["cfg"]
    T, E, C, H = c["T"], c["E"], c["C"], c["H"]
    ti, ew, x = inp["token_indices"], inp["expert_weights"], inp["x"]
    ref_l = oracle.ec_layout(ti, T, R)
    routing, lay, flags = gpu_ec_layout(ti, T, R)
    assert flags == 0
    check_ec_layout(lay, ref_l)
    ref_recv = oracle.ec_dispatch(x, ti)
    recv = torch.empty((E * C, H), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch_expert_choice(to_dev(x, bf16=True), routing, lay, recv)
    assert np.array_equal(host(recv), ref_recv)
    wd = to_dev(ew)
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        out = nan_filled((T, H), torch.float32 if dt == W.FP32 else torch.bfloat16)
        B.ep_combine_expert_choice(to_dev(ref_recv, bf16=True), routing, lay, wd, out)
        ref = oracle.ec_combine(ref_recv, ref_l, ew, T, out_dtype=dt)
        got = host(out)
        assert_combine_close(got, ref, bf, "expert choice")
        assert exact_fraction(got, ref) == 1.0
    assert B.ep_get_device_error(lay) == 0


EC_EDGE = [
    # T, E, C, R, H, p_neg, p_bad, seed
    (50, 8, 16, 2, 256, 0.0, 0.0, 1),   # the page's randint table: duplicates within rows
    (20, 16, 8, 4, 136, 0.2, 0.05, 2),  # empty and bad slots, ragged segment
    (5, 40, 6, 8, 64, 0.1, 0.0, 3),     # every token picked far more than 32 times
    (3000, 4, 5, 1, 64, 0.0, 0.0, 4),   # most tokens unpicked
    (1, 3, 2, 3, 8, 0.5, 0.0, 5),
    (20000, 2, 700, 1, 8, 0.0, 0.0, 6),  # scan over several 8192-token passes
    (3000, 64, 1024, 4, 64, 0.0, 0.0, 7),  # ~3000 tokens with >= 16 picks: more than the combine lists
    (70000, 2, 1000, 1, 8, 0.0, 0.0, 8),  # T above the combine's heavy-listing limit
    (100, 128, 64, 1, 1000, 0.0, 0.0, 9),  # lists of ~80 picks: the narrow heavy segments, ragged hidden
]


@pytest.mark.parametrize("case", EC_EDGE, ids=[str(c[:4]) for c in EC_EDGE])
def test_ec_edges(case):
    T, E, C, R, H, p_neg, p_bad, seed = case
    r = rng(seed)
    ti = W.random_token_indices(r, T, E, C, p_neg=p_neg, p_bad=p_bad)
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    ew = r.standard_normal((E, C)).astype(np.float32)
    ref_l = oracle.ec_layout(ti, T, R)
    routing, lay, flags = gpu_ec_layout(ti, T, R)
    assert bool(flags & B.EP_DEVERR_BAD_INDEX) == (ref_l["bad_index_count"] > 0)
    check_ec_layout(lay, ref_l)
    sentinel = np.full((E * C, H), 0x7FC1, np.uint16)
    ref_recv = oracle.ec_dispatch(x, ti, recv=sentinel.copy())
    recv = to_dev(sentinel, bf16=True)
    B.ep_dispatch_expert_choice(to_dev(x, bf16=True), routing, lay, recv)
    assert np.array_equal(host(recv), ref_recv)
    y = W.to_bf16_bits(r.standard_normal((E * C, H)).astype(np.float32))
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        out = nan_filled((T, H), torch.float32 if dt == W.FP32 else torch.bfloat16)
        B.ep_combine_expert_choice(to_dev(y, bf16=True), routing, lay, to_dev(ew), out)
        ref = oracle.ec_combine(y, ref_l, ew, T, out_dtype=dt)
        assert_combine_close(host(out), ref, bf, "ec edges")
        assert exact_fraction(host(out), ref) == 1.0


@pytest.mark.parametrize("T,E,C,H", [(600, 96, 64, 1000), (1000, 128, 64, 264)])
def test_ec_skewed_mixed(T, E, C, H):
    """The workload's skewed expert-choice router at a size the oracle checks
    whole: unpicked tokens, light tokens and heavy ones of every degree class
    (>= 64, 32-63, 16-31 picks) in one launch, ragged hidden sizes."""
    r = rng(T)
    ti, ew = W.route_expert_choice(r, T, E, C)
    deg = np.bincount(ti[ti >= 0].ravel(), minlength=T)
    assert (deg >= 64).any() and ((deg >= 32) & (deg < 64)).any() and ((deg >= 16) & (deg < 32)).any()
    assert ((deg > 0) & (deg < 16)).any() and (deg == 0).any()
    ref_l = oracle.ec_layout(ti, T, 2)
    routing, lay, flags = gpu_ec_layout(ti, T, 2)
    assert flags == 0
    y = W.to_bf16_bits(r.standard_normal((E * C, H)).astype(np.float32))
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        out = nan_filled((T, H), torch.float32 if dt == W.FP32 else torch.bfloat16)
        B.ep_combine_expert_choice(to_dev(y, bf16=True), routing, lay, to_dev(ew), out)
        ref = oracle.ec_combine(y, ref_l, ew, T, out_dtype=dt)
        assert_combine_close(host(out), ref, bf, "ec skewed")
        assert exact_fraction(host(out), ref) == 1.0
    assert B.ep_get_device_error(lay) == 0


EC_ONE_CALL = [None, EC_EDGE[1], EC_EDGE[2], EC_EDGE[5], EC_EDGE[7]]  # None: the expert-choice workload, R = 8


@pytest.mark.parametrize("case", EC_ONE_CALL, ids=["workload"] + [str(c[:4]) for c in EC_ONE_CALL[1:]])
def test_ec_layout_dispatch_one_call_equals_the_two_calls(case):
    """ep_layout_dispatch_expert_choice: the layout and the copy in one call
    (the copy runs under the layout kernel and ends after it) writes the same
    CSR, counts, rows and error bits as the two calls, against the oracle,
    with the rows of empty or bad slots untouched and num_valid_host
    reported; a combine queued right after it on the same stream, with no
    synchronisation in between, reads the finished CSR (bit for bit)."""
    if case is None:
        inp = inputs(4)
        c = inp["cfg"]
        T, E, C, H, R = c["T"], c["E"], c["C"], c["H"], 8
        ti, ew, x = inp["token_indices"], inp["expert_weights"], inp["x"]
        r = rng(44)
    else:
        T, E, C, R, H, p_neg, p_bad, seed = case
        r = rng(seed)
        ti = W.random_token_indices(r, T, E, C, p_neg=p_neg, p_bad=p_bad)
        x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
        ew = r.standard_normal((E, C)).astype(np.float32)
    ref_l = oracle.ec_layout(ti, T, R)
    sentinel = np.full((E * C, H), 0x7FC1, np.uint16)
    ref_recv = oracle.ec_dispatch(x, ti, recv=sentinel.copy())
    tid, xd = to_dev(np.ascontiguousarray(ti, np.int32)), to_dev(x, bf16=True)
    routing = B.Routing.expert_choice(tid, T, R)
    lay = B.Layout(routing, report_num_valid=True)
    recv = to_dev(sentinel, bf16=True)
    B.ep_layout_dispatch_expert_choice(xd, routing, lay, recv)
    assert lay.num_valid == int(ref_l["token_offsets"][-1])
    check_ec_layout(lay, ref_l)
    assert np.array_equal(host(recv), ref_recv)
    flags = B.ep_get_device_error(lay)
    assert bool(flags & B.EP_DEVERR_BAD_INDEX) == (ref_l["bad_index_count"] > 0)
    # again without the host report, the combine queued straight behind it
    lay2 = B.Layout(routing)
    recv2 = to_dev(sentinel, bf16=True)
    out = nan_filled((T, H), torch.float32)
    B.ep_layout_dispatch_expert_choice(xd, routing, lay2, recv2)
    B.ep_combine_expert_choice(recv2, routing, lay2, to_dev(ew), out)
    ref = oracle.ec_combine(ref_recv, ref_l, ew, T, out_dtype=W.FP32)
    assert exact_fraction(host(out), ref) == 1.0
    assert np.array_equal(host(recv2), ref_recv)


def test_device_error_word_clears():
    idx = np.array([[0, 9], [1, -1]], np.int64)  # 9 is out of range for E = 4
    _, lay, flags = gpu_tc_layout(idx, 4, 2)
    assert flags == B.EP_DEVERR_BAD_INDEX
    assert B.ep_get_device_error(lay) == 0  # cleared by the previous read


def test_long_sequence_in_rounds():
    """Long-sequence rounds ("ant moving home"): 32768 tokens of the skewed
    routing in rounds of 8192, each with its own layout and a receive buffer
    of 8192 * K rows; the combined output equals the one-shot oracle combine
    (identity experts), checked on sampled tokens, and each round's buffer
    holds exactly that round's routed pairs."""
    inp = W.make_inputs(5, T=32768)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    T, H, E, R, K = idx.shape[0], c["H"], c["E"], c["R"], c["K"]
    P = 8192
    xd, idxd, wd = to_dev(x, bf16=True), to_dev(idx), to_dev(w)
    routing = B.Routing.topk(idxd, E, R)
    recv = torch.empty((P * K, H), dtype=torch.bfloat16, device="cuda")
    out = nan_filled((T, H), torch.bfloat16)
    rounds = B.token_rounds(T, P)
    assert len(rounds) == 4
    for t0, t1 in rounds:
        r = routing.tokens(t0, t1)
        lay = B.Layout(r, report_num_valid=True)
        B.ep_get_layout(r, lay)  # returns with the round's routed-pair count on the host
        n = lay.num_valid
        assert n == int((idx[t0:t1] >= 0).sum()) <= P * K
        B.ep_dispatch(xd[t0:t1], r, lay, recv, num_recv_rows=n)
        B.ep_combine(recv, r, lay, wd[t0:t1], out[t0:t1], num_y_rows=n)
        assert B.ep_get_device_error(lay) == 0
    tokens = np.sort(rng(17).choice(T, size=256, replace=False)).astype(np.int32)
    # per sampled token, the one-shot path restricted to that token (its
    # combine reads only its own pairs' rows, which identity experts fill
    # with x[t]): the oracle's dispatch + combine of that one-token routing
    ref = np.empty((tokens.size, H), np.uint16)
    for i, t in enumerate(tokens):
        l1 = oracle.tc_layout(idx[t:t + 1], E, R)
        y1 = oracle.tc_dispatch(x[t:t + 1], idx[t:t + 1], E, l1)["recv"]
        ref[i] = oracle.tc_combine(y1, idx[t:t + 1], E, l1, w[t:t + 1], out_dtype=W.BF16)[0]
    got = host(out[torch.from_numpy(tokens).cuda()])
    assert_combine_close(got, ref, True, "rounds")
    assert exact_fraction(got, ref) == 1.0


def test_combine_into_pinned_host_memory():
    """`out` may be pinned host memory (mapped under unified addressing): the
    combine's stores then cross PCIe directly, and the bytes equal those of
    a device output."""
    inp = inputs(2, T=512)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    routing, lay, _ = gpu_tc_layout(idx, c["E"], c["R"])
    n = int(host(lay.expert_offsets)[-1])
    recv = torch.empty((n, c["H"]), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, recv)
    wd = to_dev(w)
    out_d = torch.empty((512, c["H"]), dtype=torch.bfloat16, device="cuda")
    out_h = torch.zeros((512, c["H"]), dtype=torch.bfloat16).pin_memory()
    B.ep_combine(recv, routing, lay, wd, out_d)
    B.ep_combine(recv, routing, lay, wd, out_h)
    torch.cuda.synchronize()
    assert B.ep_get_device_error(lay) == 0
    assert torch.equal(out_d.cpu().view(torch.int16), out_h.view(torch.int16))


def test_num_valid_host_reports_the_filled_rows():
    """layout->num_valid_host: the layout call copies the filled-row count to
    the host and returns after the stream caught up; the value equals the
    oracle's expert_offsets[E] (token choice) or token_offsets[T] (expert
    choice), for the plain, the fused low-latency and the no-alloc layouts."""
    for wl in (2, 5):
        inp = inputs(wl, T=3000)
        c = inp["cfg"]
        idx = inp["topk_idx"]
        ref = oracle.tc_layout(idx, c["E"], c["R"])
        routing = B.Routing.topk(to_dev(idx), c["E"], c["R"])
        lay = B.Layout(routing, report_num_valid=True)
        lay.num_valid_host[0] = -5
        B.ep_get_layout(routing, lay)
        assert lay.num_valid == int(ref["expert_offsets"][-1])
        lay.num_valid_host[0] = -5
        B.ep_get_layout_no_alloc(routing, lay)
        assert lay.num_valid == int(ref["expert_offsets"][-1])
    inp = inputs(3)
    c = inp["cfg"]
    idx, mt = inp["topk_idx"], c["max_tokens"]
    routing = B.Routing.topk(to_dev(idx), c["E"], c["R"])
    lay = B.Layout(routing, report_num_valid=True)
    q = torch.empty((c["E"] * mt, c["H"]), dtype=torch.uint8, device="cuda")
    sc = torch.empty((c["E"] * mt, c["H"] // 128), dtype=torch.float32, device="cuda")
    B.ep_dispatch_low_latency(to_dev(inp["x"], bf16=True), routing, lay, q, max_tokens_per_expert=mt,
                              recv_scales=sc)
    assert lay.num_valid == int(oracle.tc_layout(idx, c["E"], c["R"])["expert_offsets"][-1])
    inp = inputs(4)
    c = inp["cfg"]
    ti = inp["token_indices"]
    routing = B.Routing.expert_choice(to_dev(ti), c["T"], 1)
    lay = B.Layout(routing, report_num_valid=True)
    B.ep_get_layout(routing, lay)
    assert lay.num_valid == int(oracle.ec_layout(ti, c["T"], 1)["token_offsets"][-1])
    assert B.ep_get_device_error(lay) == 0



@pytest.mark.parametrize("T,H", [(8192, 512), (9000, 264)])
def test_tc_combine_large_batches_every_output(T, H):
    """From 8192 tokens on, the token-choice and per-rank combines read pairs
    of 16-byte vectors with one 32-byte load when the rows allow it (H = 512
    here; H = 264 keeps 16-byte loads): every output element against the
    oracle, fp32 and bf16, from NaN-filled buffers."""
    r = rng(41)
    E, R, K = 64, 8, 6
    idx = W.random_topk(r, T, E, K, p_neg=0.1)
    x = W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32))
    w = r.random((T, K)).astype(np.float32)
    ref_l = oracle.tc_layout(idx, E, R)
    routing, lay, flags = gpu_tc_layout(idx, E, R)
    assert flags == 0
    n = int(ref_l["expert_offsets"][-1])
    y = W.to_bf16_bits(r.standard_normal((n, H)).astype(np.float32))
    yd = to_dev(y, bf16=True)
    for dt, bf in ((W.FP32, False), (W.BF16, True)):
        out = nan_filled((T, H), torch.float32 if dt == W.FP32 else torch.bfloat16)
        B.ep_combine(yd, routing, lay, to_dev(w), out)
        ref = oracle.tc_combine(y, idx, E, ref_l, w, out_dtype=dt)
        assert_combine_close(host(out), ref, bf, "large-batch combine")
        assert exact_fraction(host(out), ref) == 1.0
    # per rank: the rank rows of the same routing, summed per token
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    rl = B.RankLayout(routing)
    B.ep_get_rank_layout(routing, lay, rl)
    nr = int(ref_rl["rank_offsets"][-1])
    yr = W.to_bf16_bits(r.standard_normal((nr, H)).astype(np.float32))
    rout = nan_filled((T, H), torch.float32)
    B.ep_combine_ranks(to_dev(yr, bf16=True), routing, lay, rl, rout)
    ref_r = oracle.rank_combine(yr, ref_rl, out_dtype=W.FP32)
    assert np.array_equal(host(rout).view(np.uint32), ref_r.view(np.uint32))
    assert B.ep_get_device_error(lay) == 0


def test_layout_dispatch_one_call_equals_the_two_calls():
    """ep_layout_dispatch: the layout and the dispatch in one call (the
    dispatch's row loads overlap the layout kernel) writes the same layout,
    rows and quantised codes as ep_get_layout + ep_dispatch, against the
    oracle, and reports the filled rows through num_valid_host."""
    inp = inputs(2, T=2048)
    c = inp["cfg"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    E, R, H = c["E"], c["R"], c["H"]
    ref_l = oracle.tc_layout(idx, E, R)
    n = int(ref_l["expert_offsets"][-1])
    routing = B.Routing.topk(to_dev(idx), E, R)
    lay = B.Layout(routing, report_num_valid=True)
    recv = to_dev(np.full((n, H), 0x7FC1, np.uint16), bf16=True)
    B.ep_layout_dispatch(to_dev(x, bf16=True), routing, lay, recv)
    assert lay.num_valid == n
    check_tc_layout(lay, ref_l)
    assert np.array_equal(host(recv), oracle.tc_dispatch(x, idx, E, ref_l)["recv"])
    q = torch.zeros((n, H), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((n, H // 128), dtype=torch.float32, device="cuda")
    B.ep_layout_dispatch(to_dev(x, bf16=True), routing, lay, q, recv_scales=sc, topk_weights=to_dev(w),
                         recv_weights=(rw := torch.zeros(n, dtype=torch.float32, device="cuda")))
    ref_q = oracle.tc_dispatch(x, idx, E, ref_l, out_dtype=W.FP8_E4M3, topk_weights=w, want_weights=True)
    assert np.array_equal(host(q), ref_q["recv"])
    assert np.array_equal(host(sc).view(np.uint32), ref_q["recv_scales"].view(np.uint32))
    assert np.array_equal(host(rw), ref_q["recv_weights"])
    assert B.ep_get_device_error(lay) == 0


@pytest.mark.parametrize("wl", [2, 5])
def test_layout_dispatch_full_size_equals_the_two_calls(wl):
    """ep_layout_dispatch at full size (the dispatch's CTAs start under the
    layout and read its slots and offsets after waiting for it), three times
    with layout outputs pre-filled with zeros: every received row equals the
    row the separate ep_get_layout + ep_dispatch calls write."""
    inp = inputs(wl)
    c = inp["cfg"]
    E, R, H = c["E"], c["R"], c["H"]
    xd = to_dev(inp["x"], bf16=True)
    routing = B.Routing.topk(to_dev(inp["topk_idx"]), E, R)
    lay0 = B.Layout(routing)
    B.ep_get_layout(routing, lay0)
    n = int(host(lay0.expert_offsets)[-1])
    ref = torch.full((n, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.ep_dispatch(xd, routing, lay0, ref, num_recv_rows=n)
    want = ref.view(torch.int16)
    for _ in range(3):
        lay = B.Layout(routing)
        lay.slot.fill_(0)
        lay.expert_offsets.fill_(0)
        out = torch.full((n, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        B.ep_layout_dispatch(xd, routing, lay, out, num_recv_rows=n)
        assert B.ep_get_device_error(lay) == 0
        assert int((out.view(torch.int16) != want).any(dim=1).sum().item()) == 0
        del out


def test_combine_queued_right_behind_a_layout_reads_the_finished_layout():
    """A combine (and a rank combine) queued directly behind ep_get_layout
    (and ep_get_rank_layout), with no synchronisation in between: the plain
    layout calls do not let the next kernel start early, so the combine's
    read-only loads of slots, offsets and rank rows see the finished
    layout; outputs bit for bit against the oracle."""
    inp = inputs(2, T=2048)
    c = inp["cfg"]
    idx, w = inp["topk_idx"], inp["topk_weights"]
    E, R, H, T = c["E"], c["R"], c["H"], 2048
    ref_l = oracle.tc_layout(idx, E, R)
    n = int(ref_l["expert_offsets"][-1])
    r = rng(77)
    y = W.to_bf16_bits(r.standard_normal((n, H)).astype(np.float32))
    yd, wd = to_dev(y, bf16=True), to_dev(w)
    routing = B.Routing.topk(to_dev(idx), E, R)
    lay = B.Layout(routing)
    lay.slot.fill_(0)
    lay.expert_offsets.fill_(0)
    out = nan_filled((T, H), torch.float32)
    B.ep_get_layout(routing, lay)
    B.ep_combine(yd, routing, lay, wd, out, num_y_rows=n)
    assert exact_fraction(host(out), oracle.tc_combine(y, idx, E, ref_l, w, out_dtype=W.FP32)) == 1.0
    ref_rl = oracle.rank_layout(ref_l["is_token_in_rank"])
    m = int(ref_rl["rank_offsets"][-1])
    yr = W.to_bf16_bits(r.standard_normal((m, H)).astype(np.float32))
    rl = B.RankLayout(routing)
    rl.rank_row.fill_(0)
    out_r = nan_filled((T, H), torch.float32)
    B.ep_get_rank_layout(routing, lay, rl)
    B.ep_combine_ranks(to_dev(yr, bf16=True), routing, lay, rl, out_r)
    assert exact_fraction(host(out_r), oracle.rank_combine(yr, ref_rl, out_dtype=W.FP32)) == 1.0
    assert B.ep_get_device_error(lay) == 0


def test_dispatch_reads_x_written_by_the_kernel_just_before():
    """ep_dispatch after a kernel that writes x on the same stream (the
    layout computed earlier): the dispatch waits for that kernel before its
    first read, so every dispatched row is the new x."""
    inp = inputs(2, T=1024)
    c = inp["cfg"]
    idx = inp["topk_idx"]
    E, R, H = c["E"], c["R"], c["H"]
    ref_l = oracle.tc_layout(idx, E, R)
    n = int(ref_l["expert_offsets"][-1])
    routing, lay, flags = gpu_tc_layout(idx, E, R)
    assert flags == 0
    r = rng(5)
    xd = torch.empty((1024, H), dtype=torch.bfloat16, device="cuda")
    recv = torch.empty((n, H), dtype=torch.bfloat16, device="cuda")
    for it in range(4):
        x = W.to_bf16_bits(r.standard_normal((1024, H)).astype(np.float32))
        src = to_dev(x, bf16=True)
        xd.copy_(src)  # a kernel on the stream writing x right before the dispatch
        B.ep_dispatch(xd, routing, lay, recv)
        assert np.array_equal(host(recv), oracle.tc_dispatch(x, idx, E, ref_l)["recv"]), it
