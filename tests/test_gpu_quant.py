"""GPU parity of the quantised dispatch formats (DeepEP-Ascend README,
"Quantization Modes in Normal Dispatch": int8 and scalar FP8 per token, MX
FP8 e4m3 / e5m2 and MX FP4 e2m1 per 32 elements, and the 128-channel FP8 of
low_latency_dispatch) against the CPU oracle: codes and scales bit for bit,
rows the routing does not name left untouched."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import host, to_dev

pytestmark = pytest.mark.gpu

QUANT = [W.FP8_E4M3, W.INT8_PER_TOKEN, W.FP8_E4M3_PER_TOKEN, W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1]
NAMES = {W.FP8_E4M3: "fp8_g128", W.INT8_PER_TOKEN: "int8_tok", W.FP8_E4M3_PER_TOKEN: "fp8_tok",
         W.MXFP8_E4M3: "mx_e4m3", W.MXFP8_E5M2: "mx_e5m2", W.MXFP4_E2M1: "mx_e2m1"}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _buffers(dt, rows, H, fill_code=0xAB, fill_scale=0x5A):
    """Device code / scale buffers in the layout of format dt, pre-filled
    with a sentinel so untouched rows can be recognised."""
    cb = oracle.row_code_bytes(dt, H)
    codes = torch.full((rows, cb), fill_code, dtype=torch.uint8, device="cuda")
    sb = oracle.row_scale_bytes(dt, H)
    scales = torch.full((rows, sb), fill_scale, dtype=torch.uint8, device="cuda")
    return codes, scales


def _host_bytes(ref, dt, rows, H):
    """Oracle outputs as byte matrices [rows, code bytes] / [rows, scale bytes]."""
    codes = np.ascontiguousarray(ref["recv"]).view(np.uint8).reshape(rows, -1)
    scales = np.ascontiguousarray(ref["recv_scales"]).view(np.uint8).reshape(rows, -1)
    return codes, scales


def _run(x, idx, E, R, dt, mode=W.COMPACT, mt=0, w=None, extra=False):
    T, H = x.shape
    ref_l = oracle.tc_layout(idx, E, R)
    rows = E * mt if mode == W.PADDED else int(ref_l["expert_offsets"][-1])
    want_w = extra and w is not None
    ref = oracle.tc_dispatch(x, idx, E, ref_l, mode=mode, max_tokens=mt, out_dtype=dt, topk_weights=w,
                             want_src=extra, want_weights=want_w)
    idx_d = to_dev(np.ascontiguousarray(idx, np.int64))
    routing = B.Routing.topk(idx_d, E, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    codes, scales = _buffers(dt, rows, H)
    src = torch.full((rows,), -1, dtype=torch.int32, device="cuda") if extra else None
    rw = torch.zeros(rows, dtype=torch.float32, device="cuda") if want_w else None
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, codes, mode=mode, max_tokens_per_expert=mt,
                  topk_weights=None if w is None else to_dev(w), recv_scales=scales, recv_src=src,
                  recv_weights=rw, out_dtype=dt)
    flags = B.ep_get_device_error(lay)
    return ref, ref_l, host(codes), host(scales), flags, (host(src) if extra else None), (host(rw) if want_w else None)


def _valid_rows(ref_l, E, mt, mode):
    counts = ref_l["num_tokens_per_expert"]
    if mode == W.COMPACT:
        return np.ones(int(ref_l["expert_offsets"][-1]), bool)
    valid = np.zeros(E * mt, bool)
    for e in range(E):
        valid[e * mt:e * mt + min(int(counts[e]), mt)] = True
    return valid


@pytest.mark.parametrize("dt", QUANT, ids=lambda d: NAMES[d])
def test_quant_dispatch_decode_padded(dt):
    """Decode workload (128 x 7168, 256 experts in 8 ranks, top-8) into the
    padded per-expert buffers of 128 rows."""
    inp = W.make_inputs(3)
    c = inp["cfg"]
    E, R, mt, H = c["E"], c["R"], c["max_tokens"], c["H"]
    ref, ref_l, gc, gs, flags, _, _ = _run(inp["x"], inp["topk_idx"], E, R, dt, mode=W.PADDED, mt=mt)
    assert flags == 0
    rc, rs = _host_bytes(ref, dt, E * mt, H)
    valid = _valid_rows(ref_l, E, mt, W.PADDED)
    assert np.array_equal(gc[valid], rc[valid]) and np.array_equal(gs[valid], rs[valid])
    assert (gc[~valid] == 0xAB).all() and (gs[~valid] == 0x5A).all()  # padding rows untouched


@pytest.mark.parametrize("dt", QUANT, ids=lambda d: NAMES[d])
def test_quant_dispatch_prefill_compact(dt):
    """Prefill-shaped routing (hidden 7168, 256 experts, top-8), 384 tokens,
    compact buffers, with recv_src / recv_weights."""
    inp = W.make_inputs(2, T=384)
    c = inp["cfg"]
    ref, ref_l, gc, gs, flags, src, rw = _run(inp["x"], inp["topk_idx"], c["E"], c["R"], dt,
                                              w=inp["topk_weights"], extra=True)
    assert flags == 0
    rows = int(ref_l["expert_offsets"][-1])
    rc, rs = _host_bytes(ref, dt, rows, c["H"])
    assert np.array_equal(gc, rc) and np.array_equal(gs, rs)
    assert np.array_equal(src, ref["recv_src"]) and np.array_equal(rw, ref["recv_weights"])


@pytest.mark.parametrize("dt", QUANT, ids=lambda d: NAMES[d])
def test_quant_dispatch_full_prefill_sampled(dt):
    """The full prefill workload (4096 tokens, hidden 7168, 256 experts,
    top-8, compact) in the call the benchmark times: for a seeded sample of
    tokens, every destination row the oracle's layout names holds the
    oracle's codes and scales of that token, bit for bit (a token's codes
    depend on its own row only, so the oracle encodes the sample alone)."""
    inp = W.make_inputs(2)
    c = inp["cfg"]
    T, H, E, R = c["T"], c["H"], c["E"], c["R"]
    x, idx = inp["x"], inp["topk_idx"]
    ref_l = oracle.tc_layout(idx, E, R)
    rows = int(ref_l["expert_offsets"][-1])
    idx_d = to_dev(np.ascontiguousarray(idx, np.int64))
    routing = B.Routing.topk(idx_d, E, R)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    codes, scales = _buffers(dt, rows, H)
    B.ep_dispatch(to_dev(x, bf16=True), routing, lay, codes, recv_scales=scales, out_dtype=dt)
    assert B.ep_get_device_error(lay) == 0
    sample = np.sort(_rng(2024).choice(T, size=48, replace=False))
    one = np.zeros((len(sample), 1), np.int64)  # every sampled token to one expert, in sample order
    ref = oracle.tc_dispatch(x[sample], one, 1, oracle.tc_layout(one, 1, 1), out_dtype=dt)
    rc, rs = _host_bytes(ref, dt, len(sample), H)
    want_rows, want_i = [], []
    for i, t in enumerate(sample):
        for k in range(idx.shape[1]):
            e = int(idx[t, k])
            if e >= 0:
                want_rows.append(int(ref_l["expert_offsets"][e]) + int(ref_l["slot"][t, k]))
                want_i.append(i)
    sel = torch.tensor(want_rows, dtype=torch.int64, device="cuda")
    gc, gs = host(codes[sel]), host(scales[sel])
    assert np.array_equal(gc, rc[want_i]) and np.array_equal(gs, rs[want_i])


@pytest.mark.parametrize("dt", QUANT, ids=lambda d: NAMES[d])
@pytest.mark.parametrize("H", [128, 4224, 32768])
def test_quant_dispatch_ragged_hidden_and_magnitudes(dt, H):
    """Row widths that leave threads idle (4224 = 528 vectors) or fill the
    largest register tile (32768); every 32-channel block at its own
    magnitude in 2^-60 .. 2^60, plus zero blocks, -0, bf16 subnormals and
    values near the bf16 maximum."""
    r = _rng(300 + dt)
    T = 40 if H < 32768 else 8
    nb = H // 32
    mag = np.float32(2.0) ** r.integers(-60, 60, size=(T, nb, 1)).astype(np.float32)
    xf = (r.standard_normal((T, nb, 32)).astype(np.float32) * mag).reshape(T, H)
    xf[0, :] = 0.0  # all-zero token, with negative zeros
    xf[0, 1::3] = -0.0
    xf[1, 32:64] = 0.0  # zero block
    xf[6, H - 128:] = -0.0  # a 128-channel group of negative zeros
    xf[2, 7] = -0.0
    xf[3, :] = r.standard_normal(H).astype(np.float32) * np.float32(1e-39)  # bf16 subnormals
    xf[4, :64] = np.float32(3.3e38) * np.sign(r.standard_normal(64)).astype(np.float32)
    xf[5, :] *= np.float32(1e-36)  # tiny amax: qmax/amax is clamped to FLT_MAX
    x = W.to_bf16_bits(xf)
    E = 4
    idx = (np.arange(T, dtype=np.int64) % E).reshape(T, 1)
    ref, ref_l, gc, gs, flags, src, _ = _run(x, idx, E, 2, dt, extra=True)
    assert flags == 0
    rc, rs = _host_bytes(ref, dt, T, H)
    bad = np.nonzero((gc != rc).any(axis=1) | (gs != rs).any(axis=1))[0]
    detail = []
    for row in bad[:3]:
        t = int(src[row])
        for c in np.nonzero(gc[row] != rc[row])[0][:4]:
            ch = c if dt != W.MXFP4_E2M1 else 2 * c
            detail.append("token %d byte %d: x=%r got %#x want %#x" % (t, c, float(xf[t, ch]), gc[row, c],
                                                                      rc[row, c]))
    assert bad.size == 0, "rows differing from the oracle: %s %s" % (bad[:10].tolist(), detail)


@pytest.mark.parametrize("dt", QUANT, ids=lambda d: NAMES[d])
def test_quant_dispatch_edges(dt):
    """Padded overflow (flagged, skipped), duplicate experts in a row, -1,
    bad ids (flagged), K > 32, H = 384."""
    r = _rng(400 + dt)
    T, E, R, K, H, mt = 45, 12, 3, 36, 384, 5
    idx = W.random_topk(r, T, E, K, p_neg=0.2, allow_dup=True, p_bad=0.02)
    xf = r.standard_normal((T, H)).astype(np.float32) * np.float32(3.0)
    x = W.to_bf16_bits(xf)
    w = r.random((T, K)).astype(np.float32)
    for mode, m in ((W.PADDED, mt), (W.COMPACT, 0)):
        ref, ref_l, gc, gs, flags, src, rw = _run(x, idx, E, R, dt, mode=mode, mt=m, w=w, extra=True)
        assert flags & B.EP_DEVERR_BAD_INDEX
        assert bool(flags & B.EP_DEVERR_OVERFLOW) == (ref["overflow_count"] > 0)
        rows = E * m if mode == W.PADDED else int(ref_l["expert_offsets"][-1])
        rc, rs = _host_bytes(ref, dt, rows, H)
        valid = _valid_rows(ref_l, E, m, mode)
        assert np.array_equal(gc[valid], rc[valid]) and np.array_equal(gs[valid], rs[valid])
        assert np.array_equal(src, ref["recv_src"]) and np.array_equal(rw, ref["recv_weights"])


def test_quant_dispatch_rejects_bad_shapes():
    """Host-side checks: MX needs H % 32 == 0, rows wider than 32768
    channels are unsupported, fp32 scales must be 4-byte aligned."""
    idx = to_dev(np.zeros((4, 1), np.int64))
    routing = B.Routing.topk(idx, 4, 1)
    lay = B.Layout(routing)
    B.ep_get_layout(routing, lay)
    codes = torch.zeros((4, 32776), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(4 * 4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.EPError) as ei:  # 40 channels: not a whole MX block
        B.ep_dispatch(torch.zeros((4, 40), dtype=torch.bfloat16, device="cuda"), routing, lay, codes,
                      recv_scales=sc, out_dtype=W.MXFP8_E4M3)
    assert ei.value.status == 1
    with pytest.raises(B.EPError) as ei:  # wider than the register-resident row
        B.ep_dispatch(torch.zeros((4, 32776), dtype=torch.bfloat16, device="cuda"), routing, lay, codes,
                      recv_scales=sc, out_dtype=W.INT8_PER_TOKEN)
    assert ei.value.status == 6
    with pytest.raises(B.EPError) as ei:  # fp32 scales one byte off alignment
        B.ep_dispatch(torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda"), routing, lay, codes,
                      recv_scales=sc[1:], out_dtype=W.FP8_E4M3_PER_TOKEN)
    assert ei.value.status == 1


def _codec_sweep_rows(H=7168):
    """bf16 rows for an exhaustive codec check: groups of 128 channels that
    hold one amax value and 127 others bounded by it, such that every finite
    bf16 value of magnitude <= amax appears (both signs) under every amax of
    the sweep (each exponent field 0..254, subnormal amax included, positive
    and negative amax).  2^24 values and more; padded with zero groups."""
    mags = np.arange(0x7F80, dtype=np.uint16)  # finite magnitudes, as bits
    groups = []
    for e in range(255):
        m = (e * 37 + 1) % 128 or 1
        amax = np.uint16((e << 7) | m)
        for sign in (0, 0x8000):
            vals = mags[mags <= amax]
            vals = np.concatenate([vals, vals | 0x8000]).astype(np.uint16)
            ng = (len(vals) + 126) // 127
            vals = np.concatenate([vals, np.zeros(ng * 127 - len(vals), np.uint16)]).reshape(ng, 127)
            g = np.empty((ng, 128), np.uint16)
            g[:, 0] = amax | sign
            g[:, 1:] = vals
            groups.append(g)
    g = np.concatenate(groups)
    n_values = g.size
    per = H // 128
    T = (g.shape[0] + per - 1) // per
    g = np.concatenate([g, np.zeros((T * per - g.shape[0], 128), np.uint16)])
    return g.reshape(T, H), n_values


@pytest.mark.parametrize("dt", [W.FP8_E4M3, W.MXFP8_E4M3, W.MXFP8_E5M2, W.MXFP4_E2M1], ids=lambda d: NAMES[d])
def test_codec_every_bf16_under_a_sweep_of_scales(dt):
    """The device conversion against the oracle codec on more than 2^24
    values: every finite bf16 input under every exponent of the group amax,
    codes and scales bit for bit (the 128-channel FP8 scale reaches the fp32
    overflow of 448 / amax for subnormal amax)."""
    x, n_values = _codec_sweep_rows()
    assert n_values >= 1 << 24
    T = x.shape[0]
    idx = (np.arange(T, dtype=np.int64) % 4).reshape(T, 1)
    ref, _, g_codes, g_scales, flags, _, _ = _run(x, idx, 4, 1, dt)
    assert flags == 0
    r_codes, r_scales = _host_bytes(ref, dt, T, x.shape[1])
    bad = np.argwhere(g_codes != r_codes)
    assert bad.size == 0, ("codes differ", bad[:5], g_codes[tuple(bad[0])], r_codes[tuple(bad[0])])
    assert np.array_equal(g_scales, r_scales), "scales differ"
