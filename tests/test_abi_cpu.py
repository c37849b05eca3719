"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/ep.h declares, and rejects bad arguments on the host before it
touches CUDA (no compute call runs here)."""
import ctypes
import os
import re

import pytest

from combine_ep_get_10_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from combine_ep_get_10_b200 import build

    build.build()
    return B.lib()


def declared_entry_points():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ("ep_get_layout", "ep_dispatch", "ep_combine", "ep_dispatch_expert_choice",
                     "ep_combine_expert_choice"):
        assert required in names
    assert set(B.EXPORTED) <= set(names)


def test_every_declared_symbol_is_exported(L):
    for name in declared_entry_points():
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    assert B.ep_version() == B.EP_ABI_VERSION == 3
    # ep_layout_t: nine pointer-sized fields, then num_valid_host (version 2)
    assert ctypes.sizeof(B.LayoutDesc) == 10 * 8
    assert B.LayoutDesc.num_valid_host.offset == 9 * 8
    # ep_peers_t (version 3): two int32, the int64 capacity, six tables
    assert ctypes.sizeof(B.PeersDesc) == 8 + 8 + 6 * 8
    assert B.PeersDesc.capacity.offset == 8 and B.PeersDesc.rank_counts.offset == 8 + 8 + 5 * 8
    for s in range(8):
        assert B.ep_status_string(s)
    assert B.ep_status_string(99) == "unknown status"


def _topk_desc(T=16, K=2, E=8, R=2, ptr=0x1000):
    return B.RoutingDesc(B.EP_ROUTING_TOPK, ptr, None, T, K, 0, E, R)


def _ec_desc(T=16, E=8, C=4, R=2, ptr=0x1000):
    return B.RoutingDesc(B.EP_ROUTING_EXPERT_CHOICE, None, ptr, T, 0, C, E, R)


def test_workspace_bytes(L):
    n_tc = L.ep_workspace_bytes(ctypes.byref(_topk_desc(E=8)))
    assert n_tc >= 256 + 4 * 64 * (8 + 32) and n_tc % 256 == 0
    n = L.ep_workspace_bytes(ctypes.byref(_ec_desc(T=1000, E=128, C=128)))
    assert n >= 256 + 4 * (2 * 1000 + 128 * 128) and n % 256 == 0
    assert L.ep_workspace_bytes(ctypes.byref(_topk_desc(E=9, R=2))) == 0  # E % R != 0
    assert L.ep_workspace_bytes(None) == 0


@pytest.mark.parametrize("desc", [
    _topk_desc(E=9, R=2), _topk_desc(R=0), _topk_desc(R=33, E=66), _topk_desc(K=0), _topk_desc(T=-1),
    _topk_desc(ptr=0), _topk_desc(ptr=0x1004), _topk_desc(T=1 << 28, K=8), _ec_desc(C=0), _ec_desc(ptr=0),
    _ec_desc(E=1 << 16, C=1 << 16, R=1), B.RoutingDesc(7, 0x1000, 0x1000, 4, 2, 2, 4, 1)])
def test_layout_rejects_bad_routing(L, desc):
    lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x100000, 1 << 20)
    assert L.ep_get_layout(ctypes.byref(desc), ctypes.byref(lay), None) == 1


def test_layout_rejects_bad_workspace(L):
    d = _topk_desc()
    for ws, n in [(0, 1 << 20), (0x100010, 1 << 20), (0x100000, 255)]:
        lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, ws, n)
        assert L.ep_get_layout(ctypes.byref(d), ctypes.byref(lay), None) == 4
    ec = _ec_desc(T=100, E=8, C=4)
    lay = B.LayoutDesc(0x1000, None, 0x1000, 0x1000, None, 0x1000, 0x1000, 0x100000, 512)
    assert L.ep_get_layout(ctypes.byref(ec), ctypes.byref(lay), None) == 4


def test_layout_unsupported_expert_count(L):
    d = _topk_desc(E=2048, R=1)
    lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 1 << 20)
    assert L.ep_get_layout(ctypes.byref(d), ctypes.byref(lay), None) == 6


def test_dispatch_and_combine_reject_bad_args(L):
    d = _topk_desc()
    lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 256)
    ok = dict(x=0x2000, hidden=256, mode=0, mt=0, rows=32, dt=B.EP_BF16, w=0x3000, recv=0x4000, sc=None)

    def disp(**kw):
        a = dict(ok, **kw)
        return L.ep_dispatch(a["x"], a["hidden"], ctypes.byref(d), ctypes.byref(lay), a["mode"], a["mt"], a["rows"],
                             a["dt"], a["w"], a["recv"], a["sc"], None, None, None)

    assert disp(hidden=12) == 1  # not a multiple of 8
    assert disp(x=0x2008) == 1  # x not 16-byte aligned
    assert disp(recv=0x4004) == 1
    assert disp(mode=5) == 1
    assert disp(mode=1, mt=0) == 1  # padded needs max_tokens >= 1
    assert disp(dt=B.EP_FP32) == 1  # dispatch writes bf16 or fp8
    assert disp(dt=B.EP_FP8_E4M3, hidden=136) == 1  # fp8 needs H % 128 == 0
    assert disp(dt=B.EP_FP8_E4M3, sc=None) == 1  # fp8 needs scales
    assert disp(rows=-1) == 1
    assert disp(dt=8) == 1  # no such format
    assert disp(dt=B.EP_MXFP8_E4M3, hidden=264, sc=0x6000) == 1  # MX needs H % 32 == 0
    assert disp(dt=B.EP_MXFP4_E2M1, hidden=256, sc=None) == 1  # scales required
    assert disp(dt=B.EP_INT8_PER_TOKEN, hidden=256, sc=0x6002) == 1  # fp32 scales misaligned
    assert disp(dt=B.EP_FP8_E4M3_PER_TOKEN, hidden=32776, sc=0x6000) == 6  # row wider than 32768
    assert disp(dt=B.EP_MXFP8_E5M2, hidden=32800, sc=0x6001) == 6
    assert L.ep_combine(0x2000, 256, 32, ctypes.byref(d), ctypes.byref(lay), 0, 0, None, 0x5000, B.EP_BF16,
                        None) == 1  # weights missing
    assert L.ep_combine(0x2000, 256, 32, ctypes.byref(d), ctypes.byref(lay), 0, 0, 0x3000, 0x5000, B.EP_FP8_E4M3,
                        None) == 1  # combine writes bf16 or fp32
    ec = _ec_desc()
    assert L.ep_dispatch(0x2000, 256, ctypes.byref(ec), ctypes.byref(lay), 0, 0, 32, 0, None, 0x4000, None, None,
                         None, None) == 1  # token-choice call with expert-choice routing
    assert L.ep_dispatch_expert_choice(0x2000, 256, ctypes.byref(d), ctypes.byref(lay), 0x4000, None) == 1
    assert L.ep_combine_expert_choice(0x2000, 256, ctypes.byref(ec), ctypes.byref(lay), None, 0x5000, 0, None) == 1


def test_low_latency_dispatch_rejects_bad_args(L):
    d = _topk_desc()
    ws = L.ep_workspace_bytes(ctypes.byref(d))
    lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, ws)

    def ll(desc=d, layout=lay, hidden=256, mt=4, dt=B.EP_BF16, x=0x2000, recv=0x4000, sc=None):
        return L.ep_dispatch_low_latency(x, hidden, ctypes.byref(desc), ctypes.byref(layout), mt, dt, None, recv,
                                         sc, None, None, None)

    assert ll(mt=0) == 1  # padded rows need max_tokens >= 1
    assert ll(desc=_ec_desc()) == 1  # token choice only
    assert ll(hidden=12) == 1
    assert ll(dt=B.EP_FP32) == 1
    assert ll(dt=B.EP_MXFP8_E4M3, sc=None) == 1  # scales required
    assert ll(x=0x2008) == 1
    small = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 256)
    assert ll(layout=small) == 4  # needs the full layout workspace (the two-call path may run)
    assert ll(desc=_topk_desc(E=2048, R=1), layout=B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None,
                                                                  0x100000, 1 << 24)) == 6


def test_device_error_rejects_missing_workspace(L):
    lay = B.LayoutDesc(None, None, None, None, None, None, None, None, 0)
    flags = ctypes.c_uint32(0)
    assert L.ep_get_device_error(ctypes.byref(lay), ctypes.byref(flags), 1, None) == 4


def test_token_rounds_cover_the_batch_in_order():
    assert B.token_rounds(0, 8) == []
    assert B.token_rounds(10, 4) == [(0, 4), (4, 8), (8, 10)]
    assert B.token_rounds(8192, 8192) == [(0, 8192)]
    r = B.token_rounds(131072, 8192)
    assert len(r) == 16 and r[0] == (0, 8192) and r[-1] == (122880, 131072)
    assert all(b0 == a1 for (_, a1), (b0, _) in zip(r, r[1:]))
    with pytest.raises(ValueError):
        B.token_rounds(10, 0)


def test_layout_dispatch_checks_both_calls_before_launching(L):
    """ep_layout_dispatch rejects what either ep_dispatch or ep_get_layout
    would reject, before anything is launched (no GPU here)."""
    desc = _topk_desc()
    good_ws = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 1 << 20)
    call = lambda lay, hidden=256, x=0x2000: L.ep_layout_dispatch(  # noqa: E731
        x, hidden, ctypes.byref(desc), ctypes.byref(lay), 0, 0, 32, 0, None, 0x4000, None, None, None, None)
    assert call(good_ws, hidden=12) == 1  # hidden not a multiple of 8
    assert call(good_ws, x=0x2008) == 1  # x not 16-byte aligned
    small = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 256)
    assert call(small) == 4  # the layout needs its whole workspace
    no_counts = B.LayoutDesc(None, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 1 << 20)
    assert call(no_counts) == 1


def test_binding_constants_match_the_header():
    """Every enum value and device-error bit of include/ep.h has the same value
    in the binding (the binding marshals them as plain ints)."""
    here = os.path.dirname(os.path.abspath(__file__))
    text = open(os.path.join(here, "..", "include", "ep.h")).read()
    values = {m.group(1): int(m.group(2), 0) for m in re.finditer(r"\b(EP_[A-Z0-9_]+) = (\d+)\b", text)}
    values["EP_ABI_VERSION"] = int(re.search(r"#define EP_ABI_VERSION (\d+)", text).group(1))
    values.update({m.group(1): int(m.group(2), 16) for m in
                   re.finditer(r"#define (EP_DEVERR_[A-Z_]+) 0x([0-9a-fA-F]+)u", text)})
    assert len(values) >= 22, sorted(values)
    for name, v in values.items():
        assert getattr(B, name) == v, name
    for v, name in B.STATUS_NAMES.items():
        assert values[name] == v


def test_peer_calls_reject_bad_args(L):
    """The peer-memory calls check routing, layout, rank layout and tables on
    the host before anything is launched or allocated (no GPU here)."""
    d = _topk_desc(R=2)
    lay = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 256)
    rl = B.RankLayoutDesc(0x7000, 0x7100)

    def peers(**kw):
        f = dict(num_ranks=2, rank=0, capacity=64, recv_x=0x8000, recv_topk_idx=None, recv_topk_weights=None,
                 recv_src=None, y=0x8100, rank_counts=0x8200)
        f.update(kw)
        return B.PeersDesc(*(f[n] for n, _ in B.PeersDesc._fields_))

    def disp(p, x=0x2000, hidden=256, w=None, routing=d):
        return L.ep_dispatch_peers(x, hidden, ctypes.byref(routing), ctypes.byref(lay), ctypes.byref(rl), w,
                                   ctypes.byref(p), None)

    def comb(p, hidden=256, out=0x5000, dt=B.EP_BF16):
        return L.ep_combine_peers(hidden, ctypes.byref(d), ctypes.byref(lay), ctypes.byref(rl), ctypes.byref(p),
                                  out, dt, None)

    def publish(p, layout=lay):
        return L.ep_peer_publish_counts(ctypes.byref(d), ctypes.byref(layout), ctypes.byref(p), None)

    bad = [peers(num_ranks=4), peers(rank=2), peers(rank=-1), peers(capacity=-1), peers(recv_x=None),
           peers(y=None), peers(rank_counts=None), peers(recv_x=0x8004), peers(recv_src=0x8304)]
    for p in bad:
        assert disp(p) == 1 and comb(p) == 1 and publish(p) == 1
    assert L.ep_dispatch_peers(0x2000, 256, ctypes.byref(d), ctypes.byref(lay), ctypes.byref(rl), None, None,
                               None) == 1  # no tables
    assert disp(peers(), hidden=12) == 1
    assert disp(peers(), x=0x2008) == 1
    assert disp(peers(recv_topk_weights=0x8400)) == 1  # weights asked for, topk_weights missing
    assert disp(peers(), routing=_ec_desc()) == 1  # token-choice routing only
    assert comb(peers(), dt=B.EP_FP8_E4M3) == 1
    assert comb(peers(), out=0x5008) == 1
    no_rank_row = B.RankLayoutDesc(0x7000, None)
    assert L.ep_combine_peers(256, ctypes.byref(d), ctypes.byref(lay), ctypes.byref(no_rank_row),
                              ctypes.byref(peers()), 0x5000, 0, None) == 1
    no_counts = B.LayoutDesc(0x1000, 0x1000, None, 0x1000, 0x1000, None, None, 0x100000, 256)
    assert publish(peers(), layout=no_counts) == 1
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(B.EP_IPC_HANDLE_BYTES)
    assert L.ep_peer_alloc(0, ctypes.byref(ptr), handle) == 1
    assert L.ep_peer_alloc(256, None, handle) == 1
    assert L.ep_peer_alloc(256, ctypes.byref(ptr), None) == 1
    assert L.ep_peer_open(None, ctypes.byref(ptr)) == 1
    assert L.ep_peer_open(handle, None) == 1
    assert L.ep_peer_close(None) == 1 and L.ep_peer_free(None) == 1


def test_layout_dispatch_expert_choice_checks_both_calls_before_launching(L):
    """ep_layout_dispatch_expert_choice rejects what either
    ep_dispatch_expert_choice or ep_get_layout would reject, before anything
    is launched (no GPU here)."""
    ec = _ec_desc()
    ws = L.ep_workspace_bytes(ctypes.byref(ec))
    good = B.LayoutDesc(0x1000, None, 0x1000, 0x1000, None, 0x1000, 0x1000, 0x100000, ws)
    call = lambda lay, routing=ec, hidden=256, x=0x2000, recv=0x4000: L.ep_layout_dispatch_expert_choice(  # noqa: E731
        x, hidden, ctypes.byref(routing), ctypes.byref(lay), recv, None)
    assert call(good, routing=_topk_desc()) == 1  # token-choice routing
    assert call(good, hidden=12) == 1
    assert call(good, x=0x2008) == 1
    assert call(good, recv=None) == 1
    small = B.LayoutDesc(0x1000, None, 0x1000, 0x1000, None, 0x1000, 0x1000, 0x100000, 256)
    assert call(small) == 4  # the layout needs its whole workspace
    no_csr = B.LayoutDesc(0x1000, None, 0x1000, 0x1000, None, None, 0x1000, 0x100000, ws)
    assert call(no_csr) == 1


def test_layout_dispatch_ranks_checks_every_call_before_launching(L):
    """ep_layout_dispatch_ranks rejects what ep_get_layout, ep_get_rank_layout
    or ep_dispatch_ranks would reject, before anything is launched."""
    d = _topk_desc()
    ws = L.ep_workspace_bytes(ctypes.byref(d))
    good = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, ws)
    rl = B.RankLayoutDesc(0x7000, 0x7100)
    call = lambda lay, hidden=256, x=0x2000, rank_layout=rl, routing=d: L.ep_layout_dispatch_ranks(  # noqa: E731
        x, hidden, ctypes.byref(routing), ctypes.byref(lay), ctypes.byref(rank_layout), 32, None, 0x4000, None, None,
        None, None)
    assert call(good, hidden=12) == 1
    assert call(good, x=0x2008) == 1
    assert call(good, routing=_ec_desc()) == 1
    assert call(good, rank_layout=B.RankLayoutDesc(None, 0x7100)) == 1
    small = B.LayoutDesc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, None, None, 0x100000, 256)
    assert call(small) == 4  # the layout needs its whole workspace
    no_in_rank = B.LayoutDesc(0x1000, 0x1000, 0x1000, None, 0x1000, None, None, 0x100000, ws)
    assert call(no_in_rank) == 1
