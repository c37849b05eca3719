"""Canary bytes around every output buffer: each output is a view into a
larger buffer whose guard regions (before and after) hold a known pattern.
After layout, dispatch (bf16, FP8 padded, MXFP4, per rank), combine and the
expert-choice calls, the guards must be untouched -- no kernel writes
outside the rows it owns, on shapes with ragged tails and overflowing
padded buffers."""
import numpy as np
import pytest
import torch

from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()


class Guarded:
    """A device tensor of `shape`/`dtype` with GUARD canary bytes on both sides."""

    def __init__(self, shape, dtype, fill=0):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), 0xC5, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape) if n else torch.empty(shape, dtype=dtype,
                                                                                        device="cuda")
        if n:
            self.t.fill_(fill)

    def intact(self):
        h = self.raw.cpu().numpy()
        return bool((h[:GUARD] == 0xC5).all() and (h[len(h) - GUARD:] == 0xC5).all())


def _check(*bufs):
    for i, b in enumerate(bufs):
        if b is not None:
            assert b.intact(), "guard bytes of buffer %d overwritten" % i


def test_token_choice_outputs_stay_in_bounds():
    r = np.random.Generator(np.random.PCG64(5))
    T, E, R, K, H, mt = 300, 24, 4, 6, 520, 7  # ragged H, padded overflow
    idx = W.random_topk(r, T, E, K, p_neg=0.2, allow_dup=True, p_bad=0.01)
    x = to_dev(W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32)), bf16=True)
    w = to_dev(r.random((T, K)).astype(np.float32))
    routing = B.Routing.topk(to_dev(idx), E, R)
    lay = B.Layout(routing)
    g = dict(cnt=Guarded((E,), torch.int32), off=Guarded((E + 1,), torch.int32), rc=Guarded((R,), torch.int32),
             inr=Guarded((T, R), torch.uint8), slot=Guarded((T, K), torch.int32))
    lay.num_tokens_per_expert, lay.expert_offsets = g["cnt"].t, g["off"].t
    lay.num_tokens_per_rank, lay.is_token_in_rank, lay.slot = g["rc"].t, g["inr"].t, g["slot"].t
    lay.desc.num_tokens_per_expert = g["cnt"].t.data_ptr()
    lay.desc.expert_offsets = g["off"].t.data_ptr()
    lay.desc.num_tokens_per_rank = g["rc"].t.data_ptr()
    lay.desc.is_token_in_rank = g["inr"].t.data_ptr()
    lay.desc.slot = g["slot"].t.data_ptr()
    B.ep_get_layout(routing, lay)
    _check(*g.values())
    n = int(lay.expert_offsets[-1].item())
    recv = Guarded((n, H), torch.bfloat16)
    src = Guarded((n,), torch.int32)
    rw = Guarded((n,), torch.float32)
    B.ep_dispatch(x, routing, lay, recv.t, topk_weights=w, recv_src=src.t, recv_weights=rw.t)
    _check(recv, src, rw)
    # padded FP8 and MXFP4 with overflowing experts (mt = 7)
    H4 = 512
    x4 = to_dev(W.to_bf16_bits(r.standard_normal((T, H4)).astype(np.float32)), bf16=True)
    q8 = Guarded((E * mt, H4), torch.uint8)
    s8 = Guarded((E * mt, H4 // 128), torch.float32)
    B.ep_dispatch(x4, routing, lay, q8.t, mode=B.EP_LAYOUT_PADDED, max_tokens_per_expert=mt, recv_scales=s8.t)
    q4 = Guarded((E * mt, H4 // 2), torch.uint8)
    s4 = Guarded((E * mt, H4 // 32), torch.uint8)
    B.ep_dispatch(x4, routing, lay, q4.t, mode=B.EP_LAYOUT_PADDED, max_tokens_per_expert=mt, recv_scales=s4.t,
                  out_dtype=B.EP_MXFP4_E2M1)
    _check(q8, s8, q4, s4)
    for dt in (torch.float32, torch.bfloat16):
        out = Guarded((T, H), dt)
        B.ep_combine(recv.t, routing, lay, w, out.t)
        _check(out)
    # per rank
    rl = B.RankLayout(routing)
    ro, rr = Guarded((R + 1,), torch.int32), Guarded((T, R), torch.int32)
    rl.rank_offsets, rl.rank_row = ro.t, rr.t
    rl.desc.rank_offsets, rl.desc.rank_row = ro.t.data_ptr(), rr.t.data_ptr()
    B.ep_get_rank_layout(routing, lay, rl)
    _check(ro, rr)
    nr = int(rl.rank_offsets[-1].item())
    rrecv = Guarded((nr, H), torch.bfloat16)
    ridx = Guarded((nr, K), torch.int64)
    rwt = Guarded((nr, K), torch.float32)
    B.ep_dispatch_ranks(x, routing, lay, rl, rrecv.t, topk_weights=w, recv_topk_idx=ridx.t, recv_topk_weights=rwt.t)
    rout = Guarded((T, H), torch.bfloat16)
    B.ep_combine_ranks(rrecv.t, routing, lay, rl, rout.t)
    _check(rrecv, ridx, rwt, rout)
    flags = B.ep_get_device_error(lay)
    assert flags & B.EP_DEVERR_BAD_INDEX and flags & B.EP_DEVERR_OVERFLOW


def test_expert_choice_outputs_stay_in_bounds():
    r = np.random.Generator(np.random.PCG64(6))
    T, E, C, R, H = 700, 12, 40, 3, 264
    ti = W.random_token_indices(r, T, E, C, p_neg=0.1)
    routing = B.Routing.expert_choice(to_dev(ti), T, R)
    lay = B.Layout(routing)
    g = dict(cnt=Guarded((E,), torch.int32), rc=Guarded((R,), torch.int32), inr=Guarded((T, R), torch.uint8),
             toff=Guarded((T + 1,), torch.int32), tsl=Guarded((E * C,), torch.int32))
    lay.desc.num_tokens_per_expert = g["cnt"].t.data_ptr()
    lay.desc.num_tokens_per_rank = g["rc"].t.data_ptr()
    lay.desc.is_token_in_rank = g["inr"].t.data_ptr()
    lay.desc.token_offsets = g["toff"].t.data_ptr()
    lay.desc.token_slots = g["tsl"].t.data_ptr()
    B.ep_get_layout(routing, lay)
    _check(*g.values())
    x = to_dev(W.to_bf16_bits(r.standard_normal((T, H)).astype(np.float32)), bf16=True)
    recv = Guarded((E * C, H), torch.bfloat16)
    B.ep_dispatch_expert_choice(x, routing, lay, recv.t)
    ew = to_dev(r.standard_normal((E, C)).astype(np.float32))
    out = Guarded((T, H), torch.bfloat16)
    B.ep_combine_expert_choice(recv.t, routing, lay, ew, out.t)
    _check(recv, out)
    assert B.ep_get_device_error(lay) == 0
