"""ep_get_layout_no_alloc: the layout entry point for callers that cannot
allocate device memory (plugins handed only their tensors, latency-critical
decode loops where an allocation could stall the step).  It must write exactly what ep_get_layout writes;
here both are called through the C ABI on the same routing and compared
(integer outputs: bit for bit), twice in a row so that a second call over the
shared scratch array left by the first is covered too.

This file is collected last on purpose: it runs after every other test when
the whole suite runs, and it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _outputs(layout):
    names = ("num_tokens_per_expert", "expert_offsets", "num_tokens_per_rank", "is_token_in_rank", "slot",
             "token_offsets")
    out = {n: getattr(layout, n).cpu().numpy() for n in names if getattr(layout, n) is not None}
    if layout.token_slots is not None:
        n = int(out["token_offsets"][-1])
        out["token_slots"] = layout.token_slots.cpu().numpy()[:n]
    return out


def _compare(routing):
    ref = B.Layout(routing)
    B.ep_get_layout(routing, ref)
    ref_flags = B.ep_get_device_error(ref)
    want = _outputs(ref)
    for call in range(2):
        lay = B.Layout(routing)  # outputs only; its workspace is not used by this entry point
        for t in (lay.num_tokens_per_expert, lay.num_tokens_per_rank, lay.slot, lay.token_offsets,
                  lay.token_slots, lay.expert_offsets):
            if t is not None:
                t.fill_(-7)
        flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        st = B.lib().ep_get_layout_no_alloc(ctypes.byref(routing.desc), ctypes.byref(lay.desc),
                                            ctypes.c_void_p(flags.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == B.EP_OK, B.ep_status_string(st)
        torch.cuda.synchronize()
        got = _outputs(lay)
        assert got.keys() == want.keys()
        for k in want:
            assert np.array_equal(got[k], want[k]), (call, k)
        assert int(flags.item()) == ref_flags, call


def test_no_alloc_matches_layout_token_choice():
    inp = W.make_inputs(2)  # 32768 pairs: the 16-CTA cluster layout
    _compare(B.Routing.topk(_dev(inp["topk_idx"]), 256, 8))
    inp = W.make_inputs(5)  # 131072 pairs: the grid-wide layout (its barrier words in the scratch array)
    _compare(B.Routing.topk(_dev(inp["topk_idx"]), 256, 8))
    rng = np.random.Generator(np.random.PCG64(3))
    idx = W.random_topk(rng, 300, 24, 5, p_neg=0.2, allow_dup=True, p_bad=0.05)
    _compare(B.Routing.topk(_dev(idx), 24, 4))


def test_no_alloc_matches_layout_expert_choice():
    inp = W.make_inputs(4)
    _compare(B.Routing.expert_choice(_dev(inp["token_indices"]), 8192, 1))
    _compare(B.Routing.expert_choice(_dev(inp["token_indices"]), 8192, 8))
    rng = np.random.Generator(np.random.PCG64(4))
    ti = W.random_token_indices(rng, 40, 16, 8, p_neg=0.2, p_bad=0.05)
    _compare(B.Routing.expert_choice(_dev(ti), 40, 4))


def test_no_alloc_matches_layout_expert_choice_past_the_cluster_limits():
    # 20000 tokens (more than one thread-block cluster handles): the
    # multi-kernel expert-choice layout, whose per-token counters and
    # unordered slot list live in the scratch array (256 + 4 (2T + EC) bytes,
    # about 226 KB here, inside the 4 MiB)
    rng = np.random.Generator(np.random.PCG64(5))
    ti = W.random_token_indices(rng, 20000, 64, 256, p_neg=0.1, p_bad=0.01)
    _compare(B.Routing.expert_choice(_dev(ti), 20000, 8))


def test_no_alloc_rejects_problems_beyond_the_fixed_scratch():
    # expert choice needing 256 + 4 * (2 T + E C) bytes > 4 MiB
    ti = torch.zeros((1024, 1024), dtype=torch.int32, device="cuda")
    routing = B.Routing.expert_choice(ti, 1000, 1)
    lay = B.Layout(routing)
    st = B.lib().ep_get_layout_no_alloc(ctypes.byref(routing.desc), ctypes.byref(lay.desc), None, None)
    assert st == 4  # EP_ERR_WORKSPACE, before anything is launched
    assert "workspace" in B.ep_status_string(st)
