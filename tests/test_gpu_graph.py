"""The path captured in a CUDA graph: the decode-size step (fused
low-latency layout + FP8 dispatch, then the padded combine) is captured once
and replayed; every replay gives the same bytes as the eager calls, and the
replayed outputs match the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_get_10_b200 import binding as B
from combine_ep_get_10_b200 import workloads as W
from gpu_util import assert_combine_close, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_ep_get_10_b200 import build

    build.build()
    B.lib()
    oracle.build()


def test_decode_step_in_a_cuda_graph():
    inp = W.make_inputs(3)
    c = inp["cfg"]
    T, H, E, R, K, mt = c["T"], c["H"], c["E"], c["R"], c["K"], c["max_tokens"]
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    xd, wd = to_dev(x, bf16=True), to_dev(w)
    routing = B.Routing.topk(to_dev(idx), E, R)
    lay = B.Layout(routing)
    q = torch.zeros((E * mt, H), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((E * mt, H // 128), dtype=torch.float32, device="cuda")
    y = torch.empty((E * mt, H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    # the "experts": dequantise the FP8 rows (a stand-in computed with torch)
    def experts():
        e4 = q.view(torch.float8_e4m3fn).to(torch.float32).view(E * mt, H // 128, 128)
        y.copy_((e4 * sc.view(E * mt, H // 128, 1)).view(E * mt, H).to(torch.bfloat16))

    def step(stream):
        B.ep_dispatch_low_latency(xd, routing, lay, q, max_tokens_per_expert=mt, recv_scales=sc, stream=stream)
        with torch.cuda.stream(stream):
            experts()
        B.ep_combine(y, routing, lay, wd, out, mode=B.EP_LAYOUT_PADDED, max_tokens_per_expert=mt, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    step(s)  # eager warm-up (library lookups happen outside the capture)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    assert B.ep_get_device_error(lay) == 0
    # against the oracle: layout, FP8 rows, then combine of the dequantised rows
    ref_l = oracle.tc_layout(idx, E, R)
    assert np.array_equal(host(lay.slot), ref_l["slot"])
    ref_d = oracle.tc_dispatch(x, idx, E, ref_l, mode=W.PADDED, max_tokens=mt, out_dtype=W.FP8_E4M3)
    counts = ref_l["num_tokens_per_expert"]
    valid = np.zeros(E * mt, bool)
    for e in range(E):
        valid[e * mt:e * mt + counts[e]] = True
    assert np.array_equal(host(q)[valid], ref_d["recv"][valid])
    y_host = host(y)
    ref_out = oracle.tc_combine(y_host, idx, E, ref_l, w, mode=W.PADDED, max_tokens=mt, out_dtype=W.BF16)
    assert_combine_close(host(out), ref_out, True, "graph replay")
