"""Write the stored regression digests under tests/golden/.

Calls only the CPU oracle (``oracle/``) on seeded inputs from
``combine_ep_get_10_b200.workloads``; nothing here comes from the CUDA path.
The pages print no worked example with values for this path, so these files
are regression anchors for the oracle itself: a later change to the oracle's
arithmetic shows up as a digest change and must be justified by the passage
it follows.

Run: python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from combine_ep_get_10_b200 import workloads as W  # noqa: E402


def digest(a):
    return hashlib.sha256(a.tobytes()).hexdigest()


def workload1():
    inp = W.make_inputs(1)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    L = oracle.tc_layout(idx, 8, 2)
    D = oracle.tc_dispatch(x, idx, 8, L, topk_weights=w, want_src=True, want_weights=True)
    C32 = oracle.tc_combine(D["recv"], idx, 8, L, w, out_dtype=oracle.FP32)
    C16 = oracle.tc_combine(D["recv"], idx, 8, L, w, out_dtype=oracle.BF16)
    return {
        "inputs": {"x": digest(x), "topk_idx": digest(idx), "topk_weights": digest(w)},
        "slot": digest(L["slot"]), "expert_offsets": L["expert_offsets"].tolist(),
        "num_tokens_per_rank": L["num_tokens_per_rank"].tolist(),
        "recv": digest(D["recv"]), "recv_src": digest(D["recv_src"]),
        "combine_fp32": digest(C32), "combine_bf16": digest(C16),
    }


def workload3_small():
    inp = W.make_inputs(3, T=16)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    L = oracle.tc_layout(idx, 256, 8)
    D = oracle.tc_dispatch(x, idx, 256, L, mode=oracle.PADDED, max_tokens=16, out_dtype=oracle.FP8_E4M3)
    return {"inputs": {"x": digest(x), "topk_idx": digest(idx)}, "recv_fp8": digest(D["recv"]),
            "recv_scales": digest(D["recv_scales"])}


def workload4_small():
    inp = W.make_inputs(4, T=512)
    ti, w = inp["token_indices"], inp["expert_weights"]
    L = oracle.ec_layout(ti, 512, 1)
    n = int(L["token_offsets"][-1])
    y = oracle.ec_dispatch(inp["x"], ti)
    C = oracle.ec_combine(y, L, w, 512, out_dtype=oracle.FP32)
    return {"inputs": {"token_indices": digest(ti), "expert_weights": digest(w)},
            "token_offsets": digest(L["token_offsets"]), "token_slots": digest(L["token_slots"][:n]),
            "combine_fp32": digest(C)}


def workload3_quant_formats():
    """Every quantised dispatch format on 16 decode tokens, compact rows."""
    inp = W.make_inputs(3, T=16)
    x, idx = inp["x"], inp["topk_idx"]
    L = oracle.tc_layout(idx, 256, 8)
    out = {}
    for name, dt in (("int8_per_token", oracle.INT8_PER_TOKEN), ("fp8_per_token", oracle.FP8_E4M3_PER_TOKEN),
                     ("mxfp8_e4m3", oracle.MXFP8_E4M3), ("mxfp8_e5m2", oracle.MXFP8_E5M2),
                     ("mxfp4_e2m1", oracle.MXFP4_E2M1)):
        D = oracle.tc_dispatch(x, idx, 256, L, out_dtype=dt)
        out[name] = {"codes": digest(D["recv"]), "scales": digest(D["recv_scales"])}
    return out


def workload1_ranks():
    """The per-rank (deduplicated) path on workload 1."""
    inp = W.make_inputs(1)
    x, idx, w = inp["x"], inp["topk_idx"], inp["topk_weights"]
    L = oracle.tc_layout(idx, 8, 2)
    RL = oracle.rank_layout(L["is_token_in_rank"])
    D = oracle.rank_dispatch(x, idx, 8, 2, RL, w, want_src=True)
    C = oracle.rank_combine(D["recv"], RL, out_dtype=oracle.FP32)
    return {"rank_offsets": RL["rank_offsets"].tolist(), "rank_row": digest(RL["rank_row"]),
            "recv": digest(D["recv"]), "recv_topk_idx": digest(D["recv_topk_idx"]),
            "recv_topk_weights": digest(D["recv_topk_weights"]), "combine_fp32": digest(C)}


def compute():
    return {"workload1": workload1(), "workload3_T16": workload3_small(), "workload4_T512": workload4_small(),
            "workload3_T16_quant": workload3_quant_formats(), "workload1_ranks": workload1_ranks()}


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_digests.json"), "w") as f:
        json.dump(compute(), f, indent=1, sort_keys=True)
        f.write("\n")
    print("wrote", os.path.join(HERE, "oracle_digests.json"))
