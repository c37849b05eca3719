"""Seeded synthetic inputs for the five MoE dispatch/combine workloads.

This module only makes inputs: token activations, router indices and gate
weights (token choice) or the per-expert token table and its weights (expert
choice).  It holds none of the layout / dispatch / combine arithmetic, and
both the CUDA library's tests and the CPU oracle's tests draw from it.

Generator: numpy ``PCG64`` seeded per workload.  Draw order inside a workload
is fixed (activations first, then routing) so a seed names one input set.
Activations are drawn in fp32 and narrowed to bf16 by torch's CPU cast; bf16
arrays are returned as ``uint16`` bit patterns.  Top-k selections sort by
descending score with ties to the lower index, and the k order of a row is
that descending order.

The workloads (sizes from the problem statement of the dispatch/combine path;
routing recipes where the statement is loose are the readings listed in the
design notes):

1. tiny token choice: T=128, H=256, E=8 in R=2 ranks, top-2 of softmax(N(0,1)
   logits), weights renormalised; seed 0.
2. prefill token choice: T=4096, H=7168, E=256 in R=8 ranks, top-8 of
   sigmoid(logits N(0,1) + per-expert bias N(0, 0.5)), weights = selected
   sigmoid values over their sum; seed 2.
3. decode low-latency: T=128, H=7168, E=256 in R=8, top-8 as in 1; FP8 e4m3
   dispatch into padded per-expert buffers of 128 rows; seed 3.
4. expert choice: T=8192, H=4096, E=128, C=128; token popularity log-Zipf
   (s=1.1) over a random permutation, scores = N(0,1) + popularity, each
   expert keeps its top-C tokens; weight of a pick = softmax, over the experts
   that picked that token, of their scores; seed 4.
5. skewed token choice: T=16384, H=7168, E=256 in R=8, 8 experts per token
   drawn without replacement from Zipf(s=1.2) popularity, each slot -1 with
   probability 0.1, weights Dirichlet(1) over the valid slots; seed 5.
"""
from __future__ import annotations

import numpy as np

BF16, FP32, FP8_E4M3 = 0, 1, 2
INT8_PER_TOKEN, FP8_E4M3_PER_TOKEN, MXFP8_E4M3, MXFP8_E5M2, MXFP4_E2M1 = 3, 4, 5, 6, 7
COMPACT, PADDED = 0, 1

CONFIGS = {
    1: dict(name="tiny-topk-128x256-top2", routing="topk", T=128, H=256, E=8, R=2, K=2, seed=0,
            router="softmax", mode=COMPACT, max_tokens=0, dispatch_dtype=BF16, combine_dtype=BF16),
    2: dict(name="prefill-topk-4096x7168-top8", routing="topk", T=4096, H=7168, E=256, R=8, K=8, seed=2,
            router="sigmoid_bias", mode=COMPACT, max_tokens=0, dispatch_dtype=BF16, combine_dtype=BF16),
    3: dict(name="decode-ll-fp8-128x7168-top8", routing="topk", T=128, H=7168, E=256, R=8, K=8, seed=3,
            router="softmax", mode=PADDED, max_tokens=128, dispatch_dtype=FP8_E4M3, combine_dtype=BF16),
    4: dict(name="expert-choice-8192x4096-E128-C128", routing="ec", T=8192, H=4096, E=128, C=128, R=1,
            seed=4, combine_dtype=BF16),
    5: dict(name="skewed-topk-16384x7168-top8", routing="topk", T=16384, H=7168, E=256, R=8, K=8, seed=5,
            router="zipf", mode=COMPACT, max_tokens=0, dispatch_dtype=BF16, combine_dtype=BF16),
}


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns via torch's CPU cast (input preparation only)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _topk_desc(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of each row, descending, ties -> lower index."""
    order = np.argsort(-scores, axis=-1, kind="stable")
    return order[..., :k]


def activations(rng: np.random.Generator, T: int, H: int, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal((T, H), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return to_bf16_bits(x)


def route_softmax_topk(rng, T, E, K):
    logits = rng.standard_normal((T, E), dtype=np.float32).astype(np.float64)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    idx = _topk_desc(p, K)
    sel = np.take_along_axis(p, idx, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return idx.astype(np.int64), w.astype(np.float32)


def route_sigmoid_bias_topk(rng, T, E, K):
    logits = rng.standard_normal((T, E), dtype=np.float32).astype(np.float64)
    bias = rng.normal(0.0, 0.5, size=E)
    s = 1.0 / (1.0 + np.exp(-(logits + bias[None, :])))
    idx = _topk_desc(s, K)
    sel = np.take_along_axis(s, idx, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return idx.astype(np.int64), w.astype(np.float32)


def route_zipf_dropped(rng, T, E, K, s=1.2, drop=0.1):
    p = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    p /= p.sum()
    idx = np.empty((T, K), np.int64)
    for t in range(T):
        idx[t] = rng.choice(E, K, replace=False, p=p)
    dropped = rng.random((T, K)) < drop
    idx[dropped] = -1
    w = np.zeros((T, K), np.float32)
    for t in range(T):
        valid = ~dropped[t]
        n = int(valid.sum())
        if n:
            w[t, valid] = rng.dirichlet(np.ones(n)).astype(np.float32)
    return idx, w


def route_expert_choice(rng, T, E, C, s=1.1):
    perm = rng.permutation(T)
    log_pop = np.empty(T, np.float64)
    log_pop[perm] = -s * np.log(np.arange(1, T + 1, dtype=np.float64))
    scores = rng.standard_normal((E, T)) + log_pop[None, :]
    ti = _topk_desc(scores, C).astype(np.int32)  # [E, C]
    picked = np.take_along_axis(scores, ti.astype(np.int64), axis=1)  # [E, C]
    # softmax, per token, over the experts that picked it
    flat_t = ti.reshape(-1).astype(np.int64)
    flat_s = picked.reshape(-1)
    tok_max = np.full(T, -np.inf)
    np.maximum.at(tok_max, flat_t, flat_s)
    ex = np.exp(flat_s - tok_max[flat_t])
    den = np.zeros(T)
    np.add.at(den, flat_t, ex)
    w = (ex / den[flat_t]).reshape(E, C).astype(np.float32)
    return ti, w


def make_inputs(cfg_id: int, seed: int | None = None, T: int | None = None) -> dict:
    """Inputs of workload ``cfg_id``.  ``seed`` overrides the workload seed
    (e.g. one seed per rank); ``T`` overrides the token count (test sizes)."""
    cfg = dict(CONFIGS[cfg_id])
    if seed is not None:
        cfg["seed"] = int(seed)
    if T is not None:
        cfg["T"] = int(T)
    rng = np.random.Generator(np.random.PCG64(cfg["seed"]))
    T_, H, E = cfg["T"], cfg["H"], cfg["E"]
    out = dict(cfg=cfg, x=activations(rng, T_, H))
    if cfg["routing"] == "topk":
        K = cfg["K"]
        if cfg["router"] == "softmax":
            idx, w = route_softmax_topk(rng, T_, E, K)
        elif cfg["router"] == "sigmoid_bias":
            idx, w = route_sigmoid_bias_topk(rng, T_, E, K)
        elif cfg["router"] == "zipf":
            idx, w = route_zipf_dropped(rng, T_, E, K)
        else:
            raise ValueError(cfg["router"])
        out["topk_idx"], out["topk_weights"] = idx, w
    else:
        ti, w = route_expert_choice(rng, T_, E, cfg["C"])
        out["token_indices"], out["expert_weights"] = ti, w
    return out


def random_topk(rng: np.random.Generator, T: int, E: int, K: int, p_neg: float = 0.0,
                allow_dup: bool = False, p_bad: float = 0.0) -> np.ndarray:
    """Small adversarial routing tables for edge-case tests: optional -1
    slots, duplicate experts within a row, and out-of-range ids."""
    if allow_dup or T == 0:
        idx = rng.integers(0, E, size=(T, K), dtype=np.int64)
    else:
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int64) if K <= E else \
            rng.integers(0, E, size=(T, K), dtype=np.int64)
    if p_neg:
        idx[rng.random((T, K)) < p_neg] = -1
    if p_bad:
        bad = rng.random((T, K)) < p_bad
        vals = rng.choice(np.array([E, E + 7, -2, -100, 1 << 40], np.int64), size=int(bad.sum()))
        idx[bad] = vals
    return idx


def random_token_indices(rng: np.random.Generator, T: int, E: int, C: int, p_neg: float = 0.0,
                         p_bad: float = 0.0) -> np.ndarray:
    """Expert-choice table like the page's example (uniform ids, duplicates
    allowed), with optional empty (-1) and out-of-range entries."""
    ti = rng.integers(0, T, size=(E, C), dtype=np.int32)
    if p_neg:
        ti[rng.random((E, C)) < p_neg] = -1
    if p_bad:
        bad = rng.random((E, C)) < p_bad
        ti[bad] = rng.choice(np.array([T, T + 3, -2, -77], np.int32), size=int(bad.sum()))
    return ti
