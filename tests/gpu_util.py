"""Helpers for the GPU parity tests: host <-> device copies of the seeded
inputs and the comparison rules (bit-exact for integer / byte outputs; the
combine tolerance: fp32 within rtol 1e-5 / atol 1e-6, bf16 within 1 ulp)."""
from __future__ import annotations

import numpy as np
import torch


def to_dev(a: np.ndarray, bf16: bool = False) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if bf16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_host(t)
    return t.cpu().numpy()


def assert_combine_close(got: np.ndarray, ref: np.ndarray, bf16: bool, what: str = "") -> None:
    """fp32: |got - ref| <= 1e-6 + 1e-5 |ref|.  bf16 (uint16 bits): the two
    values are at most one bf16 ulp apart (adjacent codes on one sign)."""
    if bf16:
        g = got.astype(np.int32)
        r = ref.astype(np.int32)
        # order-preserving integer view of bf16 bit patterns
        go = np.where(g & 0x8000, -(g & 0x7FFF), g & 0x7FFF)
        ro = np.where(r & 0x8000, -(r & 0x7FFF), r & 0x7FFF)
        bad = np.abs(go - ro) > 1
        assert not bad.any(), "%s: %d bf16 values more than 1 ulp apart" % (what, int(bad.sum()))
    else:
        bad = ~(np.abs(got.astype(np.float64) - ref) <= 1e-6 + 1e-5 * np.abs(ref.astype(np.float64)))
        assert not bad.any(), "%s: %d fp32 values outside rtol 1e-5 / atol 1e-6" % (what, int(bad.sum()))


def exact_fraction(got: np.ndarray, ref: np.ndarray) -> float:
    g = got.view(np.uint32) if got.dtype == np.float32 else got
    r = ref.view(np.uint32) if ref.dtype == np.float32 else ref
    return float((g == r).mean()) if g.size else 1.0
