"""CPU oracle for the MoE layout / dispatch / combine path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  The
product path (``combine_ep_get_10_b200``) never imports it.

The arithmetic lives in ``ep_oracle.c`` (plain single-threaded C, one loop per
definition).  This module compiles it with gcc into ``libep_oracle.so`` next
to the source and wraps each routine for numpy arrays.  bf16 arrays are
carried as ``uint16`` bit patterns and FP8 arrays as ``uint8`` codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "libep_oracle.so")

# numeric codes shared with the public interface (dtype / buffer layout)
BF16, FP32, FP8_E4M3 = 0, 1, 2
INT8_PER_TOKEN, FP8_E4M3_PER_TOKEN, MXFP8_E4M3, MXFP8_E5M2, MXFP4_E2M1 = 3, 4, 5, 6, 7
QUANT_DTYPES = (FP8_E4M3, INT8_PER_TOKEN, FP8_E4M3_PER_TOKEN, MXFP8_E4M3, MXFP8_E5M2, MXFP4_E2M1)
COMPACT, PADDED = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ep_oracle.c to libep_oracle.so (gcc, -O2, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def load(path: str):
    """Load an oracle shared library built from ep_oracle.c (any path) and
    declare its signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    L.oracle_bf16_to_f32.restype = ctypes.c_float
    L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.oracle_f32_to_bf16.restype = ctypes.c_uint16
    L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    L.oracle_e4m3_to_f32.restype = ctypes.c_float
    L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    for name in ("oracle_f32_to_bf16_array", "oracle_f32_to_e4m3_array", "oracle_e4m3_to_f32_array",
                 "oracle_f32_to_e5m2_array", "oracle_e5m2_to_f32_array", "oracle_f32_to_e2m1_array",
                 "oracle_e2m1_to_f32_array", "oracle_f32_to_int8_array"):
        fn = getattr(L, name)
        fn.restype = None
        fn.argtypes = [P, P, i64]
    for name in ("oracle_fp8_quant_row", "oracle_int8_quant_row", "oracle_fp8_pertoken_quant_row"):
        fn = getattr(L, name)
        fn.restype = None
        fn.argtypes = [P, i32, P, P]
    L.oracle_mx_quant_row.restype = None
    L.oracle_mx_quant_row.argtypes = [i32, P, i32, P, P]
    L.oracle_quant_row.restype = None
    L.oracle_quant_row.argtypes = [i32, P, i32, P, P]
    L.oracle_mx_shared_exp.restype = i32
    L.oracle_mx_shared_exp.argtypes = [ctypes.c_float, i32]
    L.oracle_row_code_bytes.restype = i64
    L.oracle_row_code_bytes.argtypes = [i32, i32]
    L.oracle_row_scale_bytes.restype = i64
    L.oracle_row_scale_bytes.argtypes = [i32, i32]
    L.oracle_tc_layout.restype = i64
    L.oracle_tc_layout.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P]
    L.oracle_tc_dispatch.restype = i64
    L.oracle_tc_dispatch.argtypes = [P, i32, i32, P, i32, i32, P, P, i32, i32, i64, i32, P, P, P, P, P]
    L.oracle_tc_combine.restype = None
    L.oracle_tc_combine.argtypes = [P, i64, i32, i32, P, i32, i32, P, P, i32, i32, P, P, i32, i32, P]
    L.oracle_rank_layout.restype = None
    L.oracle_rank_layout.argtypes = [P, i32, i32, P, P]
    L.oracle_rank_dispatch.restype = None
    L.oracle_rank_dispatch.argtypes = [P, i32, i32, P, i32, i32, i32, P, P, P, P, P, P]
    L.oracle_rank_combine.restype = None
    L.oracle_rank_combine.argtypes = [P, i32, i32, i32, P, P, i32, i32, P]
    L.oracle_ec_layout.restype = i64
    L.oracle_ec_layout.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P]
    L.oracle_ec_dispatch.restype = None
    L.oracle_ec_dispatch.argtypes = [P, i32, i32, P, i32, i32, P]
    L.oracle_ec_combine.restype = None
    L.oracle_ec_combine.argtypes = [P, i32, i32, P, P, P, P, i32, i32, P]
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(_LIB)
    return _lib


def use(L) -> None:
    """Point this module's wrappers at another oracle library (tests that
    plant a mistake in a copy of the oracle use this); None restores it."""
    global _lib
    _lib = L


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def bf16_to_f32(bits):
    bits = _c(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a):
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_p(a), _p(out), a.size)
    return out


def f32_to_e4m3(a):
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().oracle_f32_to_e4m3_array(_p(a), _p(out), a.size)
    return out


def e4m3_to_f32(codes):
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, np.float32)
    lib().oracle_e4m3_to_f32_array(_p(codes), _p(out), codes.size)
    return out


def fp8_quant_row(xrow_bits):
    """One bf16 row -> (uint8 codes [H], float32 scales [H/128])."""
    x = _c(xrow_bits, np.uint16)
    H = x.size
    q = np.empty(H, np.uint8)
    s = np.empty(H // 128, np.float32)
    lib().oracle_fp8_quant_row(_p(x), H, _p(q), _p(s))
    return q, s


def _array_fn(name, in_dtype, out_dtype):
    def fn(a):
        a = _c(a, in_dtype)
        out = np.empty(a.shape, out_dtype)
        getattr(lib(), name)(_p(a), _p(out), a.size)
        return out

    fn.__name__ = name.replace("oracle_", "").replace("_array", "")
    return fn


f32_to_e5m2 = _array_fn("oracle_f32_to_e5m2_array", np.float32, np.uint8)
e5m2_to_f32 = _array_fn("oracle_e5m2_to_f32_array", np.uint8, np.float32)
f32_to_e2m1 = _array_fn("oracle_f32_to_e2m1_array", np.float32, np.uint8)  # 4-bit codes, one per byte
e2m1_to_f32 = _array_fn("oracle_e2m1_to_f32_array", np.uint8, np.float32)
f32_to_int8 = _array_fn("oracle_f32_to_int8_array", np.float32, np.int8)


def row_code_bytes(dtype, hidden):
    return int(lib().oracle_row_code_bytes(int(dtype), int(hidden)))


def row_scale_bytes(dtype, hidden):
    return int(lib().oracle_row_scale_bytes(int(dtype), int(hidden)))


def scale_array(dtype, rows, hidden):
    """Zeroed scale buffer of the layout the output format uses."""
    if dtype == FP8_E4M3:
        return np.zeros((rows, hidden // 128), np.float32)
    if dtype in (INT8_PER_TOKEN, FP8_E4M3_PER_TOKEN):
        return np.zeros(rows, np.float32)
    if dtype in (MXFP8_E4M3, MXFP8_E5M2, MXFP4_E2M1):
        return np.zeros((rows, hidden // 32), np.uint8)
    return None


def code_array(dtype, rows, hidden):
    """Zeroed code buffer of the layout the output format uses."""
    if dtype == BF16:
        return np.zeros((rows, hidden), np.uint16)
    if dtype == INT8_PER_TOKEN:
        return np.zeros((rows, hidden), np.int8)
    return np.zeros((rows, row_code_bytes(dtype, hidden)), np.uint8)


def quant_row(dtype, xrow_bits):
    """One bf16 row -> (codes, scales) in output format `dtype` (any of
    QUANT_DTYPES); shapes as one row of code_array / scale_array."""
    x = _c(xrow_bits, np.uint16)
    H = x.size
    q = code_array(dtype, 1, H)[0]
    s = scale_array(dtype, 1, H)
    s = s[0] if s.ndim == 2 else s
    lib().oracle_quant_row(int(dtype), _p(x), H, _p(q), _p(s))
    return q, s


def mx_shared_exp(amax, emax_elem):
    return int(lib().oracle_mx_shared_exp(float(amax), int(emax_elem)))


# ---------------------------------------------------------- token choice
def tc_layout(topk_idx, num_experts, num_ranks):
    idx = _c(topk_idx, np.int64)
    T, K = idx.shape
    E, R = int(num_experts), int(num_ranks)
    out = dict(
        num_tokens_per_expert=np.empty(E, np.int32),
        expert_offsets=np.empty(E + 1, np.int32),
        num_tokens_per_rank=np.empty(R, np.int32),
        is_token_in_rank=np.empty((T, R), np.uint8),
        slot=np.empty((T, K), np.int32),
    )
    bad = lib().oracle_tc_layout(_p(idx), T, K, E, R, _p(out["num_tokens_per_expert"]),
                                 _p(out["expert_offsets"]), _p(out["num_tokens_per_rank"]),
                                 _p(out["is_token_in_rank"]), _p(out["slot"]))
    out["bad_index_count"] = int(bad)
    return out


def tc_dispatch(x_bits, topk_idx, num_experts, layout, mode=COMPACT, max_tokens=0, out_dtype=BF16,
                topk_weights=None, num_recv_rows=None, want_src=False, want_weights=False):
    """Returns dict(recv, recv_scales, recv_src, recv_weights, overflow_count)."""
    x = _c(x_bits, np.uint16)
    idx = _c(topk_idx, np.int64)
    T, H = x.shape
    K = idx.shape[1]
    E = int(num_experts)
    slot = _c(layout["slot"], np.int32)
    offs = _c(layout["expert_offsets"], np.int32)
    if num_recv_rows is None:
        num_recv_rows = E * max_tokens if mode == PADDED else int(offs[E])
    rows = int(num_recv_rows)
    recv = code_array(out_dtype, rows, H)
    scales = scale_array(out_dtype, rows, H)
    if want_weights and topk_weights is None:
        raise ValueError("recv_weights needs topk_weights")
    src = np.full(rows, -1, np.int32) if want_src else None
    wts = np.zeros(rows, np.float32) if want_weights else None
    w = _c(topk_weights, np.float32) if topk_weights is not None else None
    ovf = lib().oracle_tc_dispatch(_p(x), T, H, _p(idx), K, E, _p(slot), _p(offs), int(mode), int(max_tokens),
                                   rows, int(out_dtype), _p(w), _p(recv), _p(scales), _p(src), _p(wts))
    return dict(recv=recv, recv_scales=scales, recv_src=src, recv_weights=wts, overflow_count=int(ovf))


def tc_combine(y_bits, topk_idx, num_experts, layout, topk_weights, mode=COMPACT, max_tokens=0,
               out_dtype=FP32, tokens=None):
    y = _c(y_bits, np.uint16)
    idx = _c(topk_idx, np.int64)
    T, K = idx.shape
    H = y.shape[1]
    slot = _c(layout["slot"], np.int32)
    offs = _c(layout["expert_offsets"], np.int32)
    w = _c(topk_weights, np.float32)
    tok = None if tokens is None else _c(tokens, np.int32)
    n = T if tok is None else tok.size
    out = np.empty((n, H), np.float32 if out_dtype == FP32 else np.uint16)
    lib().oracle_tc_combine(_p(y), y.shape[0], H, T, _p(idx), K, int(num_experts), _p(slot), _p(offs),
                            int(mode), int(max_tokens), _p(w), _p(tok), n, int(out_dtype), _p(out))
    return out


# ------------------------------------------- per-rank (deduplicated) path
def rank_layout(is_token_in_rank):
    """is_token_in_rank [T, R] -> dict(rank_offsets [R+1], rank_row [T, R])."""
    m = _c(is_token_in_rank, np.uint8)
    T, R = m.shape
    out = dict(rank_offsets=np.empty(R + 1, np.int32), rank_row=np.empty((T, R), np.int32))
    lib().oracle_rank_layout(_p(m), T, R, _p(out["rank_offsets"]), _p(out["rank_row"]))
    return out


def rank_dispatch(x_bits, topk_idx, num_experts, num_ranks, rlayout, topk_weights=None, want_src=False):
    """Returns dict(recv [rows, H] bf16 bits, recv_topk_idx [rows, K], recv_topk_weights [rows, K], recv_src)."""
    x = _c(x_bits, np.uint16)
    idx = _c(topk_idx, np.int64)
    T, H = x.shape
    K = idx.shape[1]
    rr = _c(rlayout["rank_row"], np.int32)
    rows = int(rlayout["rank_offsets"][-1])
    w = _c(topk_weights, np.float32) if topk_weights is not None else np.zeros((T, K), np.float32)
    recv = np.zeros((rows, H), np.uint16)
    ridx = np.full((rows, K), -2, np.int64)
    rw = np.full((rows, K), np.nan, np.float32)
    src = np.full(rows, -1, np.int32) if want_src else None
    lib().oracle_rank_dispatch(_p(x), T, H, _p(idx), K, int(num_experts), int(num_ranks), _p(rr), _p(w), _p(recv),
                               _p(ridx), _p(rw), _p(src))
    return dict(recv=recv, recv_topk_idx=ridx, recv_topk_weights=rw, recv_src=src)


def rank_combine(y_bits, rlayout, out_dtype=FP32, tokens=None):
    y = _c(y_bits, np.uint16)
    H = y.shape[1]
    rr = _c(rlayout["rank_row"], np.int32)
    T, R = rr.shape
    tok = None if tokens is None else _c(tokens, np.int32)
    n = T if tok is None else tok.size
    out = np.empty((n, H), np.float32 if out_dtype == FP32 else np.uint16)
    lib().oracle_rank_combine(_p(y), H, T, R, _p(rr), _p(tok), n, int(out_dtype), _p(out))
    return out


# --------------------------------------------------------- expert choice
def ec_layout(token_indices, num_tokens, num_ranks):
    ti = _c(token_indices, np.int32)
    E, C = ti.shape
    T, R = int(num_tokens), int(num_ranks)
    out = dict(
        num_tokens_per_expert=np.empty(E, np.int32),
        num_tokens_per_rank=np.empty(R, np.int32),
        is_token_in_rank=np.empty((T, R), np.uint8),
        token_offsets=np.empty(T + 1, np.int32),
        token_slots=np.full(E * C, -1, np.int32),
    )
    bad = lib().oracle_ec_layout(_p(ti), T, E, C, R, _p(out["num_tokens_per_expert"]),
                                 _p(out["num_tokens_per_rank"]), _p(out["is_token_in_rank"]),
                                 _p(out["token_offsets"]), _p(out["token_slots"]))
    out["bad_index_count"] = int(bad)
    return out


def ec_dispatch(x_bits, token_indices, recv=None):
    x = _c(x_bits, np.uint16)
    ti = _c(token_indices, np.int32)
    T, H = x.shape
    E, C = ti.shape
    if recv is None:
        recv = np.zeros((E * C, H), np.uint16)
    lib().oracle_ec_dispatch(_p(x), T, H, _p(ti), E, C, _p(recv))
    return recv


def ec_combine(y_bits, layout, expert_weights, num_tokens, out_dtype=FP32, tokens=None):
    y = _c(y_bits, np.uint16)
    H = y.shape[1]
    offs = _c(layout["token_offsets"], np.int32)
    slots = _c(layout["token_slots"], np.int32)
    w = _c(expert_weights, np.float32).reshape(-1)
    tok = None if tokens is None else _c(tokens, np.int32)
    T = int(num_tokens)
    n = T if tok is None else tok.size
    out = np.empty((n, H), np.float32 if out_dtype == FP32 else np.uint16)
    lib().oracle_ec_combine(_p(y), H, T, _p(offs), _p(slots), _p(w), _p(tok), n, int(out_dtype), _p(out))
    return out
