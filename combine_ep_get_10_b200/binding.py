"""Thin ctypes binding of libep_b200.so (C ABI in include/ep.h).

Argument marshalling only: torch tensors are turned into device pointers and
sizes, the current CUDA stream is passed through, and a non-OK status raises
EPError.  Every step of layout / dispatch / combine runs in the library's
CUDA kernels; this module does no arithmetic on the data and has no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libep_b200.so")

# ABI version and enums of include/ep.h
EP_ABI_VERSION = 3  # the structures below follow this version of the header
EP_OK = 0
EP_ERR_INVALID_ARG, EP_ERR_BAD_INDEX, EP_ERR_OVERFLOW, EP_ERR_WORKSPACE = 1, 2, 3, 4
EP_ERR_CUDA, EP_ERR_UNSUPPORTED, EP_ERR_TIMEOUT = 5, 6, 7
STATUS_NAMES = {0: "EP_OK", 1: "EP_ERR_INVALID_ARG", 2: "EP_ERR_BAD_INDEX", 3: "EP_ERR_OVERFLOW",
                4: "EP_ERR_WORKSPACE", 5: "EP_ERR_CUDA", 6: "EP_ERR_UNSUPPORTED", 7: "EP_ERR_TIMEOUT"}
EP_BF16, EP_FP32, EP_FP8_E4M3 = 0, 1, 2
EP_INT8_PER_TOKEN, EP_FP8_E4M3_PER_TOKEN, EP_MXFP8_E4M3, EP_MXFP8_E5M2, EP_MXFP4_E2M1 = 3, 4, 5, 6, 7
EP_LAYOUT_COMPACT, EP_LAYOUT_PADDED = 0, 1
EP_ROUTING_TOPK, EP_ROUTING_EXPERT_CHOICE = 0, 1
EP_DEVERR_BAD_INDEX, EP_DEVERR_OVERFLOW, EP_DEVERR_TIMEOUT = 0x1, 0x2, 0x4

EXPORTED = ("ep_workspace_bytes", "ep_workspace_init", "ep_get_layout", "ep_dispatch", "ep_combine",
            "ep_dispatch_expert_choice", "ep_combine_expert_choice", "ep_get_device_error", "ep_status_string",
            "ep_version", "ep_get_layout_no_alloc", "ep_get_rank_layout", "ep_dispatch_ranks", "ep_combine_ranks",
            "ep_dispatch_low_latency", "ep_layout_dispatch", "ep_peer_alloc", "ep_peer_free", "ep_peer_open",
            "ep_peer_close", "ep_peer_publish_counts", "ep_dispatch_peers", "ep_combine_peers",
            "ep_layout_dispatch_expert_choice", "ep_layout_dispatch_ranks")


class EPError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (what, STATUS_NAMES.get(status, status), _status_text(status)))


class RoutingDesc(ctypes.Structure):
    _fields_ = [("routing", ctypes.c_int), ("topk_idx", ctypes.c_void_p), ("token_indices", ctypes.c_void_p),
                ("num_tokens", ctypes.c_int32), ("num_topk", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("num_ranks", ctypes.c_int32)]


class LayoutDesc(ctypes.Structure):
    _fields_ = [("num_tokens_per_expert", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p),
                ("num_tokens_per_rank", ctypes.c_void_p), ("is_token_in_rank", ctypes.c_void_p),
                ("slot", ctypes.c_void_p), ("token_offsets", ctypes.c_void_p), ("token_slots", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("num_valid_host", ctypes.c_void_p)]


class RankLayoutDesc(ctypes.Structure):
    _fields_ = [("rank_offsets", ctypes.c_void_p), ("rank_row", ctypes.c_void_p)]


class PeersDesc(ctypes.Structure):
    _fields_ = [("num_ranks", ctypes.c_int32), ("rank", ctypes.c_int32), ("capacity", ctypes.c_int64),
                ("recv_x", ctypes.c_void_p), ("recv_topk_idx", ctypes.c_void_p),
                ("recv_topk_weights", ctypes.c_void_p), ("recv_src", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("rank_counts", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded library; raises if it is missing (build it with
    ``python -m combine_ep_get_10_b200.build``).  There is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libep_b200.so is not built (%s); run python -m combine_ep_get_10_b200.build"
                              % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int
        RP, LP = ctypes.POINTER(RoutingDesc), ctypes.POINTER(LayoutDesc)
        L.ep_workspace_bytes.restype = ctypes.c_size_t
        L.ep_workspace_bytes.argtypes = [RP]
        L.ep_workspace_init.restype = st
        L.ep_workspace_init.argtypes = [P, ctypes.c_size_t, P]
        L.ep_get_layout.restype = st
        L.ep_get_layout.argtypes = [RP, LP, P]
        L.ep_dispatch.restype = st
        L.ep_dispatch.argtypes = [P, i32, RP, LP, st, i32, i64, st, P, P, P, P, P, P]
        L.ep_combine.restype = st
        L.ep_combine.argtypes = [P, i32, i64, RP, LP, st, i32, P, P, st, P]
        L.ep_dispatch_expert_choice.restype = st
        L.ep_dispatch_expert_choice.argtypes = [P, i32, RP, LP, P, P]
        L.ep_layout_dispatch_expert_choice.restype = st
        L.ep_layout_dispatch_expert_choice.argtypes = [P, i32, RP, LP, P, P]
        L.ep_combine_expert_choice.restype = st
        L.ep_combine_expert_choice.argtypes = [P, i32, RP, LP, P, P, st, P]
        L.ep_get_device_error.restype = st
        L.ep_get_device_error.argtypes = [LP, ctypes.POINTER(ctypes.c_uint32), st, P]
        L.ep_status_string.restype = ctypes.c_char_p
        L.ep_status_string.argtypes = [st]
        L.ep_version.restype = ctypes.c_int
        L.ep_version.argtypes = []
        L.ep_get_layout_no_alloc.restype = st
        L.ep_get_layout_no_alloc.argtypes = [RP, LP, P, P]
        KP = ctypes.POINTER(RankLayoutDesc)
        L.ep_get_rank_layout.restype = st
        L.ep_get_rank_layout.argtypes = [RP, LP, KP, P]
        L.ep_dispatch_ranks.restype = st
        L.ep_dispatch_ranks.argtypes = [P, i32, RP, LP, KP, i64, P, P, P, P, P, P]
        L.ep_layout_dispatch_ranks.restype = st
        L.ep_layout_dispatch_ranks.argtypes = [P, i32, RP, LP, KP, i64, P, P, P, P, P, P]
        L.ep_combine_ranks.restype = st
        L.ep_combine_ranks.argtypes = [P, i32, i64, RP, LP, KP, P, st, P]
        L.ep_dispatch_low_latency.restype = st
        L.ep_dispatch_low_latency.argtypes = [P, i32, RP, LP, i32, st, P, P, P, P, P, P]
        L.ep_layout_dispatch.restype = st
        L.ep_layout_dispatch.argtypes = [P, i32, RP, LP, st, i32, i64, st, P, P, P, P, P, P]
        PP = ctypes.POINTER(PeersDesc)
        L.ep_peer_alloc.restype = st
        L.ep_peer_alloc.argtypes = [ctypes.c_size_t, ctypes.POINTER(P), P]
        L.ep_peer_free.restype = st
        L.ep_peer_free.argtypes = [P]
        L.ep_peer_open.restype = st
        L.ep_peer_open.argtypes = [P, ctypes.POINTER(P)]
        L.ep_peer_close.restype = st
        L.ep_peer_close.argtypes = [P]
        L.ep_peer_publish_counts.restype = st
        L.ep_peer_publish_counts.argtypes = [RP, LP, PP, P]
        L.ep_dispatch_peers.restype = st
        L.ep_dispatch_peers.argtypes = [P, i32, RP, LP, KP, P, PP, P]
        L.ep_combine_peers.restype = st
        L.ep_combine_peers.argtypes = [i32, RP, LP, KP, PP, P, st, P]
        if L.ep_version() != EP_ABI_VERSION:
            raise ImportError("libep_b200.so has ABI version %d, the binding expects %d; rebuild it"
                              % (L.ep_version(), EP_ABI_VERSION))
        _lib = L
    return _lib


def _status_text(status: int) -> str:
    try:
        return lib().ep_status_string(status).decode()
    except Exception:
        return "?"


def _check(status: int, what: str) -> None:
    if status != EP_OK:
        raise EPError(status, what)


def _ptr(t):
    """Device (or pinned host) address of a dense row-major tensor; the C ABI
    takes plain pointers, so strided views are refused here."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("the C ABI takes dense row-major tensors; got a strided view of shape %s"
                         % (tuple(t.shape),))
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return EP_BF16
    if t.dtype == torch.float32:
        return EP_FP32
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return EP_FP8_E4M3
    raise TypeError("unsupported dtype %s" % t.dtype)


class Routing:
    """A routing decision on the device plus its C descriptor."""

    def __init__(self, desc: RoutingDesc, keep):
        self.desc = desc
        self._keep = keep

    @staticmethod
    def topk(topk_idx: torch.Tensor, num_experts: int, num_ranks: int) -> "Routing":
        if topk_idx.dtype != torch.int64 or topk_idx.dim() != 2 or not topk_idx.is_contiguous():
            raise TypeError("topk_idx must be a contiguous int64 [T, K] tensor")
        d = RoutingDesc(EP_ROUTING_TOPK, topk_idx.data_ptr(), None, topk_idx.shape[0], topk_idx.shape[1], 0,
                        num_experts, num_ranks)
        return Routing(d, topk_idx)

    @staticmethod
    def expert_choice(token_indices: torch.Tensor, num_tokens: int, num_ranks: int) -> "Routing":
        if token_indices.dtype != torch.int32 or token_indices.dim() != 2 or not token_indices.is_contiguous():
            raise TypeError("token_indices must be a contiguous int32 [E, C] tensor")
        E, C = token_indices.shape
        d = RoutingDesc(EP_ROUTING_EXPERT_CHOICE, None, token_indices.data_ptr(), num_tokens, 0, C, E, num_ranks)
        return Routing(d, token_indices)

    def tokens(self, t0: int, t1: int) -> "Routing":
        """Token-choice routing of tokens [t0, t1) only (a view: the topk_idx
        pointer is offset).  With Layout.tokens() it lets dispatch and combine
        run on a chunk of tokens, e.g. to overlap host transfers of the next
        chunk, or to bound per-call working sets on long sequences."""
        if self.desc.routing != EP_ROUTING_TOPK or not (0 <= t0 <= t1 <= self.desc.num_tokens):
            raise ValueError("token range [%d, %d) of a token-choice routing of %d tokens"
                             % (t0, t1, self.desc.num_tokens))
        d = RoutingDesc(EP_ROUTING_TOPK, self.desc.topk_idx + t0 * self.desc.num_topk * 8, None, t1 - t0,
                        self.desc.num_topk, 0, self.desc.num_experts, self.desc.num_ranks)
        return Routing(d, self)

    @property
    def T(self):
        return self.desc.num_tokens

    @property
    def E(self):
        return self.desc.num_experts

    @property
    def R(self):
        return self.desc.num_ranks


def ep_workspace_bytes(routing: Routing) -> int:
    n = lib().ep_workspace_bytes(ctypes.byref(routing.desc))
    if n == 0:
        raise EPError(EP_ERR_INVALID_ARG, "ep_workspace_bytes")
    return int(n)


def ep_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().ep_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "ep_workspace_init")


class Layout:
    """Device buffers of one layout (allocated by torch, i.e. by the caller
    of the C ABI) plus the C descriptor pointing at them.  With
    report_num_valid=True a pinned host int32 is attached as num_valid_host:
    every layout call then copies the filled-row count into it and returns
    after the stream caught up (read it as .num_valid)."""

    def __init__(self, routing: Routing, device="cuda", workspace: torch.Tensor | None = None, stream=None,
                 report_num_valid: bool = False):
        T, E, R = routing.T, routing.E, routing.R
        i32 = dict(dtype=torch.int32, device=device)
        self.num_tokens_per_expert = torch.empty(E, **i32)
        self.num_tokens_per_rank = torch.empty(R, **i32)
        self.is_token_in_rank = torch.empty((T, R), dtype=torch.uint8, device=device)
        self.expert_offsets = self.slot = self.token_offsets = self.token_slots = None
        if routing.desc.routing == EP_ROUTING_TOPK:
            self.expert_offsets = torch.empty(E + 1, **i32)
            self.slot = torch.empty((T, routing.desc.num_topk), **i32)
        else:
            self.token_offsets = torch.empty(T + 1, **i32)
            self.token_slots = torch.empty(E * routing.desc.capacity, **i32)
        need = ep_workspace_bytes(routing)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=device)
            ep_workspace_init(workspace, stream)
        elif workspace.numel() * workspace.element_size() < need:
            raise ValueError("workspace too small: %d < %d" % (workspace.numel(), need))
        self.workspace = workspace
        self.num_valid_host = torch.zeros(1, dtype=torch.int32).pin_memory() if report_num_valid else None
        self.desc = LayoutDesc(*(None if t is None else t.data_ptr() for t in (
            self.num_tokens_per_expert, self.expert_offsets, self.num_tokens_per_rank, self.is_token_in_rank,
            self.slot, self.token_offsets, self.token_slots, self.workspace)),
            self.workspace.numel() * self.workspace.element_size(),
            None if self.num_valid_host is None else self.num_valid_host.data_ptr())

    @property
    def num_valid(self) -> int:
        """Filled rows reported by the last layout call (needs report_num_valid)."""
        if self.num_valid_host is None:
            raise ValueError("this layout was made without report_num_valid")
        return int(self.num_valid_host[0])


class LayoutView:
    """A token-choice layout restricted to tokens [t0, t1) of its routing:
    the slot pointer is offset; counts, offsets and workspace are shared."""

    def __init__(self, parent: Layout, t0: int, k: int):
        self.parent = parent
        self.desc = LayoutDesc.from_buffer_copy(parent.desc)
        self.desc.num_valid_host = None  # counts are the parent's; a view never reports them
        if parent.slot is not None:
            self.desc.slot = parent.desc.slot + t0 * k * 4
        self.desc.is_token_in_rank = parent.desc.is_token_in_rank + t0 * parent.num_tokens_per_rank.numel()


def layout_tokens(layout: Layout, routing: Routing, t0: int, t1: int) -> LayoutView:
    """View of `layout` for tokens [t0, t1) of `routing` (see Routing.tokens)."""
    if not (0 <= t0 <= t1 <= routing.T):
        raise ValueError("bad token range")
    return LayoutView(layout, t0, routing.desc.num_topk)


def token_rounds(num_tokens: int, per_round_tokens: int) -> list[tuple[int, int]]:
    """Token ranges [t0, t1) of a long batch processed in rounds of at most
    per_round_tokens tokens (the README's "ant moving home" long-sequence
    mode: DEEPEP_NORMAL_LONG_SEQ_PER_ROUND_TOKENS tokens per round).  Each
    round is an independent layout -> dispatch -> (experts) -> combine on
    Routing.tokens(t0, t1), so the receive buffers need only
    per_round_tokens * K rows; per-token results equal the one-shot ones."""
    if num_tokens < 0 or per_round_tokens < 1:
        raise ValueError("num_tokens >= 0 and per_round_tokens >= 1")
    return [(t0, min(num_tokens, t0 + per_round_tokens)) for t0 in range(0, num_tokens, per_round_tokens)]


def ep_get_layout(routing: Routing, layout: Layout, stream=None) -> Layout:
    _check(lib().ep_get_layout(ctypes.byref(routing.desc), ctypes.byref(layout.desc), _stream(stream)),
           "ep_get_layout")
    return layout


def ep_dispatch(x: torch.Tensor, routing: Routing, layout: Layout, recv_x: torch.Tensor, *, mode=EP_LAYOUT_COMPACT,
                max_tokens_per_expert=0, num_recv_rows=None, topk_weights=None, recv_scales=None, recv_src=None,
                recv_weights=None, out_dtype=None, stream=None) -> None:
    """out_dtype: one of the EP_* element formats; by default it follows
    recv_x (bfloat16, or uint8 / float8_e4m3fn for 128-channel FP8)."""
    out_dtype = _dtype_code(recv_x) if out_dtype is None else int(out_dtype)
    rows = recv_x.shape[0] if num_recv_rows is None else int(num_recv_rows)
    _check(lib().ep_dispatch(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc), int(mode),
                             int(max_tokens_per_expert), rows, out_dtype, _ptr(topk_weights), _ptr(recv_x),
                             _ptr(recv_scales), _ptr(recv_src), _ptr(recv_weights), _stream(stream)), "ep_dispatch")


def ep_layout_dispatch(x: torch.Tensor, routing: Routing, layout: Layout, recv_x: torch.Tensor, *,
                       mode=EP_LAYOUT_COMPACT, max_tokens_per_expert=0, num_recv_rows=None, topk_weights=None,
                       recv_scales=None, recv_src=None, recv_weights=None, out_dtype=None, stream=None) -> None:
    """ep_get_layout + ep_dispatch in one call (the dispatch's row loads
    overlap the layout kernel); arguments as for ep_dispatch."""
    out_dtype = _dtype_code(recv_x) if out_dtype is None else int(out_dtype)
    rows = recv_x.shape[0] if num_recv_rows is None else int(num_recv_rows)
    _check(lib().ep_layout_dispatch(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                    int(mode), int(max_tokens_per_expert), rows, out_dtype, _ptr(topk_weights),
                                    _ptr(recv_x), _ptr(recv_scales), _ptr(recv_src), _ptr(recv_weights),
                                    _stream(stream)), "ep_layout_dispatch")


def ep_dispatch_low_latency(x: torch.Tensor, routing: Routing, layout: Layout, recv_x: torch.Tensor, *,
                            max_tokens_per_expert: int, out_dtype=None, topk_weights=None, recv_scales=None,
                            recv_src=None, recv_weights=None, stream=None) -> None:
    """ep_get_layout + padded ep_dispatch in one launch for small batches
    (layout outputs land in `layout`); out_dtype as for ep_dispatch."""
    out_dtype = _dtype_code(recv_x) if out_dtype is None else int(out_dtype)
    _check(lib().ep_dispatch_low_latency(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                         int(max_tokens_per_expert), out_dtype, _ptr(topk_weights), _ptr(recv_x),
                                         _ptr(recv_scales), _ptr(recv_src), _ptr(recv_weights), _stream(stream)),
           "ep_dispatch_low_latency")


def ep_combine(y: torch.Tensor, routing: Routing, layout: Layout, topk_weights: torch.Tensor, out: torch.Tensor, *,
               mode=EP_LAYOUT_COMPACT, max_tokens_per_expert=0, num_y_rows=None, stream=None) -> None:
    """out dtype follows `out` (bfloat16 or float32)."""
    rows = y.shape[0] if num_y_rows is None else int(num_y_rows)
    _check(lib().ep_combine(_ptr(y), y.shape[1], rows, ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                            int(mode), int(max_tokens_per_expert), _ptr(topk_weights), _ptr(out), _dtype_code(out),
                            _stream(stream)), "ep_combine")


def ep_dispatch_expert_choice(x: torch.Tensor, routing: Routing, layout: Layout, recv_x: torch.Tensor,
                              stream=None) -> None:
    _check(lib().ep_dispatch_expert_choice(_ptr(x), x.shape[1], ctypes.byref(routing.desc),
                                           ctypes.byref(layout.desc), _ptr(recv_x), _stream(stream)),
           "ep_dispatch_expert_choice")


def ep_layout_dispatch_expert_choice(x: torch.Tensor, routing: Routing, layout: Layout, recv_x: torch.Tensor,
                                     stream=None) -> Layout:
    """ep_get_layout + ep_dispatch_expert_choice in one call; the copy runs
    under the layout kernel."""
    _check(lib().ep_layout_dispatch_expert_choice(_ptr(x), x.shape[1], ctypes.byref(routing.desc),
                                                  ctypes.byref(layout.desc), _ptr(recv_x), _stream(stream)),
           "ep_layout_dispatch_expert_choice")
    return layout


def ep_combine_expert_choice(y: torch.Tensor, routing: Routing, layout: Layout, expert_weights: torch.Tensor,
                             out: torch.Tensor, stream=None) -> None:
    _check(lib().ep_combine_expert_choice(_ptr(y), y.shape[1], ctypes.byref(routing.desc),
                                          ctypes.byref(layout.desc), _ptr(expert_weights), _ptr(out),
                                          _dtype_code(out), _stream(stream)), "ep_combine_expert_choice")


def ep_get_device_error(layout: Layout, clear: bool = True, stream=None) -> int:
    """Synchronises the stream; returns the EP_DEVERR_* bits (0 = none)."""
    flags = ctypes.c_uint32(0)
    st = lib().ep_get_device_error(ctypes.byref(layout.desc), ctypes.byref(flags), 1 if clear else 0,
                                   _stream(stream))
    if st not in (EP_OK, EP_ERR_BAD_INDEX, EP_ERR_OVERFLOW, EP_ERR_TIMEOUT):  # these report the flags
        raise EPError(st, "ep_get_device_error")
    return int(flags.value)


def ep_status_string(status: int) -> str:
    return lib().ep_status_string(status).decode()


class RankLayout:
    """Device buffers of a per-rank layout: rank_offsets [R+1] and
    rank_row [T, R] (allocated by torch), plus the C descriptor."""

    def __init__(self, routing: Routing, device="cuda"):
        d = device
        T, R = routing.desc.num_tokens, routing.desc.num_ranks
        self.rank_offsets = torch.empty(R + 1, dtype=torch.int32, device=d)
        self.rank_row = torch.empty((T, R), dtype=torch.int32, device=d)
        self.desc = RankLayoutDesc(self.rank_offsets.data_ptr(), self.rank_row.data_ptr() if T > 0 else None)


def ep_get_rank_layout(routing: Routing, layout: Layout, rank_layout: RankLayout, stream=None) -> None:
    _check(lib().ep_get_rank_layout(ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                    ctypes.byref(rank_layout.desc), _stream(stream)), "ep_get_rank_layout")


def ep_dispatch_ranks(x: torch.Tensor, routing: Routing, layout: Layout, rank_layout: RankLayout,
                      recv_x: torch.Tensor, *, num_recv_rows=None, topk_weights=None, recv_topk_idx=None,
                      recv_topk_weights=None, recv_src=None, stream=None) -> None:
    rows = recv_x.shape[0] if num_recv_rows is None else int(num_recv_rows)
    _check(lib().ep_dispatch_ranks(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                   ctypes.byref(rank_layout.desc), rows, _ptr(topk_weights), _ptr(recv_x),
                                   _ptr(recv_topk_idx), _ptr(recv_topk_weights), _ptr(recv_src), _stream(stream)),
           "ep_dispatch_ranks")


def ep_layout_dispatch_ranks(x: torch.Tensor, routing: Routing, layout: Layout, rank_layout: RankLayout,
                             recv_x: torch.Tensor, *, num_recv_rows=None, topk_weights=None, recv_topk_idx=None,
                             recv_topk_weights=None, recv_src=None, stream=None) -> None:
    """ep_get_layout + ep_get_rank_layout + ep_dispatch_ranks in one call;
    the rows are loaded while the rank layout runs."""
    rows = recv_x.shape[0] if num_recv_rows is None else int(num_recv_rows)
    _check(lib().ep_layout_dispatch_ranks(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                          ctypes.byref(rank_layout.desc), rows, _ptr(topk_weights), _ptr(recv_x),
                                          _ptr(recv_topk_idx), _ptr(recv_topk_weights), _ptr(recv_src),
                                          _stream(stream)), "ep_layout_dispatch_ranks")


def ep_combine_ranks(y: torch.Tensor, routing: Routing, layout: Layout, rank_layout: RankLayout, out: torch.Tensor,
                     *, num_y_rows=None, stream=None) -> None:
    """out dtype follows `out` (bfloat16 or float32)."""
    rows = y.shape[0] if num_y_rows is None else int(num_y_rows)
    _check(lib().ep_combine_ranks(_ptr(y), y.shape[1], rows, ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                  ctypes.byref(rank_layout.desc), _ptr(out), _dtype_code(out), _stream(stream)),
           "ep_combine_ranks")


# ------------------------------------------------------ per rank over peer memory
EP_IPC_HANDLE_BYTES = 64


def ep_peer_alloc(nbytes: int) -> tuple[int, bytes]:
    """Device memory other processes can map: (address, IPC handle)."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    _check(lib().ep_peer_alloc(int(nbytes), ctypes.byref(ptr), handle), "ep_peer_alloc")
    return int(ptr.value), handle.raw


def ep_peer_free(ptr: int) -> None:
    _check(lib().ep_peer_free(ctypes.c_void_p(ptr)), "ep_peer_free")


def ep_peer_open(handle: bytes) -> int:
    """Map another process's ep_peer_alloc buffer; returns its address here."""
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has %d bytes, got %d" % (EP_IPC_HANDLE_BYTES, len(handle)))
    ptr = ctypes.c_void_p()
    _check(lib().ep_peer_open(ctypes.create_string_buffer(handle, EP_IPC_HANDLE_BYTES), ctypes.byref(ptr)),
           "ep_peer_open")
    return int(ptr.value)


def ep_peer_close(ptr: int) -> None:
    _check(lib().ep_peer_close(ctypes.c_void_p(ptr)), "ep_peer_close")


class _CudaArray:
    """A device address, shape and element type in the CUDA array interface,
    for torch.as_tensor to view without a copy."""

    def __init__(self, ptr: int, shape: tuple, typestr: str):
        self.__cuda_array_interface__ = {"data": (int(ptr), False), "shape": tuple(shape), "typestr": typestr,
                                         "strides": None, "version": 3}


_TYPESTR = {torch.bfloat16: "<i2", torch.int16: "<i2", torch.int32: "<i4", torch.int64: "<i8",
            torch.float32: "<f4", torch.uint8: "|u1"}


def device_view(ptr: int, shape: tuple, dtype: torch.dtype, device) -> torch.Tensor:
    """A tensor over device memory the library handed out (no copy; the
    memory must outlive the tensor)."""
    t = torch.as_tensor(_CudaArray(ptr, shape, _TYPESTR[dtype]), device=device)
    return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t


class Peers:
    """The descriptor of ep_peers_t over device tables of R addresses each
    (int64 tensors on this rank's GPU)."""

    def __init__(self, rank: int, capacity: int, recv_x, y, rank_counts, recv_topk_idx=None,
                 recv_topk_weights=None, recv_src=None):
        tables = dict(recv_x=recv_x, y=y, rank_counts=rank_counts, recv_topk_idx=recv_topk_idx,
                      recv_topk_weights=recv_topk_weights, recv_src=recv_src)
        for name, t in tables.items():
            if t is not None and (t.dtype != torch.int64 or t.dim() != 1 or t.shape[0] != recv_x.shape[0]):
                raise ValueError("peer table %s must be an int64 vector of one address per rank" % name)
        self.tables = tables  # keeps the tables alive
        self.desc = PeersDesc(recv_x.shape[0], rank, capacity, *(None if tables[n] is None else tables[n].data_ptr()
                                                                for n in ("recv_x", "recv_topk_idx",
                                                                          "recv_topk_weights", "recv_src", "y",
                                                                          "rank_counts")))


def ep_peer_publish_counts(routing: Routing, layout: Layout, peers: Peers, stream=None) -> None:
    _check(lib().ep_peer_publish_counts(ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                        ctypes.byref(peers.desc), _stream(stream)), "ep_peer_publish_counts")


def ep_dispatch_peers(x: torch.Tensor, routing: Routing, layout: Layout, rank_layout: RankLayout, peers: Peers, *,
                      topk_weights=None, stream=None) -> None:
    _check(lib().ep_dispatch_peers(_ptr(x), x.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                   ctypes.byref(rank_layout.desc), _ptr(topk_weights), ctypes.byref(peers.desc),
                                   _stream(stream)), "ep_dispatch_peers")


def ep_combine_peers(routing: Routing, layout: Layout, rank_layout: RankLayout, peers: Peers, out: torch.Tensor, *,
                     stream=None) -> None:
    """out dtype follows `out` (bfloat16 or float32)."""
    _check(lib().ep_combine_peers(out.shape[1], ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                  ctypes.byref(rank_layout.desc), ctypes.byref(peers.desc), _ptr(out),
                                  _dtype_code(out), _stream(stream)), "ep_combine_peers")


def ep_get_layout_no_alloc(routing: Routing, layout: Layout, device_error_flags: torch.Tensor | None = None,
                           stream=None) -> Layout:
    """The layout without a caller workspace (for callers that cannot
    allocate): layout.workspace is ignored; the library's fixed scratch
    array is used.  device_error_flags: optional one-element int32/uint32
    device tensor that receives the EP_DEVERR_* bits of this call."""
    _check(lib().ep_get_layout_no_alloc(ctypes.byref(routing.desc), ctypes.byref(layout.desc),
                                        _ptr(device_error_flags), _stream(stream)), "ep_get_layout_no_alloc")
    return layout


def ep_version() -> int:
    return int(lib().ep_version())
