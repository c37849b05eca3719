"""Expert parallelism across GPUs: the exchange between the per-rank dispatch
and the rank-level combine.

The DeepEP-Ascend README ("Normal Mode (Prefill / Training)"; the strategy
table's ``alltoall`` entry, a ``torch.distributed`` all-to-all-v) sends each
token once to every rank that holds one of its experts and brings one
partial row per (token, rank) back.  Here the W processes of a process group
are those ranks: rank r owns experts [r*E/W, (r+1)*E/W), the logical ranks of
the layout are the W processes, and the step is

    ep_get_layout (R = W) -> ep_get_rank_layout -> ep_dispatch_ranks
        send rows grouped by destination rank, each with its K top-k entries
        seen by that rank (local expert id or -1, gate weight or 0)
    counts exchange            rows each rank sends to each rank
    row exchange               all-to-all-v of the rows and their entries
        -> every rank holds the rows of all ranks' tokens for its experts,
           source rank 0's rows first, each source's rows in token order
    local experts              per received row: sum over its local entries
                               (ascending k) of weight * expert(row), fp32
                               fmaf chain, one bf16 row (the same layout ->
                               dispatch -> combine path with R = 1)
    reverse row exchange       the partial rows go back to their source ranks,
                               landing in the send order
    ep_combine_ranks           out[t] = sum over the token's ranks, ascending,
                               fp32 additions from 0

so a token's result is the two-level sum (per rank, then over ranks) that
DeepEP's combine forms.  The transfers are ``torch.distributed``
all-to-all-v calls (NCCL over NVLink between GPUs, gloo between CPU
processes; device tensors are staged through host memory for gloo): the
counts on the host size the receive buffers, which is the one host
synchronisation of a step.  bf16 rows travel as their 16-bit patterns.  No
transfer here hands a peer's memory to a library kernel.

The compute steps are the CUDA kernels of the C ABI (``CudaRowOps``); the
exchange itself takes any object with the same three methods, so that the
protocol can be exercised on CPU processes.

``PeerExpertParallel`` runs the same step with the transfers fused into the
kernels over peer memory instead of a library all-to-all between them: the
dispatch (ep_dispatch_peers) stores each (token, rank) row straight into
that rank's receive buffer, mapped into this process through CUDA IPC, and
the combine (ep_combine_peers) reads the partial rows straight from the
ranks' buffers.  No kernel waits for another rank: the phases are separated
by a stream synchronisation and a process-group barrier.  Its memory and
compute steps likewise come from an object (``CudaPeerOps``) that a test can
replace.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


# ------------------------------------------------------------------ protocol
def _host_transport(t: torch.Tensor, group) -> bool:
    """gloo moves host tensors only: device tensors are staged through host
    memory (a process group of CPU processes sharing a GPU, or a test)."""
    return t.is_cuda and dist.get_backend(group) == "gloo"


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """send_counts[j] = rows this rank sends to rank j (int64 [W]); returns
    recv_counts[i] = rows rank i sends to this rank."""
    if send_counts.dtype != torch.int64 or send_counts.dim() != 1:
        raise TypeError("send_counts must be an int64 vector of one entry per rank")
    wire = send_counts.cpu() if _host_transport(send_counts, group) else send_counts
    recv_counts = torch.empty_like(wire)
    dist.all_to_all_single(recv_counts, wire, group=group)
    return recv_counts.to(send_counts.device)


def exchange_rows(send: torch.Tensor, send_splits: list[int], recv_splits: list[int], group=None) -> torch.Tensor:
    """All-to-all-v of the rows of `send` (rows for rank 0 first, then rank 1,
    ...; send_splits[j] rows for rank j).  Returns the received rows, rank 0's
    first, recv_splits[i] rows from rank i.  bf16 rows travel as their bit
    patterns, two values per int32 (every backend moves int32)."""
    if sum(send_splits) != send.shape[0]:
        raise ValueError("send splits cover %d rows, the buffer has %d" % (sum(send_splits), send.shape[0]))
    send = send.contiguous()
    bf16 = send.dtype == torch.bfloat16
    if bf16 and send.shape[-1] % 2 != 0:
        raise ValueError("bf16 rows travel in pairs: the last dimension must be even")
    wire = send.view(torch.int32) if bf16 else send
    staged = _host_transport(wire, group)
    if staged:
        wire = wire.cpu()
    recv = torch.empty((sum(recv_splits),) + tuple(wire.shape[1:]), dtype=wire.dtype, device=wire.device)
    dist.all_to_all_single(recv, wire, output_split_sizes=list(recv_splits),
                           input_split_sizes=list(send_splits), group=group)
    if staged:
        recv = recv.to(send.device)
    return recv.view(torch.bfloat16) if bf16 else recv


@dataclass
class SendRows:
    """What a rank's per-rank dispatch produced: rows for rank j at
    [offsets[j], offsets[j+1]) of x / topk_idx / topk_weights, and the handle
    its rank-level combine needs."""
    x: torch.Tensor             # bf16 [N_send, H]
    topk_idx: torch.Tensor      # int64 [N_send, K]: local expert id on the destination rank, or -1
    topk_weights: torch.Tensor  # fp32 [N_send, K]
    counts: list[int]           # rows per destination rank
    handle: object              # passed back to combine_ranks


@dataclass
class Received:
    """The rows this rank's experts process, source rank 0's first."""
    x: torch.Tensor
    topk_idx: torch.Tensor
    topk_weights: torch.Tensor
    recv_counts: list[int]
    send: SendRows


class ExpertParallel:
    """The exchange of one process group (W ranks; rank r owns experts
    [r*E/W, (r+1)*E/W)).  ``ops`` runs the compute steps (CudaRowOps by
    default)."""

    def __init__(self, num_experts: int, group=None, ops=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if num_experts % self.world != 0:
            raise ValueError("%d experts do not split over %d ranks" % (num_experts, self.world))
        self.num_experts = num_experts
        self.local_experts = num_experts // self.world
        self.ops = ops if ops is not None else CudaRowOps()

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor) -> Received:
        send = self.ops.rank_rows(x, topk_idx, topk_weights, self.num_experts, self.world)
        if len(send.counts) != self.world:
            raise ValueError("rank_rows returned %d counts for %d ranks" % (len(send.counts), self.world))
        send_counts = torch.tensor(send.counts, dtype=torch.int64, device=x.device)
        recv_counts = exchange_counts(send_counts, self.group).tolist()
        rx = exchange_rows(send.x, send.counts, recv_counts, self.group)
        ridx = exchange_rows(send.topk_idx, send.counts, recv_counts, self.group)
        rw = exchange_rows(send.topk_weights, send.counts, recv_counts, self.group)
        return Received(rx, ridx, rw, recv_counts, send)

    def experts(self, recv: Received, expert_fn) -> torch.Tensor:
        """One bf16 row per received row: the fmaf chain over its local
        entries (ascending k) of weight * expert_fn output."""
        return self.ops.local_experts(recv.x, recv.topk_idx, recv.topk_weights, self.local_experts, expert_fn)

    def combine(self, y: torch.Tensor, recv: Received, out_dtype=torch.bfloat16) -> torch.Tensor:
        """Send the partial rows back and reduce them per token (ascending
        rank, fp32 additions)."""
        if y.shape[0] != sum(recv.recv_counts):
            raise ValueError("y has %d rows, %d were received" % (y.shape[0], sum(recv.recv_counts)))
        back = exchange_rows(y, recv.recv_counts, recv.send.counts, self.group)
        return self.ops.combine_ranks(back, recv.send.handle, out_dtype)


# ------------------------------------------------------------ compute steps
class CudaRowOps:
    """The compute steps on the GPU, through the C ABI."""

    def __init__(self, stream=None):
        from . import binding as B

        self.B = B
        self.stream = stream

    def rank_rows(self, x, topk_idx, topk_weights, num_experts, world) -> SendRows:
        B = self.B
        routing = B.Routing.topk(topk_idx, num_experts, world)
        layout = B.Layout(routing, device=x.device)
        B.ep_get_layout(routing, layout, stream=self.stream)
        rl = B.RankLayout(routing, device=x.device)
        B.ep_get_rank_layout(routing, layout, rl, stream=self.stream)
        counts = layout.num_tokens_per_rank.tolist()  # sizes the send buffer
        n = sum(counts)
        H, K = x.shape[1], topk_idx.shape[1]
        sx = torch.empty((n, H), dtype=torch.bfloat16, device=x.device)
        sidx = torch.empty((n, K), dtype=torch.int64, device=x.device)
        sw = torch.empty((n, K), dtype=torch.float32, device=x.device)
        B.ep_dispatch_ranks(x, routing, layout, rl, sx, topk_weights=topk_weights, recv_topk_idx=sidx,
                            recv_topk_weights=sw, stream=self.stream)
        return SendRows(sx, sidx, sw, counts, (routing, layout, rl))

    def local_experts(self, x, topk_idx, topk_weights, local_experts, expert_fn, out=None):
        B = self.B
        n, H = x.shape
        y = torch.empty((n, H), dtype=torch.bfloat16, device=x.device) if out is None else out
        if n == 0:
            return y
        routing = B.Routing.topk(topk_idx, local_experts, 1)
        layout = B.Layout(routing, device=x.device, report_num_valid=True)
        B.ep_get_layout(routing, layout, stream=self.stream)
        rows = torch.empty((max(layout.num_valid, 1), H), dtype=torch.bfloat16, device=x.device)
        B.ep_dispatch(x, routing, layout, rows, num_recv_rows=layout.num_valid, stream=self.stream)
        out_rows = expert_fn(rows[:layout.num_valid], layout.expert_offsets)
        B.ep_combine(out_rows, routing, layout, topk_weights, y, num_y_rows=layout.num_valid, stream=self.stream)
        return y

    def combine_ranks(self, back, handle, out_dtype):
        B = self.B
        routing, layout, rl = handle
        out = torch.empty((routing.T, back.shape[1]), dtype=out_dtype, device=back.device)
        B.ep_combine_ranks(back, routing, layout, rl, out, num_y_rows=back.shape[0], stream=self.stream)
        if B.ep_get_device_error(layout) != 0:
            raise B.EPError(B.EP_ERR_BAD_INDEX, "device error flagged in the exchange step")
        return out


# ------------------------------------------------------ over peer memory
def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


@dataclass
class PeerReceived:
    """The rows this rank's experts process (views of its receive buffers),
    source rank 0's first, and what its combine needs."""
    x: torch.Tensor
    topk_idx: torch.Tensor
    topk_weights: torch.Tensor
    src: torch.Tensor
    recv_counts: list[int]
    handle: object


class PeerExpertParallel:
    """The same exchange with the all-to-all fused into the kernels over
    peer memory (ep_dispatch_peers / ep_combine_peers): the dispatch stores
    each (token, rank) row straight into that rank's receive buffer and the
    combine reads the partial rows straight from the ranks' buffers.

    Every rank allocates one block of memory that the other processes map
    (the handles travel by all_gather_object): receive rows, their top-k
    entries and source tokens, the partial rows and the [W, W] counts
    matrix, each at the same offset in every rank's block.  ``capacity``
    bounds the rows a rank can receive.  Between the phases of a step every
    rank completes its own work and passes a process-group barrier
    (``barrier``), so no kernel ever waits for another rank:

        layout -> rank layout -> publish counts | dispatch | experts | combine

    A step's results equal ExpertParallel's (all-to-all-v) bit for bit.
    ``ops`` holds the memory and the compute steps (CudaPeerOps by default)."""

    BUFFERS = ("recv_x", "y", "recv_topk_idx", "recv_topk_weights", "recv_src", "rank_counts")

    def __init__(self, num_experts: int, hidden: int, num_topk: int, capacity: int, group=None, device=None,
                 barrier=None, ops=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if num_experts % self.world != 0:
            raise ValueError("%d experts do not split over %d ranks" % (num_experts, self.world))
        if hidden % 8 != 0:
            raise ValueError("rows travel in 16-byte vectors: hidden must be a multiple of 8")
        self.num_experts, self.hidden, self.num_topk = num_experts, hidden, num_topk
        self.local_experts = num_experts // self.world
        self.capacity = int(capacity)
        self.ops = ops if ops is not None else CudaPeerOps(device)
        self._barrier_fn = barrier
        W, C, H, K = self.world, self.capacity, hidden, num_topk
        shapes = dict(recv_x=((C, H), torch.bfloat16), y=((C, H), torch.bfloat16),
                      recv_topk_idx=((C, K), torch.int64), recv_topk_weights=((C, K), torch.float32),
                      recv_src=((C,), torch.int32), rank_counts=((W, W), torch.int32))
        self.offsets, total = {}, 0
        for name in self.BUFFERS:
            shape, dtype = shapes[name]
            self.offsets[name] = total
            n = torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size()
            total += _align(max(n, 1))
        self._own, handle = self.ops.alloc(total)
        self._opened = []
        bases = []
        try:
            handles = [None] * W
            dist.all_gather_object(handles, handle, group=group)
            for r in range(W):
                if r == self.rank:
                    bases.append(self._own)
                else:
                    base = self.ops.open(handles[r])
                    self._opened.append(base)
                    bases.append(base)
        except Exception:  # no step has run: unmap what was mapped, free this rank's block
            self._release()
            self.ops.free(self._own)
            self._own = None
            raise
        self.peers = self.ops.peers(self.rank, C, {name: [b + off for b in bases]
                                                   for name, off in self.offsets.items()})
        for name in self.BUFFERS:
            shape, dtype = shapes[name]
            setattr(self, name, self.ops.view(self._own + self.offsets[name], shape, dtype))
        self._barrier()  # every rank has mapped every block before any store

    def _barrier(self):
        self.ops.sync()
        if self._barrier_fn is not None:
            self._barrier_fn()
        else:
            dist.barrier(group=self.group)

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor) -> PeerReceived:
        """The rows every rank sends here land in this rank's buffers; the
        returned tensors are views of them, valid until the next dispatch."""
        if x.shape[1] != self.hidden or topk_idx.shape[1] != self.num_topk:
            raise ValueError("x is [T, %d] and topk_idx [T, %d] for this exchange" % (self.hidden, self.num_topk))
        handle = self.ops.layout(topk_idx, self.num_experts, self.world)
        self.ops.publish(handle, self.peers)
        self._barrier()
        self.ops.dispatch(x, topk_weights, handle, self.peers)
        self._barrier()
        recv_counts = [int(c) for c in self.rank_counts[:, self.rank].tolist()]
        n = sum(recv_counts)
        if n > self.capacity:
            raise OverflowError("rank %d receives %d rows, the buffers hold %d" % (self.rank, n, self.capacity))
        return PeerReceived(self.recv_x[:n], self.recv_topk_idx[:n], self.recv_topk_weights[:n], self.recv_src[:n],
                            recv_counts, handle)

    def experts(self, recv: PeerReceived, expert_fn) -> torch.Tensor:
        """The partial rows, written into this rank's y buffer."""
        n = recv.x.shape[0]
        return self.ops.local_experts(recv.x, recv.topk_idx, recv.topk_weights, self.local_experts, expert_fn,
                                      out=self.y[:n])

    def combine(self, y: torch.Tensor, recv: PeerReceived, out_dtype=torch.bfloat16) -> torch.Tensor:
        n = recv.x.shape[0]
        if tuple(y.shape) != (n, self.hidden):
            raise ValueError("y is %s, %d rows were received" % (tuple(y.shape), n))
        if y.data_ptr() != self.y.data_ptr():
            self.y[:n].copy_(y)
        self._barrier()
        return self.ops.combine(recv.handle, self.peers, self.hidden, out_dtype)

    def _release(self):
        for base in self._opened:
            self.ops.close(base)
        self._opened = []

    def close(self):
        """Unmap the peers' blocks and free this rank's (collective)."""
        if self._own is None:
            return
        self._barrier()  # no rank still reads or writes another's block
        self._release()
        self._barrier()  # every mapping of this block is gone
        for name in self.BUFFERS:
            setattr(self, name, None)
        self.ops.free(self._own)
        self._own = None


class CudaPeerOps:
    """The peer path's memory (ep_peer_alloc / open / close / free, device
    tables) and compute steps (layout, counts publish, dispatch, local
    experts, combine) on the GPU, through the C ABI."""

    def __init__(self, device=None):
        from . import binding as B

        self.B = B
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.rows = CudaRowOps()

    # memory
    def alloc(self, nbytes: int):
        return self.B.ep_peer_alloc(nbytes)

    def open(self, handle: bytes) -> int:
        return self.B.ep_peer_open(handle)

    def close(self, base: int) -> None:
        self.B.ep_peer_close(base)

    def free(self, base: int) -> None:
        self.B.ep_peer_free(base)

    def view(self, addr: int, shape, dtype):
        return self.B.device_view(addr, shape, dtype, self.device)

    def peers(self, rank: int, capacity: int, tables: dict):
        t = {name: torch.tensor(addrs, dtype=torch.int64, device=self.device) for name, addrs in tables.items()}
        return self.B.Peers(rank, capacity, t["recv_x"], t["y"], t["rank_counts"], recv_topk_idx=t["recv_topk_idx"],
                            recv_topk_weights=t["recv_topk_weights"], recv_src=t["recv_src"])

    def sync(self) -> None:
        torch.cuda.current_stream(self.device).synchronize()

    # compute steps
    def layout(self, topk_idx, num_experts, world):
        B = self.B
        routing = B.Routing.topk(topk_idx, num_experts, world)
        layout = B.Layout(routing, device=topk_idx.device)
        B.ep_get_layout(routing, layout)
        rl = B.RankLayout(routing, device=topk_idx.device)
        B.ep_get_rank_layout(routing, layout, rl)
        return routing, layout, rl

    def publish(self, handle, peers) -> None:
        routing, layout, _ = handle
        self.B.ep_peer_publish_counts(routing, layout, peers)

    def dispatch(self, x, topk_weights, handle, peers) -> None:
        routing, layout, rl = handle
        self.B.ep_dispatch_peers(x, routing, layout, rl, peers, topk_weights=topk_weights)

    def local_experts(self, x, topk_idx, topk_weights, local_experts, expert_fn, out):
        return self.rows.local_experts(x, topk_idx, topk_weights, local_experts, expert_fn, out=out)

    def combine(self, handle, peers, hidden, out_dtype):
        B = self.B
        routing, layout, rl = handle
        out = torch.empty((routing.T, hidden), dtype=out_dtype, device=self.device)
        B.ep_combine_peers(routing, layout, rl, peers, out)
        if B.ep_get_device_error(layout) != 0:
            raise B.EPError(B.EP_ERR_OVERFLOW, "device error flagged in the peer exchange")
        return out
