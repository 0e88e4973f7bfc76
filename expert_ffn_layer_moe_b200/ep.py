"""Expert parallelism: the experts split over G ranks, token rows exchanged all-to-all.

[MoE-latency] "跨 GPU 时,激活要出门": when the experts do not fit one GPU they are
placed on different GPUs; a token whose chosen expert lives on another GPU sends its
activation row there and gets the expert's output back, every rank sending to and
receiving from every other rank at once (all-to-all), in every MoE layer.  Section
"最慢的 GPU 决定这一步": a step lasts as long as its slowest rank, so the per-rank
assignment counts and phase times of each step are what to record (``EPStats``).

Layout: rank r holds experts [r*L, (r+1)*L), L = E/G (its slices of W1, W3 and W2).
Each rank routes and permutes its own token batch with the library's kernels.  Its
permuted rows x_perm are sorted by expert, so the rows bound for rank r form one
contiguous range.  Then:

1. all-gather of the per-expert counts [G, E] -- the exchange sizes, read on the host
   (the one host synchronisation of the step);
2. all-to-all of the rows: rank r receives, from each source in rank order, that
   source's rows for r's experts, sorted by expert;
3. a row scatter into expert-major order (inside an expert: source rank, then the
   source's order -- stable, so the result is deterministic), the local grouped GEMMs
   (SwiGLU W1/W3, then W2 with fp32 out);
4. a row scatter back to the received order and the all-to-all back (fp32 rows);
5. the combine on the source rank, in pick order: the same sums, in the same order,
   as the one-device layer computes.

The plan and the exchange are device-independent; the local steps (the expert FFN and
the row scatter) are passed in.  ``moe_layer_forward_ep`` runs the library's kernels on
CUDA tensors over an NCCL process group.  The rows cross the wire as raw 32-bit words.

Two transports move the rows (steps 2 and 4):
  * ``CollectiveTransport`` -- torch.distributed all-to-all (NCCL between GPUs, gloo on
    CPU);
  * ``PeerCopyTransport`` -- every rank copies its rows straight into the receiving
    ranks' buffers, one copy per contiguous range, then all ranks meet at a host
    barrier.  On GPUs the buffers are exported once through CUDA IPC and the copies
    are the library's moe_copy_async (``CudaPeers``); the receive order is the
    all-to-all's (source rank, then the source's order), so both transports give the
    same bits.

Host synchronisations per step: the counts all-gather (the plan is made on the host),
plus, with peer copies, one per exchange (a rank's copies must have landed before the
barrier releases the receivers).  Per-phase timing (``stats``) adds one per phase.
"""
from __future__ import annotations

import dataclasses
import time
from typing import Callable, List, Optional

import numpy as np
import torch
import torch.distributed as dist


@dataclasses.dataclass
class ExchangePlan:
    """Sizes and row maps of one rank's exchange (all rows counted in [R, H] rows)."""
    send_splits: List[int]      # rows sent to each rank, in rank order (ranges of x_perm)
    recv_splits: List[int]      # rows received from each rank
    local_offsets: np.ndarray   # [L+1] int32: row offsets of the local experts, expert-major
    recv_to_local: np.ndarray   # [sum(recv_splits)] int32: expert-major row of each received row
    local_to_recv: np.ndarray   # the inverse permutation


@dataclasses.dataclass
class EPStats:
    """One step on one rank: assignments sent and received, and host-clock phase times
    (seconds; each phase ends with a device synchronisation)."""
    rows_sent: int
    rows_received: int
    seconds: dict


def exchange_plan(counts_all, rank: int) -> ExchangePlan:
    """The plan of rank `rank` from every rank's per-expert row counts [G, E]."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    G, E = counts_all.shape
    if E % G != 0:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    if not 0 <= rank < G:
        raise ValueError("rank outside the group")
    L = E // G
    per_pair = counts_all.reshape(G, G, L).sum(axis=2)       # [source, destination] rows
    loc = counts_all[:, rank * L:(rank + 1) * L]              # [source, local expert] rows
    local_offsets = np.concatenate([[0], np.cumsum(loc.sum(axis=0))]).astype(np.int64)
    earlier = np.cumsum(loc, axis=0) - loc                    # rows of expert e from earlier sources
    parts = [np.arange(loc[s, e], dtype=np.int64) + local_offsets[e] + earlier[s, e]
             for s in range(G) for e in range(L)]
    recv_to_local = np.concatenate(parts) if parts else np.zeros(0, np.int64)
    local_to_recv = np.empty_like(recv_to_local)
    local_to_recv[recv_to_local] = np.arange(recv_to_local.size)
    return ExchangePlan([int(v) for v in per_pair[rank, :]], [int(v) for v in per_pair[:, rank]],
                        local_offsets.astype(np.int32), recv_to_local.astype(np.int32),
                        local_to_recv.astype(np.int32))


def _words(t: torch.Tensor) -> torch.Tensor:
    """A row-major tensor as 32-bit words per row (the wire format of the exchange):
    2-byte values travel in pairs, 8-byte values as two words each."""
    if t.dtype in (torch.int32, torch.float32):
        return t
    return t.view(torch.int32)


def _bits(t: torch.Tensor) -> torch.Tensor:
    """The same bytes as int32 words per row (so copies between buffers never convert)."""
    return t if t.dtype == torch.int32 else t.view(torch.int32)


def _sync(dev):
    if dev.type == "cuda":
        torch.cuda.synchronize(dev)


class CollectiveTransport:
    """Rows exchanged by torch.distributed all-to-all (NCCL between GPUs, gloo on CPU)."""
    name = "collective"

    def __init__(self, group=None):
        self.group = group

    def dispatch(self, rows: torch.Tensor, plan: ExchangePlan, counts_all) -> torch.Tensor:
        recv = torch.empty((sum(plan.recv_splits), rows.shape[1]), dtype=rows.dtype, device=rows.device)
        dist.all_to_all_single(_words(recv), _words(rows.contiguous()), plan.recv_splits, plan.send_splits,
                               group=self.group)
        return recv

    def back(self, y_recv: torch.Tensor, plan: ExchangePlan, counts_all, y: torch.Tensor) -> None:
        sent = sum(plan.send_splits)
        dist.all_to_all_single(_words(y[:sent]), _words(y_recv), plan.send_splits, plan.recv_splits,
                               group=self.group)


def peer_offsets(counts_all, rank: int):
    """Where rank `rank`'s copies go, from every rank's per-expert counts [G, E]:
    (send, back), each a list over the other ranks d of (source row, destination row,
    rows).  send: rank's rows for d's experts (a range of its x_perm) land in d's
    receive buffer after the rows of the sources before it -- the all-to-all's
    receive order.  back: the outputs of the rows rank received from d go back into
    d's return buffer at the position of that range in d's own x_perm."""
    counts_all = np.asarray(counts_all, dtype=np.int64)
    G, E = counts_all.shape
    L = E // G
    per_pair = counts_all.reshape(G, G, L).sum(axis=2)          # [source, destination] rows
    send_start = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(per_pair, axis=1)], axis=1)
    recv_start = np.concatenate([np.zeros((1, G), np.int64), np.cumsum(per_pair, axis=0)], axis=0)
    send = [(int(send_start[rank, d]), int(recv_start[rank, d]), int(per_pair[rank, d])) for d in range(G)]
    back = [(int(recv_start[d, rank]), int(send_start[d, rank]), int(per_pair[d, rank])) for d in range(G)]
    return send, back


class PeerCopyTransport:
    """Rows exchanged by copies into the other ranks' buffers.

    Each rank holds a receive buffer (capacity: every rank's rows, G * max_rows) and a
    return buffer (its own rows, max_rows), shared with the other ranks once through
    `peers`.  dispatch: each rank copies its row range for rank d into d's receive
    buffer at that range's place in the all-to-all order; after `peers.fence()` (this
    rank's copies have completed, then a barrier) the receive buffer holds what an
    all-to-all would have delivered.  back: the same, with the outputs into the
    senders' return buffers.  A rank's buffers are overwritten by the others only
    after the next fence, by which time its own reads of the previous step have
    completed (its stream is synchronised before it enters the barrier)."""
    name = "peer_copy"

    def __init__(self, peers, max_rows: int, words_in: int, words_out: int):
        self.peers = peers
        G = peers.world
        self.max_rows = max_rows
        self.recv_buf = peers.alloc(G * max_rows, words_in)
        self.back_buf = peers.alloc(max_rows, words_out)
        self.recv_peer = peers.share(self.recv_buf)
        self.back_peer = peers.share(self.back_buf)

    def dispatch(self, rows: torch.Tensor, plan: ExchangePlan, counts_all) -> torch.Tensor:
        send, _ = peer_offsets(counts_all, self.peers.rank)
        w = _bits(rows.contiguous())
        if w.shape[0] > self.max_rows or w.shape[1] != self.recv_buf.shape[1]:
            raise ValueError("rows exceed the peer buffers")
        for d, (src, dst, n) in enumerate(send):
            if n:
                self.peers.copy(self.recv_peer[d], dst, w[src:src + n])
        self.peers.fence()
        n_recv = sum(plan.recv_splits)
        return self.recv_buf[:n_recv].view(rows.dtype)

    def back(self, y_recv: torch.Tensor, plan: ExchangePlan, counts_all, y: torch.Tensor) -> None:
        _, back = peer_offsets(counts_all, self.peers.rank)
        w = _bits(y_recv.contiguous())
        if w.shape[1] != self.back_buf.shape[1]:
            raise ValueError("output rows do not match the return buffer")
        for d, (src, dst, n) in enumerate(back):
            if n:
                self.peers.copy(self.back_peer[d], dst, w[src:src + n])
        self.peers.fence()
        sent = sum(plan.send_splits)
        _bits(y)[:sent].copy_(self.back_buf[:sent])  # bit copy (both int32 views)

    def close(self):
        self.peers.close()


class CudaPeers:
    """Peer buffers on the GPUs of one node: buffers exported once through CUDA IPC
    (moe_ipc_export / moe_ipc_import), rows moved by moe_copy_async on the current
    stream, and a fence = this rank's stream synchronised, then a barrier of the
    group.  A rank's own buffer is used directly."""

    def __init__(self, group=None, device=None):
        from expert_ffn_layer_moe_b200 import moe
        self.moe = moe
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.bases = {}  # (rank, handle) -> the imported allocation's base pointer (one mapping each)

    def alloc(self, rows: int, words: int) -> torch.Tensor:
        return torch.empty((max(1, rows), words), dtype=torch.int32, device=self.device)

    def share(self, buf: torch.Tensor):
        """-> for every rank, (pointer, row bytes) of its buffer as this process sees it."""
        mine = self.moe.moe_ipc_export(buf)
        allh = [None] * self.world
        dist.all_gather_object(allh, mine, group=self.group)
        rb = buf.shape[1] * buf.element_size()
        out = []
        for r, (h, off) in enumerate(allh):
            if r == self.rank:
                out.append((buf.data_ptr(), rb))
            else:
                # two buffers may share one allocation of the other process: map it once
                if (r, h) not in self.bases:
                    self.bases[(r, h)] = self.moe.moe_ipc_import(h, 0)
                out.append((self.bases[(r, h)] + off, rb))
        return out

    def copy(self, dst, row: int, src: torch.Tensor) -> None:
        ptr, rb = dst
        self.moe.moe_copy_async(ptr + row * rb, src.data_ptr(), src.numel() * src.element_size())

    def fence(self) -> None:
        torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)

    def close(self) -> None:
        torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)  # no rank still copies into a mapping being closed
        for base in self.bases.values():
            self.moe.moe_ipc_close(base, 0)
        self.bases = {}


def exchange_ffn(x_perm: torch.Tensor, counts: torch.Tensor, E: int,
                 local_ffn: Callable[[torch.Tensor, torch.Tensor], torch.Tensor],
                 scatter_rows: Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor],
                 group=None, stats: Optional[list] = None, transport=None):
    """Steps 1-4: x_perm [R, H] (this rank's rows, sorted by expert) and counts [E] ->
    y [R, H], row r the output of x_perm[r]'s expert, computed on that expert's rank.

    local_ffn(x_loc, local_offsets) -> y_loc runs the local experts on expert-major rows;
    scatter_rows(src, dst_row, dst) sets dst[dst_row[i]] = src[i].  transport moves the
    rows (default: CollectiveTransport(group)).  With `stats` each phase ends with a
    device synchronisation and its host time is recorded.  Returns (y, plan)."""
    transport = transport or CollectiveTransport(group)
    G = dist.get_world_size(group)
    rank = dist.get_rank(group)
    dev = x_perm.device
    timed = stats is not None
    t0 = time.perf_counter()
    gathered = [torch.empty_like(counts) for _ in range(G)]
    dist.all_gather(gathered, counts.contiguous(), group=group)
    counts_all = torch.stack(gathered).cpu().numpy()   # the step's one host read of device data
    plan = exchange_plan(counts_all, rank)
    t1 = time.perf_counter()
    R, H = x_perm.shape
    sent = sum(plan.send_splits)  # rows with a valid expert: the first `sent` rows of x_perm
    if sent > R:
        raise ValueError("counts exceed the permuted rows")
    recv = transport.dispatch(x_perm[:sent], plan, counts_all)
    if timed:
        _sync(dev)
    t2 = time.perf_counter()
    x_loc = torch.empty_like(recv)
    scatter_rows(recv, torch.from_numpy(plan.recv_to_local).to(dev), x_loc)
    y_loc = local_ffn(x_loc, torch.from_numpy(plan.local_offsets).to(dev))
    y_recv = torch.empty_like(y_loc)
    scatter_rows(y_loc, torch.from_numpy(plan.local_to_recv).to(dev), y_recv)
    if timed:
        _sync(dev)
    t3 = time.perf_counter()
    # rows past `sent` (assignments without a valid expert) stay unwritten; the combine skips them
    y = torch.empty((R, y_loc.shape[1]), dtype=y_loc.dtype, device=dev)
    transport.back(y_recv, plan, counts_all, y)
    if timed:
        _sync(dev)
    t4 = time.perf_counter()
    if timed:
        stats.append(EPStats(sent, int(sum(plan.recv_splits)),
                             {"plan": t1 - t0, "dispatch": t2 - t1, "experts": t3 - t2, "combine_exchange": t4 - t3}))
    return y, plan


def local_experts(W: torch.Tensor, rank: int, G: int) -> torch.Tensor:
    """This rank's slice [L, ...] of an expert stack [E, ...] (a view)."""
    E = W.shape[0]
    if E % G != 0:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    L = E // G
    return W[rank * L:(rank + 1) * L]


def moe_layer_forward_ep(x: torch.Tensor, W_gate: torch.Tensor, W1_local: torch.Tensor, W3_local: torch.Tensor,
                         W2_local: torch.Tensor, k: int, bias: Optional[torch.Tensor] = None, group=None,
                         stats: Optional[list] = None, routing=None, transport=None) -> torch.Tensor:
    """The MoE layer with the experts split over the ranks of `group` (NCCL, one GPU per
    rank).  x [N,H] bf16 is this rank's batch; W_gate [H,E] fp32 is the whole router;
    W1_local, W3_local [L,I,H] and W2_local [L,H,I] bf16 are this rank's experts
    (``local_experts``).  transport moves the rows (CollectiveTransport by default, or a
    PeerCopyTransport over CudaPeers).  routing = (topk_idx [N,k] int32, topk_w [N,k] fp32) replaces
    the router's choice when given; an index outside [0,E) is skipped (its assignment
    adds nothing) and reported through the device error word.  Returns this rank's
    out [N,H] bf16."""
    from expert_ffn_layer_moe_b200 import moe
    G = dist.get_world_size(group)
    E = W_gate.shape[1]
    if W1_local.shape[0] * G != E:
        raise ValueError("local expert slices do not match E / world size")
    if routing is not None:
        idx, w = routing
    else:
        idx, w, _ = moe.moe_route(x, W_gate, k, bias=bias)
    p = moe.moe_permute(x, idx, E)

    def ffn(x_loc, offsets_loc):
        return moe.moe_expert_ffn(x_loc, offsets_loc, W1_local, W3_local, W2_local)

    y, _ = exchange_ffn(p["x_perm"], p["counts"], E, ffn, moe.moe_scatter_rows, group=group, stats=stats,
                        transport=transport)
    return moe.moe_combine(y, p["token_to_row"], w)
