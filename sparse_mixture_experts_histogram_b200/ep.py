"""Expert parallelism: the layer's E experts split over R ranks, one GPU each.

Rank q of R holds experts [q*E/R, (q+1)*E/R).  Every step of the data path
runs in the library's kernels (``moe_route``, ``moe_ep_dispatch``,
``moe_ep_expert_ffn``, ``moe_ep_combine``; include/moe.h).  This module owns
the per-rank buffers, maps every rank's receive and output buffers into its
peers, and orders the GPUs with three stream-ordered collectives per step:
an all-gather of the per-expert counts and two one-word all-reduces used as
barriers.  Nothing is copied to the host during a step.

``ExpertParallelLayer`` is the multi-process form (torch.distributed over
NCCL, one process per GPU).  ``EmulatedExpertParallel`` runs the same kernels
for R ranks on one GPU, rank after rank on one stream, where stream order
stands in for the collectives: it is how the path is checked and timed on a
single GPU.

Method: experts placed on several GPUs ("Mistral 8x7B SMoE architecture",
jsqmd.com, deployment section, problem 4); the per-expert gathering and
weighted index_add of "MoE" (theaiera.top, LLMs-from-scratch ch.10)
sec. 10.4, across ranks.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B


def expert_block(E: int, R: int, rank: int) -> tuple[int, int]:
    """[first, last) expert index owned by ``rank``."""
    if R < 1 or E % R:
        raise ValueError(f"E={E} is not a multiple of R={R}")
    El = E // R
    return rank * El, (rank + 1) * El


@dataclass
class _Rank:
    """Buffers of one rank for tokens of at most T_max rows."""
    recv_x: torch.Tensor      # [recv_rows, d] bf16 (peers store into it)
    recv_y: torch.Tensor      # [ksplit, recv_rows, d] fp32, or bf16 with ksplit 1 (peers read it)
    ws: torch.Tensor          # moe_ep_workspace_size bytes
    route_ws: torch.Tensor    # moe_workspace_size bytes (router)
    idx: torch.Tensor         # [T_max, k] int32
    w: torch.Tensor           # [T_max, k] fp32
    counts: torch.Tensor      # [E] int32
    pos: torch.Tensor         # [T_max, k] int32
    recv_offsets: torch.Tensor  # [E/R + 1] int32
    shared_off: torch.Tensor | None
    shared_y: torch.Tensor | None
    shared_ws: torch.Tensor | None


class _Plan:
    """Sizes shared by every rank of one expert-parallel layer."""

    def __init__(self, R, T_max, d, E, d_ff, k, d_ff_shared=0):
        if R < 1 or E % R:
            raise ValueError(f"E={E} is not a multiple of R={R}")
        self.R, self.T_max, self.d, self.E, self.d_ff, self.k = R, T_max, d, E, d_ff, k
        self.El = E // R
        self.d_ff_shared = d_ff_shared
        self.recv_rows = B.moe_ep_recv_rows(T_max, E, k, R)
        self.ws_bytes = B.moe_ep_workspace_size(T_max, d, E, d_ff, k, R)
        if self.recv_rows < 1 or self.ws_bytes == 0:
            raise B.MoEError(2, "expert-parallel sizes")
        # Rows an owner expects with balanced experts: every rank sends T*k
        # pairs, spread over R owners.
        self.rows_hint = max(1, T_max * k)
        self.ksplit = B.moe_ep_ffn_splits(self.rows_hint, d, self.El, d_ff)
        # Complete rows (no K split) come back as bf16: half the bytes.
        self.y_bf16 = B.moe_ep_output_bf16(self.rows_hint, d, self.El, d_ff) == 1

    def alloc(self, device) -> _Rank:
        kw = dict(device=device)
        shared = self.d_ff_shared > 0
        shared_ws = None
        if shared:
            need = B.moe_workspace_size(self.T_max, self.d, 1, self.d_ff_shared, 1)
            shared_ws = torch.empty(need, dtype=torch.uint8, **kw)
        return _Rank(
            recv_x=torch.empty(self.recv_rows, self.d, dtype=torch.bfloat16, **kw),
            recv_y=torch.empty(self.ksplit, self.recv_rows, self.d,
                               dtype=torch.bfloat16 if self.y_bf16 else torch.float32, **kw),
            ws=torch.empty(self.ws_bytes, dtype=torch.uint8, **kw),
            route_ws=torch.empty(B.moe_workspace_size(self.T_max, self.d, self.E, 128, self.k),
                                 dtype=torch.uint8, **kw),
            idx=torch.empty(self.T_max, self.k, dtype=torch.int32, **kw),
            w=torch.empty(self.T_max, self.k, dtype=torch.float32, **kw),
            counts=torch.empty(self.E, dtype=torch.int32, **kw),
            pos=torch.empty(self.T_max, self.k, dtype=torch.int32, **kw),
            recv_offsets=torch.empty(self.El + 1, dtype=torch.int32, **kw),
            shared_off=torch.empty(2, dtype=torch.int32, **kw) if shared else None,
            shared_y=torch.empty(self.T_max, self.d, dtype=torch.float32, **kw) if shared else None,
            shared_ws=shared_ws,
        )


def _route(p: _Plan, b: _Rank, x, Wg, router_bias, counts_out):
    T = x.shape[0]
    if T > p.T_max:
        raise ValueError(f"{T} tokens > T_max={p.T_max}")
    if T == 0:
        counts_out.zero_()  # a rank with no tokens this step still takes part
        return
    B.moe_route(T, p.d, p.E, p.k, x, Wg, router_bias, b.idx, b.w, counts_out, b.route_ws)


def _shared(p: _Plan, b: _Rank, x, shared):
    """The always-on expert on this rank's own tokens (weights replicated)."""
    if shared is None or x.shape[0] == 0:
        return None
    T = x.shape[0]
    # [0, T] as the one segment's bounds, set by a device fill (no host copy,
    # so the call can be captured in a CUDA graph).
    b.shared_off[0].fill_(0)
    b.shared_off[1].fill_(T)
    Ws1, Ws3, Ws2 = shared
    B.moe_expert_ffn(T, p.d, 1, p.d_ff_shared, x, b.shared_off, Ws1, Ws3, Ws2, b.shared_y,
                     b.shared_ws)
    return b.shared_y


def _dispatch(p: _Plan, b: _Rank, rank, x, counts_all, recv_x_all):
    T = x.shape[0]
    B.moe_ep_dispatch(T, p.d, p.E, p.k, p.R, rank, x, b.idx, counts_all, recv_x_all,
                      p.recv_rows, b.pos, b.recv_offsets, b.ws)


def _ffn(p: _Plan, b: _Rank, W1, W3, W2):
    B.moe_ep_expert_ffn(p.T_max, p.d, p.E, p.d_ff, p.k, p.R, p.rows_hint, p.ksplit, p.y_bf16,
                        b.recv_x, b.recv_offsets, W1, W3, W2, b.recv_y, b.ws)


def _combine(p: _Plan, b: _Rank, T, recv_y_all, shared_y, out):
    B.moe_ep_combine(T, p.d, p.E, p.k, p.R, p.recv_rows, p.ksplit, p.y_bf16, b.idx, b.pos, b.w,
                     recv_y_all, shared_y, out)


class EmulatedExpertParallel:
    """R ranks of an expert-parallel layer on one GPU: the same kernels and
    buffers as ``ExpertParallelLayer``, the ranks run one after another on the
    current stream (which orders them as the collectives would)."""

    def __init__(self, R, T_max, d, E, d_ff, k, d_ff_shared=0, device="cuda"):
        self.plan = _Plan(R, T_max, d, E, d_ff, k, d_ff_shared)
        self.ranks = [self.plan.alloc(device) for _ in range(R)]
        self.counts_all = torch.empty(R, E, dtype=torch.int32, device=device)

    def forward(self, xs, Wg, W1, W3, W2, outs, router_bias=None, shared=None):
        """``xs``/``outs``: per-rank token batches [T_r, d] bf16 / [T_r, d]
        fp32.  W1, W3, W2 hold all E experts; rank r uses its block."""
        p = self.plan
        if len(xs) != p.R or len(outs) != p.R:
            raise ValueError(f"need {p.R} batches")
        for r in range(p.R):
            b = self.ranks[r]
            _route(p, b, xs[r], Wg, router_bias, b.counts)
            self.counts_all[r].copy_(b.counts)  # the all-gather of the counts
        recv_x_all = [b.recv_x for b in self.ranks]
        recv_y_all = [b.recv_y for b in self.ranks]
        for r in range(p.R):
            _dispatch(p, self.ranks[r], r, xs[r], self.counts_all, recv_x_all)
        for r in range(p.R):
            lo, hi = expert_block(p.E, p.R, r)
            _ffn(p, self.ranks[r], W1[lo:hi], W3[lo:hi], W2[lo:hi])
        for r in range(p.R):
            sy = _shared(p, self.ranks[r], xs[r], shared)
            _combine(p, self.ranks[r], xs[r].shape[0], recv_y_all, sy, outs[r])

    def device_errors(self):
        """Error word of every rank's workspace (waits for the stream)."""
        return [B.moe_get_device_error(b.ws)[1] for b in self.ranks]


def peer_addresses(rank, entries, local, open_handle, opened=None):
    """Addresses of every rank's buffers as this process sees them.

    ``entries[r]`` is rank r's ``(handle, offset)`` of one buffer (gathered
    from all ranks in rank order); ``local`` this rank's own address.  A
    peer's handle is opened with ``open_handle`` (which returns the base
    address of the allocation holding the buffer) and the sender's offset is
    added; this rank's own entry is never opened.  ``opened`` maps handles
    already opened in this process to their bases: an allocation is mapped
    once however many buffers it holds (CUDA maps a handle once per
    process).  Returns (addresses in rank order, the handle -> base map)."""
    opened = {} if opened is None else opened
    addrs = []
    for r, (handle, offset) in enumerate(entries):
        if r == rank:
            addrs.append(int(local))
        else:
            if handle not in opened:
                opened[handle] = int(open_handle(handle))
            addrs.append(opened[handle] + int(offset))
    return addrs, opened


class ExpertParallelLayer:
    """One rank of an expert-parallel layer (torch.distributed, one process
    per GPU on one node).  Holds this rank's expert block W1/W3/W2[E/R, ...]
    and the replicated router (and shared expert).

    The receive and output buffers are mapped into the peers with CUDA IPC,
    which needs memory from cudaMalloc: torch's caching allocator in its
    default mode (with expandable segments the handle export fails and the
    constructor raises MoEError).

    With an NCCL group the collectives are stream-ordered: nothing waits on
    the host and a step can be captured in a CUDA graph.  With any other
    backend (gloo) the same steps are ordered on the host instead: the
    counts go through host memory and each barrier first waits for this
    process's stream.  That form is slower; it serves hosts without NCCL
    and processes that share one GPU."""

    def __init__(self, T_max, d, E, d_ff, k, Wg, W1_local, W3_local, W2_local, group=None,
                 router_bias=None, shared=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        d_ffs = 0 if shared is None else shared[0].shape[0]
        self.plan = _Plan(R, T_max, d, E, d_ff, k, d_ffs)
        if W1_local.shape[0] != self.plan.El:
            raise ValueError(f"rank holds {W1_local.shape[0]} experts, expected {self.plan.El}")
        device = W1_local.device
        self.buf = self.plan.alloc(device)
        self.Wg, self.W1, self.W3, self.W2 = Wg, W1_local, W3_local, W2_local
        self.router_bias, self.shared = router_bias, shared
        self.counts_all = torch.empty(R, E, dtype=torch.int32, device=device)
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)
        self.host_ordered = dist.get_backend(group) != "nccl"
        self._opened = []
        if R == 1:
            self.recv_x_all, self.recv_y_all = [self.buf.recv_x], [self.buf.recv_y]
            return
        mine = (B.moe_ipc_get_handle(self.buf.recv_x), B.moe_ipc_get_handle(self.buf.recv_y))
        gathered = [None] * R
        dist.all_gather_object(gathered, mine, group=group)
        opened = {}
        self.recv_x_all, _ = peer_addresses(self.rank, [g[0] for g in gathered],
                                            self.buf.recv_x.data_ptr(), B.moe_ipc_open_handle,
                                            opened)
        self.recv_y_all, _ = peer_addresses(self.rank, [g[1] for g in gathered],
                                            self.buf.recv_y.data_ptr(), B.moe_ipc_open_handle,
                                            opened)
        self._opened = list(opened.values())

    def _gather_counts(self):
        b = self.buf
        if self.host_ordered:
            host = torch.empty(self.counts_all.numel(), dtype=torch.int32)
            self.dist.all_gather_into_tensor(host, b.counts.cpu(), group=self.group)
            self.counts_all.copy_(host.view_as(self.counts_all))
        else:
            self.dist.all_gather_into_tensor(self.counts_all.view(-1), b.counts, group=self.group)

    def _barrier(self):
        if self.host_ordered:
            # This process's kernels (and their stores into peers) are done
            # before the host barrier lets any rank go on.
            torch.cuda.current_stream().synchronize()
            self.dist.barrier(group=self.group)
        else:
            # One-word all-reduce on the current stream: returns on no rank
            # before every rank's stream reached it.
            self.dist.all_reduce(self.flag, group=self.group)

    def forward(self, x, out):
        p, b = self.plan, self.buf
        _route(p, b, x, self.Wg, self.router_bias, b.counts)
        self._gather_counts()
        _dispatch(p, b, self.rank, x, self.counts_all, self.recv_x_all)
        self._barrier()
        _ffn(p, b, self.W1, self.W3, self.W2)
        self._barrier()
        sy = _shared(p, b, x, self.shared)
        _combine(p, b, x.shape[0], self.recv_y_all, sy, out)

    def device_error(self):
        return B.moe_get_device_error(self.buf.ws)[1]

    def close(self):
        """Unmaps the peers' buffers, after every rank finished reading them."""
        if not self._opened:
            return
        torch.cuda.current_stream().synchronize()
        self.dist.barrier(group=self.group)
        for base in self._opened:
            B.moe_ipc_close(base)
        self._opened = []
