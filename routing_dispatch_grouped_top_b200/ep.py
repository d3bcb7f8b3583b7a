"""Expert-parallel routed MoE layer: one process per GPU, the experts split over the ranks.

Each rank routes its own T tokens, and the rows of every assignment travel to the rank that
owns the expert and back (WideEP essay, "The router writes a network schedule").  The steps
run in this library's kernels (include/moe.h, "Expert-parallel exchange across GPUs"); this
module only holds the buffers and issues the calls in protocol order:

    gating -> route -> count/scan (P = R partitions = ranks)
    all-gather of the per-expert counts (a collective supplied by the caller)
    plan -> dispatch (peer stores) -> wait -> grouped gate/up + down on the received rows
    -> return (peer stores) -> wait -> combine

:class:`EPRank` is one rank's state.  :func:`connect` fills the peer table of a real
multi-process group by exchanging CUDA IPC handles through ``torch.distributed``;
:func:`emulated_peers` builds it for several ranks whose buffers live in one process (the
single-GPU test of the kernels; the ranks' launches are then issued in protocol order so that
nothing ever waits for a kernel that has not run).
"""
from __future__ import annotations

from typing import Callable, List, Sequence

import torch

from . import binding as B


class EPRank:
    """Buffers and launches of one rank.  ``w_gate``, ``w_up`` [E/R][F][H] and ``w_down``
    [E/R][H][F] are this rank's experts; ``w_g`` [H][E] is the (replicated) router."""

    def __init__(self, T: int, H: int, E: int, K: int, F: int, R: int, rank: int, w_g, w_gate, w_up, w_down,
                 device="cuda", renormalize=True, bias=None):
        if E % R:
            raise ValueError("E must be a multiple of the number of ranks")
        self.R, self.rank, self.El = R, rank, E // R
        self.d = B.dims(T=T, H=H, E=E, K=K, F=F, P=R, renormalize=renormalize)
        self.cap = R * T * K          # every assignment of every rank may land here: no drops
        self.d_recv = B.dims(T=self.cap, H=H, E=self.El, K=1, F=F)
        dev = torch.device(device)
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        i32, bf = torch.int32, torch.bfloat16
        self.w_g_split = e((3, E, H), bf)
        B.moe_pack_router(w_g.contiguous(), self.d, self.w_g_split)
        self.bias = bias
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.ws = B.make_workspace(self.d, dev)
        self.gemm_ws = B.make_workspace(self.d_recv, dev)
        self.ep_ws = B.ep_workspace(dev)
        TK = T * K
        self.logits = e((T, E), torch.float32)
        self.topk_ids, self.topk_w = e((T, K), i32), e((T, K), torch.float32)
        self.counts, self.offsets = e((E,), i32), e((E + 1,), i32)
        self.part_counts, self.part_offsets = e((R,), i32), e((R + 1,), i32)
        self.row_of_assign, self.assign_of_row = e((TK,), i32), e((TK,), i32)
        self.counts_all = e((R, E), i32)
        self.send_base, self.recv_offsets = e((E,), i32), e((self.El + 1,), i32)
        # exchange buffers: written by the peers
        self.recv_x = torch.zeros((self.cap, H), dtype=bf, device=dev)
        self.recv_meta = torch.full((self.cap, 2), -1, dtype=i32, device=dev)
        self.ret_y = torch.zeros((TK, H), dtype=bf, device=dev)
        self.signal = torch.zeros(2 * R, dtype=i32, device=dev)
        self.h_recv, self.y_recv = e((self.cap, F), bf), e((self.cap, H), bf)
        self.out = e((T, H), bf)
        self.epoch = 0
        self.peers = None

    def exchange_buffers(self) -> List[torch.Tensor]:
        """The four buffers the peers write, in the order of moe_ep_peers' fields."""
        return [self.recv_x, self.recv_meta, self.ret_y, self.signal]

    # ---- protocol steps ----------------------------------------------------
    def route(self, x, stream=None):
        """Gating, top-K and count/scan of this rank's tokens (partitions = ranks)."""
        B.moe_gating(x, self.w_g_split, self.bias, self.d, self.logits, self.ws, stream)
        B.moe_route(self.logits, self.d, self.topk_ids, self.topk_w, stream)
        B.moe_count_scan(self.topk_ids, self.d, self.counts, self.offsets, self.part_counts, self.part_offsets,
                         self.row_of_assign, self.assign_of_row, self.ws, stream)

    def dispatch(self, x, stream=None):
        """Plan from the gathered counts (self.counts_all, filled by the caller) and send."""
        self.epoch += 1
        B.moe_ep_plan(self.counts_all, self.R, self.rank, self.d, self.send_base, self.recv_offsets, stream)
        B.moe_ep_dispatch(x, self.row_of_assign, self.topk_ids, self.offsets, self.send_base, self.d, self.R,
                          self.rank, self.cap, self.peers, self.epoch, self.ep_ws, stream)

    def experts(self, stream=None):
        """Once every source has sent: the local experts' SwiGLU FFN on the received rows."""
        B.moe_ep_wait(self.signal, self.R, 0, self.epoch, self.ep_ws, stream)
        B.moe_grouped_ffn(self.recv_x, self.recv_offsets, self.w_gate, self.w_up, self.w_down, self.d_recv,
                          self.h_recv, self.y_recv, self.gemm_ws, stream)

    def give_back(self, stream=None):
        B.moe_ep_return(self.y_recv, self.recv_meta, self.recv_offsets, self.d, self.R, self.rank, self.cap,
                        self.peers, self.epoch, self.ep_ws, stream)

    def combine(self, stream=None):
        """Once every owner has returned: the weighted sum at each token."""
        B.moe_ep_wait(self.signal, self.R, 1, self.epoch, self.ep_ws, stream)
        B.moe_combine(self.ret_y, self.row_of_assign, self.topk_w, self.d, self.out, stream=stream)
        return self.out

    def forward(self, x, all_gather_counts: Callable[[torch.Tensor, torch.Tensor], None], stream=None):
        """One layer call on this rank (a multi-process group, peers from :func:`connect`)."""
        self.route(x, stream)
        all_gather_counts(self.counts_all, self.counts)
        self.dispatch(x, stream)
        self.experts(stream)
        self.give_back(stream)
        return self.combine(stream)


def emulated_peers(ranks: Sequence[EPRank]) -> B.moe_ep_peers:
    """Peer table of ranks that all live in this process (their own device addresses)."""
    return B.ep_peers(*[[r.exchange_buffers()[i].data_ptr() for r in ranks] for i in range(4)])


def connect(rank: EPRank, group=None) -> list:
    """Fills rank.peers for a multi-process group: every rank exports CUDA IPC handles of its
    exchange buffers, all-gathers them (host objects over torch.distributed) and opens the
    others'.  Returns the opened bases, to be closed with :func:`disconnect`."""
    import torch.distributed as dist
    mine = [B.ep_ipc_export(t) for t in rank.exchange_buffers()]
    allh = [None] * rank.R
    dist.all_gather_object(allh, mine, group=group)
    addrs = [[0] * rank.R for _ in range(4)]
    bases = []
    for r in range(rank.R):
        for i, t in enumerate(rank.exchange_buffers()):
            if r == rank.rank:
                addrs[i][r] = t.data_ptr()
            else:
                base, ptr = B.ep_ipc_import(*allh[r][i])
                bases.append(base)
                addrs[i][r] = ptr
    rank.peers = B.ep_peers(*addrs)
    return bases


def disconnect(bases: Sequence[int]):
    for b in bases:
        B.ep_ipc_close(b)


def nccl_all_gather_counts(group=None):
    """The counts collective of a torch.distributed (NCCL) group, on the current stream."""
    import torch.distributed as dist

    def gather(out: torch.Tensor, mine: torch.Tensor):
        dist.all_gather_into_tensor(out.view(-1), mine, group=group)
    return gather
