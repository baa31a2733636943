"""Expert parallelism for the routed MoE layer over W ranks (W divides 8).

Rank d holds the 8/W expert groups d*8/W .. (d+1)*8/W - 1, i.e. the 128/W
experts d*n .. (d+1)*n - 1 (n = 128/W), packed as a slice with
moe_pack_experts and renumbered 0 .. n-1.  The pages put the 128 experts in 8
groups of 16 and keep 4 groups per token ("Ling-3.0-tiny on a Qualcomm board",
TensorFold issue #1247, first comment, opening paragraph): a token's 8
experts lie in at most 4 groups, so with whole groups per rank its row goes to
at most 4 ranks.  That fan-out cap is what makes the split cheap.

One layer on every rank, each with its own T tokens already routed
(moe_route on the rank's own logits):

  1. plan (source side): for each token the set of ranks owning one of its
     experts; rows are sent destination-major, token-ascending, each carrying
     its 8 slots as local expert ids at that destination (-1 for a slot whose
     expert lives elsewhere).  The y rows come back in item order (token,
     slot) per destination, so the source knows where every (token, slot)
     lands without being told.
  2. a fixed-size all-to-all of two counts per peer (rows to send, y rows to
     get back): the one host read of the layer sizes the exchanges.
  3. dispatch: all-to-all-v of the x rows and of their local slot ids.
  4. owner side: moe_permute of the local ids (empty slots skipped) and the
     grouped expert FFN on the rank's slice (moe_expert_ffn_slice); the y rows
     of the non-empty slots go back in (source, row, slot) order.
  5. combine all-to-all-v of the y rows back to their sources.
  6. source side: moe_combine over the 8 returned rows of every token, in
     slot order, plus the residual -- the single-GPU combine unchanged, so
     the layer output is the single-GPU one whenever the y rows are.

Transfers go through torch.distributed (NCCL over NVLink on GPUs, gloo for
the CPU tests) with every row viewed as 32-bit words, so the bytes cross
unchanged.  No tensor-memory-accelerator load ever reads another GPU's
memory here: every exchange lands in this rank's own buffers before a kernel
reads it.

The owner-side compute and the source-side combine are the library's CUDA
calls.  The CPU tests replace them explicitly (``compute=`` / ``combine=``)
with the float64 oracle to check the exchange's index arithmetic on gloo ranks;
there is no implicit fallback.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch

N_EXPERTS, TOPK, N_GROUPS, HIDDEN = 128, 8, 8, 1536


def experts_per_rank(world: int) -> int:
    if world < 1 or N_GROUPS % world:
        raise ValueError(f"world size {world} must divide the {N_GROUPS} expert groups")
    return N_EXPERTS // world


@dataclass
class DispatchPlan:
    """Source-side plan of one layer.

    send_counts [W]: rows sent to each rank; send_tok [S]: the token of each
    sent row (destination-major, token-ascending); send_local [S, 8] int32: the
    row's slots as local expert ids at its destination, -1 where the slot's
    expert lives elsewhere; ret_counts [W]: y rows each rank sends back (the
    slots it owns); ret_index [T*8] int32: the row of item t*8+slot in the
    concatenated returned y rows."""
    send_counts: torch.Tensor
    send_tok: torch.Tensor
    send_local: torch.Tensor
    ret_counts: torch.Tensor
    ret_index: torch.Tensor


def plan_dispatch(topk_idx: torch.Tensor, world: int) -> DispatchPlan:
    """The dispatch plan of a rank's routed tokens (topk_idx [T, 8], ids < 128)."""
    n_loc = experts_per_rank(world)
    idx = topk_idx.to(torch.int64)
    T = idx.shape[0]
    dev = idx.device
    owner = torch.div(idx, n_loc, rounding_mode="floor")                   # [T, 8]
    ranks = torch.arange(world, device=dev)
    mask = (owner.unsqueeze(2) == ranks.view(1, 1, world)).any(dim=1)      # [T, W]
    send_counts = mask.sum(dim=0)
    dst, tok = torch.nonzero(mask.t(), as_tuple=True)                      # row-major: dst-major
    own = owner.index_select(0, tok) == dst.unsqueeze(1)
    local = torch.where(own, idx.index_select(0, tok) - dst.unsqueeze(1) * n_loc,
                        torch.full_like(idx.index_select(0, tok), -1))
    flat_owner = owner.reshape(-1)
    order = torch.argsort(flat_owner, stable=True)                        # dst-major, item order
    ret_index = torch.empty_like(order)
    ret_index[order] = torch.arange(T * TOPK, device=dev)
    ret_counts = torch.bincount(flat_owner, minlength=world)
    return DispatchPlan(send_counts, tok, local.to(torch.int32).contiguous(), ret_counts,
                        ret_index.to(torch.int32))


class DistExchange:
    """All-to-all exchanges over a torch.distributed process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def fixed(self, t: torch.Tensor) -> torch.Tensor:
        """[W, k] -> [W, k]: row j goes to rank j; row i of the result came from rank i."""
        out = torch.empty_like(t)
        self.dist.all_to_all_single(out, t.contiguous(), group=self.group)
        return out

    def rows(self, t: torch.Tensor, send_counts: list[int], recv_counts: list[int]) -> torch.Tensor:
        """Variable all-to-all of the leading dimension, bytes unchanged (each
        row travels as 32-bit words, a type every backend moves)."""
        tail = tuple(t.shape[1:])
        row_bytes = t.element_size()
        for d in tail:
            row_bytes *= d
        if row_bytes % 4:
            raise ValueError("rows must be a whole number of 32-bit words")
        src = t.contiguous().view(torch.uint8).view(t.shape[0], row_bytes).view(torch.int32)
        out = src.new_empty((sum(recv_counts), row_bytes // 4))
        self.dist.all_to_all_single(out, src, output_split_sizes=recv_counts,
                                    input_split_sizes=send_counts, group=self.group)
        return out.view(torch.uint8).view(t.dtype).view((-1,) + tail)


def _library_compute(packed_slice: torch.Tensor, n_loc: int):
    """Owner-side compute with the CUDA library: permute the local ids (empty
    slots skipped), the grouped FFN on the slice, and the y rows of the
    non-empty slots in (row, slot) order."""
    from . import moe

    def compute(recv_x: torch.Tensor, recv_local: torch.Tensor) -> torch.Tensor:
        R = recv_x.shape[0]
        if R == 0:
            return torch.empty((0, HIDDEN), dtype=torch.float16, device=recv_x.device)
        _, offsets, perm_src, inv_perm = moe.moe_permute(recv_local.contiguous())
        h = torch.empty((R * TOPK, 512), dtype=torch.float16, device=recv_x.device)
        y = torch.empty((R * TOPK, HIDDEN), dtype=torch.float16, device=recv_x.device)
        moe.moe_expert_ffn_slice(recv_x.contiguous(), packed_slice, n_loc, offsets, perm_src, h, y)
        rows = inv_perm.to(torch.int64)[recv_local.reshape(-1) >= 0]
        return y.index_select(0, rows)
    return compute


def _library_combine(y_back, topk_w, ret_index, residual, out):
    from . import moe
    return moe.moe_combine(y_back, topk_w, ret_index, residual=residual, out=out)


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer (see the module text).

    packed_slice: this rank's experts rank*n .. rank*n+n-1 packed by
    moe_pack_experts (n = 128 / world).  compute / combine: replacements of the
    library calls, for the CPU tests only."""

    def __init__(self, rank: int, world: int, packed_slice: torch.Tensor | None = None,
                 compute: Callable | None = None, combine: Callable | None = None):
        self.rank, self.world = rank, world
        self.n_loc = experts_per_rank(world)
        if compute is None:
            if packed_slice is None:
                raise ValueError("packed_slice is required for the library compute")
            compute = _library_compute(packed_slice, self.n_loc)
        self.compute = compute
        self.combine = combine if combine is not None else _library_combine
        self.plan = None

    # -- the phases, each run by every rank between two exchanges ------------------
    def begin(self, topk_idx: torch.Tensor) -> torch.Tensor:
        """Plan the layer; returns [W, 2] counts for the fixed exchange: (rows
        sent to rank j, y rows expected back from rank j)."""
        self.plan = plan_dispatch(topk_idx, self.world)
        return torch.stack([self.plan.send_counts, self.plan.ret_counts], dim=1)

    def sizes(self, sent: torch.Tensor, got: torch.Tensor):
        """The host read of the layer: per-rank row counts of the three
        variable exchanges, from the sent and received fixed counts."""
        s = torch.cat([sent, got]).cpu()
        W = self.world
        self.send_counts = s[:W, 0].tolist()
        self.back_counts = s[:W, 1].tolist()   # y rows this rank gets back, per owner
        self.recv_counts = s[W:, 0].tolist()   # rows this rank receives, per source
        self.ret_counts = s[W:, 1].tolist()    # y rows this rank returns, per source

    def dispatch_rows(self, x: torch.Tensor):
        """The x rows and their local slot ids to send (destination-major)."""
        return x.index_select(0, self.plan.send_tok), self.plan.send_local

    def owner_compute(self, recv_x: torch.Tensor, recv_local: torch.Tensor) -> torch.Tensor:
        y = self.compute(recv_x, recv_local)
        if y.shape[0] != sum(self.ret_counts):
            raise RuntimeError(f"rank {self.rank}: {y.shape[0]} y rows for "
                               f"{sum(self.ret_counts)} announced slots")
        return y

    def finish(self, y_back: torch.Tensor, topk_w: torch.Tensor, residual=None, out=None):
        return self.combine(y_back, topk_w, self.plan.ret_index, residual, out)

    # -- one layer over a process group --------------------------------------------
    def forward(self, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                ex: DistExchange, residual=None, out=None):
        sent = self.begin(topk_idx)
        got = ex.fixed(sent)
        self.sizes(sent, got)
        sx, sl = self.dispatch_rows(x)
        recv_x = ex.rows(sx, self.send_counts, self.recv_counts)
        recv_local = ex.rows(sl, self.send_counts, self.recv_counts)
        y = self.owner_compute(recv_x, recv_local)
        y_back = ex.rows(y, self.ret_counts, self.back_counts)
        return self.finish(y_back, topk_w, residual, out)


def _exchange_in_process(send: list[torch.Tensor], counts: list[list[int]]) -> list[torch.Tensor]:
    """All-to-all-v among ranks held by one process: send[s] holds rank s's rows
    for every destination in order, counts[s][d] of them for d."""
    W = len(send)
    parts = [torch.split(send[s], counts[s]) for s in range(W)]
    return [torch.cat([parts[s][d] for s in range(W)]) for d in range(W)]


def forward_in_process(layers: list[ExpertParallelMoE], xs, topk_idxs, topk_ws,
                       residuals=None, outs=None):
    """The W ranks of one layer run in lockstep by a single process (on one GPU):
    the same phases as ExpertParallelMoE.forward, with the exchanges done by
    copies.  Used to check the whole data path on one device."""
    W = len(layers)
    residuals = residuals or [None] * W
    outs = outs or [None] * W
    sent = [L.begin(i) for L, i in zip(layers, topk_idxs)]
    for d, L in enumerate(layers):
        L.sizes(sent[d], torch.stack([sent[s][d] for s in range(W)]))
    disp = [L.dispatch_rows(x) for L, x in zip(layers, xs)]
    sc = [L.send_counts for L in layers]
    recv_x = _exchange_in_process([d[0] for d in disp], sc)
    recv_l = _exchange_in_process([d[1] for d in disp], sc)
    ys = [L.owner_compute(rx, rl) for L, rx, rl in zip(layers, recv_x, recv_l)]
    y_back = _exchange_in_process(ys, [L.ret_counts for L in layers])
    return [L.finish(yb, w, r, o) for L, yb, w, r, o in zip(layers, y_back, topk_ws, residuals, outs)]
