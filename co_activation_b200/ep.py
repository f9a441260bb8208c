"""Expert parallelism across GPUs: one process per GPU, each GPU one EP rank.

Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English abstracts:
under expert parallelism every MoE layer exchanges tokens all-to-all so that each token
reaches the GPUs holding its experts (with the deduplicated dispatcher: each GPU once),
and exchanges the expert outputs back to be combined; the co-activation statistics are
global.

Per layer, on every rank s of the group (R = group size = number of EP ranks):
  1. plan_dispatch over this rank's tokens, all of them homed on s
  2. exchange the count rows: C[s][r] rows and A[s][r] assignments s sends to r
     (one all_gather of 2R int32 per rank)
  3. dispatch
       transport "peer": dispatch_gather_peer writes every row straight into the
                         destination rank's receive buffer (symmetric memory over
                         NVLink) at row sum_{s'<s} C[s'][r] + ...; then a group barrier
       transport "nccl": dispatch_gather into the local send buffer, all_to_all_single
     Either way rank r receives the rank-r segment of the single-GPU plan of all ranks'
     tokens (ranks' tokens contiguous): rows by source rank, then token.
  4. the experts (caller) turn the received rows into outputs in expanded receive order
  5. combine
       "peer": group barrier, combine_scatter_peer reads each output from its rank
       "nccl": all_to_all_single back, combine_scatter
  counts: coact_count locally, then one all_reduce(sum) of pair and loads.

Only library kernels touch rows and plans; this module moves split sizes, builds the
small per-row expert-id metadata the experts need, and calls the collectives.  The
local steps are an `ops` object (the library by default) so that the exchange logic can
run on CPU test doubles.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional

import torch
import torch.distributed as dist


def exclusive_offsets(C: torch.Tensor) -> torch.Tensor:
    """off[s][r] = sum_{s' < s} C[s'][r]: where source s's rows start in rank r's buffer."""
    off = torch.zeros_like(C)
    if C.shape[0] > 1:
        off[1:] = torch.cumsum(C, dim=0)[:-1]
    return off


@dataclasses.dataclass
class Dispatched:
    """What rank r receives: its rows (source rank, then token order), the slot mask of
    each row and the expert id of every set slot (-1 elsewhere)."""
    rows: torch.Tensor          # bf16 [n_rows, H]
    kmask: torch.Tensor         # uint8 [n_rows]
    experts: torch.Tensor       # int32 [n_rows, k]
    counts: torch.Tensor        # int64 [R, R] rows s -> r
    asg: torch.Tensor           # int64 [R, R] assignments s -> r


class LibraryOps:
    """The local steps through the library's kernels (device tensors)."""

    def __init__(self, coact):
        self.c = coact

    def plan(self, ids, E, expert_rank, R, rank_node, n_nodes, src_rank):
        N, k = ids.shape
        p = self.c.alloc_plan(N, k, E, R, ids.device, with_rank_mask=False, with_src_dst=False)
        self.c.plan_dispatch(ids, E, expert_rank, R, p, rank_node=rank_node, n_nodes=n_nodes,
                             src_rank=src_rank)
        return p

    def gather(self, x, plan):
        send = torch.empty((plan.row_capacity, x.shape[1]), dtype=x.dtype, device=x.device)
        self.c.dispatch_gather(x, plan.send_row, send)
        return send

    def combine(self, y, gates, plan, out):
        return self.c.combine_scatter(y, gates, plan.comb_row, out)

    def count(self, ids, E, pair, loads):
        self.c.coact_count(ids, E, pair, loads)


class EPLayer:
    """Dispatch and combine of one MoE layer across the ranks of `group`."""

    def __init__(self, group, E: int, expert_rank: torch.Tensor,
                 rank_node: Optional[torch.Tensor] = None, n_nodes: int = 1,
                 transport: str = "nccl", ops=None, peer_capacity: Optional[int] = None):
        self.group = group
        self.R = dist.get_world_size(group)
        self.me = dist.get_rank(group)
        self.E = E
        self.expert_rank = expert_rank
        self.rank_node = rank_node
        self.n_nodes = n_nodes
        if transport not in ("nccl", "peer"):
            raise ValueError("transport must be 'nccl' or 'peer'")
        self.transport = transport
        if ops is None:
            import co_activation_b200 as coact
            ops = LibraryOps(coact)
        self.ops = ops
        self.peer_capacity = peer_capacity
        self._peer = None
        self.plan = None

    # ------------------------------------------------------------------ statistics

    def count(self, ids: torch.Tensor, pair: torch.Tensor, loads: torch.Tensor) -> None:
        """Co-activation counts of this rank's tokens, summed over the group."""
        local_p = torch.zeros_like(pair)
        local_l = torch.zeros_like(loads)
        self.ops.count(ids, self.E, local_p, local_l)
        dist.all_reduce(local_p, group=self.group)
        dist.all_reduce(local_l, group=self.group)
        pair += local_p
        loads += local_l

    # ------------------------------------------------------------------ exchange

    def _count_rows(self, plan):
        rows = plan.rank_counts.to(torch.int64)
        asg = (plan.asg_offsets[1:] - plan.asg_offsets[:-1]).to(torch.int64)
        mine = torch.cat([rows, asg]).contiguous()
        allrows = [torch.empty_like(mine) for _ in range(self.R)]
        dist.all_gather(allrows, mine, group=self.group)
        M = torch.stack(allrows)                  # [R sources, 2R]
        return M[:, :self.R].contiguous(), M[:, self.R:].contiguous()

    def _row_experts(self, ids, plan, D):
        """Expert id of every set slot of each send row (-1 elsewhere), int32 [D, k]."""
        k = ids.shape[1]
        tok = plan.row_token[:D].to(torch.int64)
        km = plan.row_kmask[:D].to(torch.int32)
        bits = (km[:, None] >> torch.arange(k, device=km.device, dtype=torch.int32)) & 1
        return torch.where(bits.bool(), ids[tok], torch.full_like(ids[tok], -1))

    def dispatch(self, ids: torch.Tensor, x: torch.Tensor) -> Dispatched:
        """Plan this rank's tokens and deliver every row to its destination rank."""
        R, me = self.R, self.me
        src = torch.full((ids.shape[0],), me, dtype=torch.int32, device=ids.device)
        plan = self.ops.plan(ids, self.E, self.expert_rank, R, self.rank_node, self.n_nodes, src)
        self.plan = plan
        C, A = self._count_rows(plan)
        Cl, Al = C.cpu(), A.cpu()
        self._C, self._A = Cl, Al
        D = int(Cl[me].sum())
        n_recv = int(Cl[:, me].sum())
        meta_send = self._row_experts(ids, plan, D)
        kmask_send = plan.row_kmask[:D].to(torch.int32)
        send_splits = Cl[me].tolist()
        recv_splits = Cl[:, me].tolist()
        H = x.shape[1]
        if self.transport == "nccl":
            send = self.ops.gather(x, plan)
            rows = torch.empty((n_recv, H), dtype=x.dtype, device=x.device)
            # rows travel as raw 32-bit words (two bf16 each): exact, any backend
            dist.all_to_all_single(rows.view(torch.int32), send[:D].contiguous().view(torch.int32),
                                   recv_splits, send_splits, group=self.group)
        else:
            rows = self._peer_dispatch(x, plan, Cl, Al, n_recv)
        experts = torch.empty((n_recv, ids.shape[1]), dtype=torch.int32, device=ids.device)
        dist.all_to_all_single(experts, meta_send.to(torch.int32).contiguous(), recv_splits,
                               send_splits, group=self.group)
        kmask = torch.empty((n_recv,), dtype=torch.int32, device=ids.device)
        dist.all_to_all_single(kmask, kmask_send.contiguous(), recv_splits, send_splits,
                               group=self.group)
        return Dispatched(rows=rows, kmask=kmask.to(torch.uint8), experts=experts, counts=Cl,
                          asg=Al)

    def combine(self, y_recv: torch.Tensor, gates: torch.Tensor,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Bring the expert outputs (expanded receive order on this rank) back to their
        source ranks and combine them in token order."""
        me, plan = self.me, self.plan
        Al = self._A
        H = y_recv.shape[1]
        N = gates.shape[0]
        if out is None:
            out = torch.empty((N, H), dtype=y_recv.dtype, device=y_recv.device)
        if self.transport == "nccl":
            back = torch.empty((int(Al[me].sum()), H), dtype=y_recv.dtype, device=y_recv.device)
            dist.all_to_all_single(back.view(torch.int32), y_recv.contiguous().view(torch.int32),
                                   Al[me].tolist(), Al[:, me].tolist(), group=self.group)
            return self.ops.combine(back, gates, plan, out)
        return self._peer_combine(y_recv, gates, out)

    # ------------------------------------------------------------------ peer transport

    def _peer_buffers(self, H, dtype, device, rows, outs):
        """Symmetric receive / output buffers on every rank and their device addresses
        (every rank asks for the same sizes: the group-wide maxima)."""
        import torch.distributed._symmetric_memory as symm
        if (self._peer is None or self._peer["rows"] < rows or self._peer["outs"] < outs
                or self._peer["H"] != H):
            cap = max(rows, self.peer_capacity or 0)
            ocap = max(outs, 8 * (self.peer_capacity or 0))
            recv = symm.empty((cap, H), dtype=dtype, device=device)
            yout = symm.empty((ocap, H), dtype=dtype, device=device)
            h_recv = symm.rendezvous(recv, self.group)
            h_y = symm.rendezvous(yout, self.group)
            self._peer = {"rows": cap, "outs": ocap, "H": H, "recv": recv, "y": yout,
                          "h_recv": h_recv,
                          "h_y": h_y,
                          "recv_ptrs": torch.tensor(list(h_recv.buffer_ptrs), dtype=torch.int64,
                                                    device=device),
                          "y_ptrs": torch.tensor(list(h_y.buffer_ptrs), dtype=torch.int64,
                                                 device=device)}
        return self._peer

    def _peer_dispatch(self, x, plan, Cl, Al, n_recv):
        import co_activation_b200 as coact
        cap, ocap = int(Cl.sum(dim=0).max()), int(Al.sum(dim=0).max())
        pb = self._peer_buffers(x.shape[1], x.dtype, x.device, cap, ocap)
        off = exclusive_offsets(Cl)[self.me].to(torch.int32).to(x.device)
        capv = torch.full((self.R,), pb["rows"], dtype=torch.int32, device=x.device)
        coact.dispatch_gather_peer(x, plan.send_row, plan.rank_offsets, pb["recv_ptrs"], off, capv)
        pb["h_recv"].barrier()
        return pb["recv"][:n_recv]

    def _peer_combine(self, y_recv, gates, out):
        import co_activation_b200 as coact
        pb = self._peer
        n = y_recv.shape[0]
        if n > pb["y"].shape[0]:
            raise ValueError("expert outputs exceed the symmetric output buffer")
        pb["y"][:n].copy_(y_recv)
        pb["h_y"].barrier()
        off = exclusive_offsets(self._A)[self.me].to(torch.int32).to(out.device)
        capv = torch.full((self.R,), pb["y"].shape[0], dtype=torch.int32, device=out.device)
        coact.combine_scatter_peer(pb["y_ptrs"], off, capv, self.plan.asg_offsets, gates,
                                   self.plan.comb_row, out, y_recv.shape[1])
        pb["h_y"].barrier()
        return out


def expand_identity(d: Dispatched) -> torch.Tensor:
    """Identity experts: one output row per set slot of every received row, in expanded
    receive order (for tests and demonstrations)."""
    reps = torch.bitwise_count(d.kmask.to(torch.int32)).to(torch.int64) \
        if hasattr(torch, "bitwise_count") else \
        torch.tensor([bin(int(v)).count("1") for v in d.kmask.cpu()], device=d.rows.device)
    return d.rows.repeat_interleave(reps, dim=0)
