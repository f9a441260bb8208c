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

Pre-reduced combine (combine(..., reduce="rows")): the rank that ran the experts first
sums, with the gates (exchanged with the rows), the outputs of each received row's slots
-- one bf16 partial row per received row -- and only those travel back: D rows instead of
N*k.  The token's rank adds them (dispatch_gather_backward, or combine_scatter_peer with
unit weights reading them in place).

Backward over the same plan (the transposed maps):
  backward_combine(grad_out): grad_out rows are dispatched like x; where the experts ran,
      combine_scatter_backward gives grad_y (expanded receive order, for the experts'
      backward) and one gate gradient per served slot, which travel back to the token's
      rank (N*k floats in all).
  backward_dispatch(grad_rows): the experts' input gradients (one row per received row)
      travel back and are summed per token (dispatch_gather_backward, or the peer combine
      with unit weights).

Token shuffling in the post-attention reduce-scatter (shuffle_reduce_scatter): every rank
holds a partial attention output for all N tokens of the group; rank r gets the tokens
predicted to live on it (ascending), each the sum of the P partials in rank order --
"peer": one shuffle_reduce_scatter reading every peer's partial buffer in place; "nccl":
the partials permuted locally (dispatch_gather over the shuffle plan), one all_to_all of
the rank segments, then the same kernel over the P received blocks.

Only library kernels touch rows, plans and their per-row metadata (plan_row_meta: each
send row's expert ids, gates and output positions at the destination; gather_row_slots:
per-slot values back to token order); this module moves split sizes and calls the
collectives.  One host synchronisation per dispatch remains: NCCL's all_to_all_single
takes its split sizes as host lists, and the received tensors' shapes depend on the
exchanged counts.  The local steps are an `ops` object (the library by default) so that
the exchange logic can run on CPU test doubles.
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
    each row, the expert id of every set slot (-1 elsewhere) and where each set slot's
    expert output goes in this rank's expanded receive order (-1 elsewhere)."""
    rows: torch.Tensor          # bf16 [n_rows, H]
    kmask: torch.Tensor         # uint8 [n_rows]
    experts: torch.Tensor       # int32 [n_rows, k]
    slots: torch.Tensor         # int32 [n_rows, k]
    counts: torch.Tensor        # int64 [R, R] rows s -> r
    asg: torch.Tensor           # int64 [R, R] assignments s -> r
    gates: Optional[torch.Tensor] = None   # fp32 [n_rows, k]: gate of each set slot, 0 elsewhere


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

    def combine_local(self, y, gates, comb, out):
        return self.c.combine_scatter(y, gates, comb, out)

    def gather_backward(self, rows, send_row, out):
        return self.c.dispatch_gather_backward(rows, send_row, out)

    def combine_backward(self, y, gates, comb, g_out, g_y, g_gates):
        return self.c.combine_scatter_backward(y, gates, comb, g_out, g_y, g_gates)

    def count(self, ids, E, pair, loads):
        self.c.coact_count(ids, E, pair, loads)

    def row_meta(self, plan, ids, gates, slot_base):
        """Per send row and slot: expert id, gate (gates given) and output position."""
        return self.c.plan_row_meta(plan, ids, gates, slot_base)

    def gather_row_slots(self, vals, plan, out):
        """Per-(send row, slot) values back to token order [N, k]."""
        return self.c.gather_row_slots(vals, plan.send_row, plan.row_kmask, out)

    def shuffle_plan(self, home, R):
        return self.c.shuffle_plan(home, R)

    def shuffle_reduce(self, blocks, row_token, N, out):
        bases = torch.tensor([b.data_ptr() for b in blocks], dtype=torch.int64, device=out.device)
        return self.c.shuffle_reduce_scatter(bases, N, row_token, out)


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
        self._sym = {}
        self.plan = None
        self._d = None

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

    def dispatch(self, ids: torch.Tensor, x: torch.Tensor,
                 gates: Optional[torch.Tensor] = None) -> Dispatched:
        """Plan this rank's tokens and deliver every row to its destination rank.  With
        gates, each row's slot gates travel too (needed by the pre-reduced combine and the
        backward).  On the peer transport the returned rows are a view of this rank's
        symmetric receive buffer: valid until the next dispatch (every rank passes the
        combine's closing barrier, after its experts have read them, before any rank
        writes that buffer again)."""
        R, me = self.R, self.me
        src = torch.full((ids.shape[0],), me, dtype=torch.int32, device=ids.device)
        plan = self.ops.plan(ids, self.E, self.expert_rank, R, self.rank_node, self.n_nodes, src)
        self.plan = plan
        self._ids = ids
        C, A = self._count_rows(plan)
        # the one host synchronisation of a layer: all_to_all_single takes its split sizes
        # as host lists, and the received tensors' shapes depend on the counts
        Cl, Al = C.cpu(), A.cpu()
        self._C, self._A = Cl, Al
        D = int(Cl[me].sum())
        # per send row and slot, computed by the library: the expert id, the gate and the
        # slot's output position in the destination's expanded receive order, i.e. past
        # the assignment rows that earlier sources send that rank
        base = (exclusive_offsets(A)[me] - plan.asg_offsets[:R].to(torch.int64)).to(torch.int32)
        ex, g, sl = self.ops.row_meta(plan, ids, gates, base)
        rows = self._send_rows(x, "recv")
        experts = self._rows_to_dest(ex[:D])
        slots = self._rows_to_dest(sl[:D])
        kmask = self._rows_to_dest(plan.row_kmask[:D].to(torch.int32))
        if g is not None:
            g = self._rows_to_dest(g[:D])
        self._d = Dispatched(rows=rows, kmask=kmask.to(torch.uint8), experts=experts, slots=slots,
                             counts=Cl, asg=Al, gates=g)
        return self._d

    def _rows_to_dest(self, t: torch.Tensor) -> torch.Tensor:
        """Per-send-row metadata (first dim D) to the destination ranks (first dim n_recv)."""
        me, Cl = self.me, self._C
        out = torch.empty((int(Cl[:, me].sum()),) + tuple(t.shape[1:]), dtype=t.dtype,
                          device=t.device)
        dist.all_to_all_single(out, t.contiguous(), Cl[:, me].tolist(), Cl[me].tolist(),
                               group=self.group)
        return out

    def _rows_to_source(self, t: torch.Tensor) -> torch.Tensor:
        """Per-received-row data (first dim n_recv) back to the token's rank, landing in
        send-row order (first dim D)."""
        me, Cl = self.me, self._C
        out = torch.empty((int(Cl[me].sum()),) + tuple(t.shape[1:]), dtype=t.dtype,
                          device=t.device)
        if t.dtype == torch.bfloat16:      # raw 32-bit words: exact on any backend
            dist.all_to_all_single(out.view(torch.int32), t.contiguous().view(torch.int32),
                                   Cl[me].tolist(), Cl[:, me].tolist(), group=self.group)
        else:
            dist.all_to_all_single(out, t.contiguous(), Cl[me].tolist(), Cl[:, me].tolist(),
                                   group=self.group)
        return out

    def _send_rows(self, x: torch.Tensor, buf: str) -> torch.Tensor:
        """Rows of this rank's tokens (bf16 [N, H]) to every destination rank of the current
        plan; returns the rows this rank receives (source rank, then token order)."""
        plan, Cl, me = self.plan, self._C, self.me
        D, n_recv, H = int(Cl[me].sum()), int(Cl[:, me].sum()), x.shape[1]
        if self.transport == "nccl":
            send = self.ops.gather(x, plan)
            rows = torch.empty((n_recv, H), dtype=x.dtype, device=x.device)
            # rows travel as raw 32-bit words (two bf16 each): exact, any backend
            dist.all_to_all_single(rows.view(torch.int32), send[:D].contiguous().view(torch.int32),
                                   Cl[:, me].tolist(), Cl[me].tolist(), group=self.group)
            return rows
        import co_activation_b200 as coact
        sb = self._symmetric(buf, int(Cl.sum(dim=0).max()), H, x.dtype, x.device)
        off = exclusive_offsets(Cl)[me].to(torch.int32).to(x.device)
        coact.dispatch_gather_peer(x, plan.send_row, plan.rank_offsets, sb["ptrs"], off, sb["cap"])
        sb["handle"].barrier()
        return sb["t"][:n_recv]

    def _sum_back(self, rows: torch.Tensor, buf: str, out: torch.Tensor) -> torch.Tensor:
        """Rows held per received row (n_recv of them, bf16) back to the token's rank and
        summed per token over its send rows: out[t] = sum of the rows of t's send rows."""
        plan, Cl, me = self.plan, self._C, self.me
        if self.transport == "nccl":
            back = self._rows_to_source(rows)
            return self.ops.gather_backward(back, plan.send_row, out)
        import co_activation_b200 as coact
        H = rows.shape[1]
        sb = self._symmetric(buf, int(Cl.sum(dim=0).max()), H, rows.dtype, rows.device)
        sb["t"][:rows.shape[0]].copy_(rows)
        sb["handle"].barrier()
        off = exclusive_offsets(Cl)[me].to(torch.int32).to(rows.device)
        coact.combine_scatter_peer(sb["ptrs"], off, sb["cap"], plan.rank_offsets, None,
                                   plan.send_row, out, H)
        sb["handle"].barrier()
        return out

    def combine(self, y_recv: torch.Tensor, gates: torch.Tensor,
                out: Optional[torch.Tensor] = None, reduce: str = "expanded") -> torch.Tensor:
        """Bring the expert outputs (expanded receive order on this rank) back to their
        source ranks and combine them in token order.  reduce="rows": pre-reduce where the
        experts ran (one bf16 partial row per received row; needs dispatch(..., gates))."""
        me, plan = self.me, self.plan
        Al = self._A
        H = y_recv.shape[1]
        N = gates.shape[0]
        if out is None:
            out = torch.empty((N, H), dtype=y_recv.dtype, device=y_recv.device)
        if reduce == "rows":
            d = self._d
            if d is None or d.gates is None:
                raise ValueError("reduce='rows' needs dispatch(..., gates=...) first")
            pre = torch.empty((d.rows.shape[0], H), dtype=torch.bfloat16, device=y_recv.device)
            self.ops.combine_local(y_recv, d.gates, d.slots, pre)
            return self._sum_back(pre, "pre", out)
        if reduce != "expanded":
            raise ValueError("reduce must be 'expanded' or 'rows'")
        if self.transport == "nccl":
            back = torch.empty((int(Al[me].sum()), H), dtype=y_recv.dtype, device=y_recv.device)
            dist.all_to_all_single(back.view(torch.int32), y_recv.contiguous().view(torch.int32),
                                   Al[me].tolist(), Al[:, me].tolist(), group=self.group)
            return self.ops.combine(back, gates, plan, out)
        return self._peer_combine(y_recv, gates, out)

    # ------------------------------------------------------------------ backward

    def backward_combine(self, grad_out: torch.Tensor, y_recv: torch.Tensor):
        """Gradients of combine() (either reduce mode; same function) for grad_out [N, H]
        (bf16, this rank's tokens).  Returns (grad_y, grad_gates): grad_y bf16 in expanded
        receive order on this rank (for the experts' backward), grad_gates fp32 [N, k] of
        this rank's tokens.  Needs dispatch(..., gates=...) first."""
        d, plan, me = self._d, self.plan, self.me
        if d is None or d.gates is None:
            raise ValueError("backward_combine needs dispatch(..., gates=...) first")
        N, k = self._ids.shape
        g_recv = self._send_rows(grad_out, "grad")
        grad_y = torch.empty_like(y_recv)
        gg = torch.zeros((d.rows.shape[0], k), dtype=torch.float32, device=y_recv.device)
        self.ops.combine_backward(y_recv, d.gates, d.slots, g_recv, grad_y, gg)
        back = self._rows_to_source(gg)                      # [D, k], send-row order
        grad_gates = torch.empty((N, k), dtype=torch.float32, device=y_recv.device)
        return grad_y, self.ops.gather_row_slots(back, plan, grad_gates)

    def backward_dispatch(self, grad_rows: torch.Tensor,
                          out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Gradient of dispatch(): grad_rows bf16 [n_recv, H] (one per received row) back to
        the token's rank, summed per token: grad_x [N, H] (bf16 or fp32 `out`)."""
        N = self._ids.shape[0]
        if out is None:
            out = torch.empty((N, grad_rows.shape[1]), dtype=grad_rows.dtype,
                              device=grad_rows.device)
        return self._sum_back(grad_rows, "gback", out)

    # ------------------------------------------------------------------ token shuffling

    def shuffle_reduce_scatter(self, partial: torch.Tensor, home: torch.Tensor,
                               out: Optional[torch.Tensor] = None):
        """partial: bf16 [N, H], this rank's partial attention output for all N tokens of
        the group; home: int32 [N], every token's predicted home rank (the same on every
        rank).  Returns (rows, tokens): the rows of the tokens homed on this rank in
        ascending token order, each the sum of the R partials in rank order, and their
        token indices."""
        R, me = self.R, self.me
        N, H = partial.shape
        sp = self.ops.shuffle_plan(home, R)
        offs = sp.rank_offsets.cpu()
        lo, hi = int(offs[me]), int(offs[me + 1])
        tokens = sp.row_token[lo:hi]
        if out is None:
            out = torch.empty((hi - lo, H), dtype=partial.dtype, device=partial.device)
        if self.transport == "peer":
            sb = self._symmetric("part", N, H, partial.dtype, partial.device)
            sb["t"][:N].copy_(partial)
            sb["handle"].barrier()
            import co_activation_b200 as coact
            coact.shuffle_reduce_scatter(sb["ptrs"], N, tokens, out)
            sb["handle"].barrier()
            return out, tokens
        counts = (offs[1:] - offs[:-1]).tolist()
        permuted = self.ops.gather(partial, sp)[:N]        # rank segments, ascending tokens
        recv = torch.empty((R * (hi - lo), H), dtype=partial.dtype, device=partial.device)
        dist.all_to_all_single(recv.view(torch.int32), permuted.contiguous().view(torch.int32),
                               [hi - lo] * R, counts, group=self.group)
        blocks = [recv[q * (hi - lo):(q + 1) * (hi - lo)] for q in range(R)]
        ident = torch.arange(hi - lo, dtype=torch.int32, device=partial.device)
        self.ops.shuffle_reduce(blocks, ident, hi - lo, out)
        return out, tokens

    # ------------------------------------------------------------------ peer transport

    def _symmetric(self, name, rows, H, dtype, device):
        """A named symmetric-memory buffer [>= rows, H] on every rank (all ranks ask for the
        same size: the group-wide maximum) and its per-rank device addresses."""
        import torch.distributed._symmetric_memory as symm
        sb = self._sym.get(name)
        if sb is None or sb["t"].shape[0] < rows or sb["t"].shape[1] != H or sb["t"].dtype != dtype:
            cap = max(rows, self.peer_capacity or 0, 1)
            t = symm.empty((cap, H), dtype=dtype, device=device)
            h = symm.rendezvous(t, self.group)
            sb = {"t": t, "handle": h,
                  "ptrs": torch.tensor(list(h.buffer_ptrs), dtype=torch.int64, device=device),
                  "cap": torch.full((self.R,), cap, dtype=torch.int32, device=device)}
            self._sym[name] = sb
        return sb

    def _peer_combine(self, y_recv, gates, out):
        import co_activation_b200 as coact
        Al, me = self._A, self.me
        H = y_recv.shape[1]
        cap = max(int(Al.sum(dim=0).max()), 8 * (self.peer_capacity or 0))
        sb = self._symmetric("y", cap, H, y_recv.dtype, y_recv.device)
        n = y_recv.shape[0]
        sb["t"][:n].copy_(y_recv)
        sb["handle"].barrier()
        off = exclusive_offsets(Al)[me].to(torch.int32).to(out.device)
        coact.combine_scatter_peer(sb["ptrs"], off, sb["cap"], self.plan.asg_offsets, gates,
                                   self.plan.comb_row, out, H)
        sb["handle"].barrier()
        return out


def expand_identity(d: Dispatched) -> torch.Tensor:
    """Identity experts: one output row per set slot of every received row, in expanded
    receive order (for tests and demonstrations)."""
    reps = torch.bitwise_count(d.kmask.to(torch.int32)).to(torch.int64) \
        if hasattr(torch, "bitwise_count") else \
        torch.tensor([bin(int(v)).count("1") for v in d.kmask.cpu()], device=d.rows.device)
    return d.rows.repeat_interleave(reps, dim=0)
