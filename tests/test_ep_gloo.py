"""Expert parallelism across ranks, host logic on CPU: gloo ranks, each with its own
contiguous block of tokens, run co_activation_b200.ep.EPLayer (transport "nccl", i.e.
torch.distributed all-to-all) with the oracle standing in for the local kernels.  Every
rank must receive exactly the rank-r segment of the single-process plan of all tokens,
with the right expert ids, and get back the combined rows of its own tokens bit for bit
(identity experts: the naive combine).  The global pair counts must be the oracle's."""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleOps:
    """The EP layer's local steps through the CPU oracle (test double)."""

    def __init__(self, oracle):
        self.o = oracle

    def plan(self, ids, E, expert_rank, R, rank_node, n_nodes, src_rank):
        p = self.o.plan(ids.numpy(), E, expert_rank.numpy(), R,
                        rank_node=None if rank_node is None else rank_node.numpy(),
                        n_nodes=n_nodes, src_rank=src_rank.numpy())
        t = lambda k: torch.from_numpy(np.ascontiguousarray(p[k]))
        return types.SimpleNamespace(row_token=t("row_token"), row_kmask=t("row_kmask"),
                                     send_row=t("send_row"), comb_row=t("comb_row"),
                                     rank_counts=t("rank_counts"), rank_offsets=t("rank_offsets"),
                                     asg_offsets=t("asg_offsets"),
                                     row_capacity=len(p["row_token"]))

    def gather(self, x, plan):
        D = int(plan.rank_offsets[-1])
        rows = self.o.gather(self.o._bits(x), plan.row_token.numpy(), D)
        out = torch.zeros((plan.row_capacity, x.shape[1]), dtype=torch.int16)
        out[:D] = torch.from_numpy(rows.view(np.int16))
        return out.view(torch.bfloat16)

    def combine(self, y, gates, plan, out):
        c = self.o.combine_f32chain(self.o._bits(y), gates.numpy(), plan.comb_row.numpy())
        out.copy_(torch.from_numpy(c))
        return out

    def count(self, ids, E, pair, loads):
        p, l, _ = self.o.count(ids.numpy(), E)
        pair += torch.from_numpy(p)
        loads += torch.from_numpy(l)

    def _store(self, out, f32):
        if out.dtype == torch.bfloat16:
            out.view(torch.int16).copy_(torch.from_numpy(self.o.bf16_rne(f32).view(np.int16)))
        else:
            out.copy_(torch.from_numpy(f32))
        return out

    def combine_local(self, y, gates, comb, out):
        return self._store(out, self.o.combine_f32chain(self.o._bits(y), gates.numpy(), comb.numpy()))

    def gather_backward(self, rows, send_row, out):
        return self._store(out, self.o.gather_backward_f32chain(self.o._bits(rows), send_row.numpy()))

    def shuffle_plan(self, home, R):
        p = self.o.shuffle_order(home.numpy(), R)
        t = lambda k: torch.from_numpy(np.ascontiguousarray(p[k]))
        return types.SimpleNamespace(row_token=t("row_token"), row_kmask=t("row_kmask"),
                                     send_row=t("send_row"), comb_row=t("comb_row"),
                                     rank_counts=t("rank_counts"), rank_offsets=t("rank_offsets"),
                                     asg_offsets=t("asg_offsets"),
                                     row_capacity=len(p["row_token"]))

    def shuffle_reduce(self, blocks, row_token, N, out):
        parts = np.stack([self.o._bits(b) for b in blocks])
        return self._store(out, self.o.shuffle_reduce_f32chain(parts, row_token.numpy()))

    def row_meta(self, plan, ids, gates, slot_base):
        p = {"D": int(plan.rank_offsets[-1]), "rank_offsets": plan.rank_offsets.numpy(),
             "row_token": plan.row_token.numpy(), "row_kmask": plan.row_kmask.numpy(),
             "comb_row": plan.comb_row.numpy()}
        g = np.zeros(ids.shape, np.float32) if gates is None else gates.numpy()
        ex, gt, sl, f = self.o.row_meta(p, ids.numpy(), g, slot_base=slot_base.numpy())
        assert f == 0
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        return t(ex), (None if gates is None else t(gt)), t(sl)

    def gather_row_slots(self, vals, plan, out):
        got, f = self.o.gather_row_slots(vals.numpy(), plan.send_row.numpy(), plan.row_kmask.numpy())
        assert f == 0
        out.copy_(torch.from_numpy(got))
        return out

    def combine_backward(self, y, gates, comb, g_out, g_y, g_gates):
        gy, gg, _ = self.o.combine_backward(self.o._bits(y), gates.numpy(), comb.numpy(),
                                            self.o._bits(g_out))
        g_y.view(torch.int16).copy_(torch.from_numpy(gy.view(np.int16)))
        g_gates.copy_(torch.from_numpy(gg.astype(np.float32)))
        return g_y, g_gates


def _worker(rank, world, port, cfg_spec, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workload
        import co_activation_b200.ep as ep
        N, E, k, H = cfg_spec
        cfg = workload.CONFIGS[0].with_(N=N, E=E, k=k, H=H, R=world, n_nodes=1)
        r = workload.make_routing(cfg)
        lo, hi = rank * N // world, (rank + 1) * N // world
        ids = torch.from_numpy(r.ids[lo:hi].copy())
        gates = torch.from_numpy(r.gates[lo:hi].copy())
        x = workload.fill_bf16(N, H, 0, 1)
        xl = x[lo:hi].contiguous()
        layer = ep.EPLayer(dist.group.WORLD, E, torch.from_numpy(r.expert_rank), transport="nccl",
                           ops=OracleOps(oracle))
        pair = torch.zeros((E, E), dtype=torch.int64)
        loads = torch.zeros(E, dtype=torch.int64)
        layer.count(ids, pair, loads)
        got = layer.dispatch(ids, xl)
        y = ep.expand_identity(got)
        res = layer.combine(y, gates, torch.empty((hi - lo, H), dtype=torch.float32))
        # expectations from the single-process plan of all tokens, homed by block
        src = np.repeat(np.arange(world), np.diff([i * N // world for i in range(world + 1)]))
        full = oracle.plan(r.ids, E, r.expert_rank, world, src_rank=src.astype(np.int32))
        seg = slice(full["rank_offsets"][rank], full["rank_offsets"][rank + 1])
        tok = full["row_token"][seg]
        xb = oracle._bits(x)
        want_rows = xb[tok]
        km = full["row_kmask"][seg]
        want_exp = np.where((km[:, None] >> np.arange(k)) & 1, r.ids[tok], -1)
        want_out = oracle.naive_combine_identity_f32(xb[lo:hi], r.gates[lo:hi])
        op, ol, _ = oracle.count(r.ids, E)
        out[rank] = (
            np.array_equal(oracle._bits(got.rows), want_rows),
            np.array_equal(got.kmask.numpy(), km),
            np.array_equal(got.experts.numpy(), want_exp),
            np.array_equal(res.numpy().view(np.uint32), want_out.view(np.uint32)),
            np.array_equal(pair.numpy(), op) and np.array_equal(loads.numpy(), ol),
            int(got.rows.shape[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,spec", [(2, (4096, 8, 2, 64)), (3, (1000, 12, 3, 32))])
def test_ep_exchange_matches_single_process_plan(world, spec):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, spec, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    for r in range(world):
        rows_ok, km_ok, exp_ok, out_ok, cnt_ok, n = out[r]
        assert rows_ok and km_ok and exp_ok, f"rank {r}: received rows or metadata differ"
        assert out_ok, f"rank {r}: combined rows differ"
        assert cnt_ok, f"rank {r}: global counts differ"
        assert n > 0


def _worker_backward(rank, world, port, cfg_spec, out):
    """Pre-reduced combine and the backward pass across gloo ranks against the oracle's
    single-process results over all tokens."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workload
        import co_activation_b200.ep as ep
        N, E, k, H = cfg_spec
        cfg = workload.CONFIGS[0].with_(N=N, E=E, k=k, H=H, R=world, n_nodes=1)
        r = workload.make_routing(cfg)
        lo, hi = rank * N // world, (rank + 1) * N // world
        ids = torch.from_numpy(r.ids[lo:hi].copy())
        gates = torch.from_numpy(r.gates[lo:hi].copy())
        x = workload.fill_bf16(N, H, 0, 1)
        g_out = workload.fill_bf16(N, H, 0, 6)
        layer = ep.EPLayer(dist.group.WORLD, E, torch.from_numpy(r.expert_rank), transport="nccl",
                           ops=OracleOps(oracle))
        got = layer.dispatch(ids, x[lo:hi].contiguous(), gates=gates)
        y = workload.fill_bf16(int(got.asg[:, rank].sum()), H, rank, 2)   # this rank's outputs
        pre_out = layer.combine(y, gates, torch.empty((hi - lo, H), dtype=torch.float32),
                                reduce="rows")
        grad_y, grad_gates = layer.backward_combine(g_out[lo:hi].contiguous(), y)
        src = np.repeat(np.arange(world), np.diff([i * N // world for i in range(world + 1)]))
        full = oracle.plan(r.ids, E, r.expert_rank, world, src_rank=src.astype(np.int32))
        ro, ao = full["rank_offsets"], full["asg_offsets"]
        G = workload.fill_bf16(int(ro[-1]), H, 0, 7)                     # input-gradient rows
        grad_x = layer.backward_dispatch(G[ro[rank]:ro[rank + 1]].contiguous(),
                                         torch.empty((hi - lo, H), dtype=torch.float32))
        # single-process expectations: every rank's outputs at its assignment segment
        ys = [oracle._bits(workload.fill_bf16(int(ao[q + 1] - ao[q]), H, q, 2)) for q in range(world)]
        y_full = np.concatenate(ys)
        seg = slice(ro[rank], ro[rank + 1])
        tok, km = full["row_token"][seg], full["row_kmask"][seg]
        want_g = np.where((km[:, None] >> np.arange(k)) & 1, r.gates[tok], 0).astype(np.float32)
        # each served slot's output position on this rank: its place in the single-process
        # plan's rank segment of assignments
        want_s = np.where((km[:, None] >> np.arange(k)) & 1, full["comb_row"][tok] - ao[rank], -1)
        _, pre_want = oracle.combine_prereduced(y_full, r.gates, full)
        gy_w, gg_w, _ = oracle.combine_backward(y_full, r.gates, full["comb_row"], oracle._bits(g_out))
        gx_w = oracle.gather_backward_f32chain(oracle._bits(G), full["send_row"])
        out[rank] = (
            np.array_equal(got.gates.numpy().view(np.uint32), want_g.view(np.uint32)),
            np.array_equal(got.slots.numpy(), want_s),
            np.array_equal(pre_out.numpy().view(np.uint32), pre_want[lo:hi].view(np.uint32)),
            np.array_equal(oracle._bits(grad_y), gy_w[ao[rank]:ao[rank + 1]]),
            np.array_equal(grad_gates.numpy(), gg_w[lo:hi].astype(np.float32)),
            np.array_equal(grad_x.numpy().view(np.uint32), gx_w[lo:hi].view(np.uint32)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,spec", [(2, (2048, 8, 2, 32)), (3, (999, 12, 4, 24))])
def test_ep_prereduced_and_backward_match_single_process(world, spec):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker_backward, args=(r, world, port, spec, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    names = ("exchanged gates", "output slots", "pre-reduced combine", "grad_y", "grad_gates",
             "grad_x")
    for r in range(world):
        for name, ok in zip(names, out[r]):
            assert ok, f"rank {r}: {name} differs from the single-process oracle"


def _worker_shuffle(rank, world, port, spec, out):
    """Token shuffling in the reduce-scatter across gloo ranks against the oracle over all
    ranks' partials."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workload
        import co_activation_b200.ep as ep
        N, H = spec
        rng = np.random.default_rng(7)
        home = rng.integers(0, world, N).astype(np.int32)
        home[: N // 3] = 0                         # uneven segments
        partial = workload.fill_bf16(N, H, 0, 100 + rank)
        layer = ep.EPLayer(dist.group.WORLD, 8, torch.zeros(8, dtype=torch.int32),
                           transport="nccl", ops=OracleOps(oracle))
        rows, tokens = layer.shuffle_reduce_scatter(partial, torch.from_numpy(home),
                                                    torch.empty((int((home == rank).sum()), H),
                                                                dtype=torch.float32))
        parts = np.stack([oracle._bits(workload.fill_bf16(N, H, 0, 100 + q)) for q in range(world)])
        want_tok = np.flatnonzero(home == rank).astype(np.int32)
        want = oracle.shuffle_reduce_f32chain(parts, want_tok)
        out[rank] = (np.array_equal(tokens.numpy(), want_tok),
                     np.array_equal(rows.numpy().view(np.uint32), want.view(np.uint32)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,spec", [(2, (1000, 32)), (3, (777, 24))])
def test_ep_shuffle_reduce_scatter_matches_oracle(world, spec):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker_shuffle, args=(r, world, port, spec, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    for r in range(world):
        tok_ok, rows_ok = out[r]
        assert tok_ok, f"rank {r}: shuffled tokens differ"
        assert rows_ok, f"rank {r}: reduced rows differ"
