"""Benchmark of the co-activation dispatch/combine hot path on B200.

One step = one pass of the whole path over one batch of N tokens:
  coact_count (pair counts + loads) -> plan_dispatch -> dispatch_gather
  -> combine_scatter (bf16 out)
with inputs already resident in HBM.  Default workload: config 3, the largest
single-GPU configuration (N=131072, E=256, top-8, H=7168 bf16, 64 logical ranks of 4
experts in 8 nodes, Zipf(1.2) expert popularity, 32 planted pairs), with the correlated
placement the library builds from the batch's own pair counts; seeded synthetic routing.
`--config 1` selects the small single-node case (N=16384, E=64, top-2, H=2048); config 4
is two consecutive layers with token shuffling (cross-layer counts, predicted home ranks).

Timing: W untimed warm-up steps, then EXACTLY K steps captured in one CUDA graph, each
step bracketed by CUDA events on the launching stream, with an L2 flush between steps
outside the events.  A barrier and torch.cuda.synchronize() bracket the timed region;
multi-GPU runs (torchrun, one rank per GPU, each rank its own batch: weak scaling, no
data-path collective) report the max over ranks.  `e2e` times the same step through the
public API from pinned host buffers.  `--impl reference` times the CPU oracle instead
(rank 0 only).

Prints ONE JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from typing import Optional

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload  # noqa: E402

METRIC = "dispatch+combine tokens/s and HBM GB/s (% of ~8 TB/s); dedup rows/naive rows"
UNIT = "tokens/s"
X_STREAM, Y_STREAM, Y2_STREAM = 1, 2, 3


# ----------------------------------------------------------------------------- helpers


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms in the background."""

    FIELDS = ("clocks.sm,clocks.max.sm,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", "50"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, n_load = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                clk, cmax, util = float(parts[0]), float(parts[1]), float(parts[2])
            except ValueError:
                continue
            smax = cmax
            if util > 0:
                n_load += 1
                sm.append(clk)
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples_under_load": n_load}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(v: float, world: int, device) -> float:
    """Max over ranks (timing: the slowest rank sets the job's time)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(v: float, world: int, device) -> float:
    """Sum over ranks (work: every rank processes its own batch)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: independent problems per GPU)."""
    return base_seed + rank


def aggregate(tokens_per_rank: float, seconds_per_rank: float, world: int, device) -> dict:
    """Whole-job throughput: all ranks' tokens over the slowest rank's device time."""
    total_s = reduce_max(seconds_per_rank, world, device)
    tokens = reduce_sum(tokens_per_rank, world, device)
    return {"tokens": tokens, "seconds": total_s, "tokens_per_s": tokens / total_s}


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- one layer


class LayerBuffers:
    """Device buffers and the four library calls of one MoE layer."""
    tma = False                 # gather through dispatch_gather_tma (--gather tma)

    @classmethod
    def gather_kernel(cls) -> str:
        return "k_gather_bulk" if cls.tma else "k_gather_v16"

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True,
                 y_stream: int = Y_STREAM, x=None):
        cfg = r.cfg
        self.coact, self.r, self.cfg, self.dev = coact, r, cfg, device
        N, k, E, R, H = cfg.N, cfg.k, cfg.E, cfg.R, cfg.H
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.ids = to(r.ids)
        self.gates = to(r.gates)
        self.expert_rank = to(r.expert_rank.astype(np.int32))
        self.rank_node = to(r.rank_node.astype(np.int32))
        self.src_rank = None
        if x is not None:
            self.x = x                                     # fed by an earlier layer
        elif fill:
            self.x = workload.fill_bf16(N, H, r.seed, X_STREAM, device=device)
        else:                                              # contents arrive by copy
            self.x = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        if fill:
            self.y = workload.fill_bf16(N * k, H, r.seed, y_stream, device=device)
        else:
            self.y = torch.empty((N * k, H), dtype=torch.bfloat16, device=device)
        self.pair = torch.zeros((E, E), dtype=torch.int64, device=device)
        self.loads = torch.zeros(E, dtype=torch.int64, device=device)
        self.plan = coact.alloc_plan(N, k, E, R, device)
        self.send = torch.empty((self.plan.row_capacity, H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)

    def count(self):
        self.coact.coact_count(self.ids, self.cfg.E, self.pair, self.loads, err_flag=self.err)

    def plan_(self):
        self.coact.plan_dispatch(self.ids, self.cfg.E, self.expert_rank, self.cfg.R, self.plan,
                                 rank_node=self.rank_node, n_nodes=self.cfg.n_nodes,
                                 src_rank=self.src_rank, err_flag=self.err)

    def gather(self):
        self.coact.dispatch_gather(self.x, self.plan.send_row, self.send, err_flag=self.err,
                                   tma=self.tma)

    def combine(self):
        self.coact.combine_scatter(self.y, self.gates, self.plan.comb_row, self.out,
                                   err_flag=self.err)

    def D(self) -> int:
        return int(self.plan.rank_offsets[-1].item())

    def bytes_gather(self, D):
        c = self.cfg
        return (c.N + D) * c.H * 2 + c.N * c.k * 4

    def bytes_combine(self):
        c = self.cfg
        return c.N * c.k * c.H * 2 + c.N * c.H * 2 + c.N * c.k * 8


def rank_balance(plan) -> dict:
    """Receive-side balance of a plan: the busiest rank's rows and assignments over the
    mean (1.0 = perfectly even)."""
    rows = plan.rank_counts.cpu().numpy().astype(np.float64)
    ao = plan.asg_offsets.cpu().numpy().astype(np.float64)
    asg = ao[1:] - ao[:-1]
    ratio = lambda a: float(a.max() / a.mean()) if a.mean() > 0 else 0.0
    return {"rank_rows_max_over_mean": ratio(rows), "rank_asg_max_over_mean": ratio(asg)}


def plan_launches(R: int, N: int) -> int:
    """Kernels plan_dispatch launches: 2 when R x tiles <= 4096 (scan folded), else 3."""
    return 2 if R * (-(-N // 256)) <= 4096 else 3


class OneLayerStep:
    """plan -> gather -> combine, with the count on a side stream beside the gather (it
    depends on nothing the other calls produce; beside the HBM-bound gather it takes SMs
    the copy leaves idle, where beside the latency-bound plan it slowed the plan)."""
    n_events = 5
    phases = {"coact_count": (2, 1), "plan_dispatch": (0, 2), "dispatch_gather": (2, 3),
              "combine_scatter": (3, 4)}
    host_inputs = ("ids", "gates", "expert_rank", "rank_node", "x", "y")

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        self.L = LayerBuffers(coact, r, device, fill)
        self.cfg, self.N = r.cfg, r.cfg.N
        self.side = torch.cuda.Stream(device=device)
        self.kernels_per_step = 1 + plan_launches(r.cfg.R, self.N) + 1 + 1

    def inputs(self):
        return {n: getattr(self.L, n) for n in self.host_inputs}

    def outputs(self):
        return [self.L.out, self.L.plan.stats]

    def clone_for_copy(self, coact, device):
        c = OneLayerStep(coact, self.L.r, device, fill=False)
        return c

    def count_beside(self, main, ev, i_end):
        """The count on the side stream from this point of the main stream; ev[i_end]
        marks its end."""
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self.L.count()
            if ev: ev[i_end].record()

    def step(self, ev=None):
        main = torch.cuda.current_stream()
        if ev: ev[0].record()
        self.L.plan_()
        if ev: ev[2].record()
        self.count_beside(main, ev, 1)
        self.L.gather()
        if ev: ev[3].record()
        self.L.combine()
        main.wait_stream(self.side)
        if ev: ev[4].record()

    def roofline_parts(self):
        """(phase, kernel, algorithmic bytes) for the HBM-bound kernels."""
        D = self.L.D()
        return [("dispatch_gather", LayerBuffers.gather_kernel(), self.L.bytes_gather(D)),
                ("combine_scatter", "k_combine_v16", self.L.bytes_combine())]

    def summary(self):
        L = self.L
        return {"dedup_rows_over_naive": L.D() / (self.N * self.cfg.k),
                **rank_balance(L.plan),
                "stats": dict(zip(L.coact.STAT_NAMES, L.plan.stats.cpu().tolist())),
                "err_flag": int(L.err.item())}


class TwoLayerStep:
    """Config 4: two consecutive MoE layers.  Layer 1 as above with contiguous home
    ranks; then cross-layer counts (layer-1 x layer-2 picks, accumulated for the next
    prediction), home-rank prediction from the calibration counts, and layer 2 with its
    tokens pre-sharded to the predicted rank; layer 2's input rows are layer 1's output."""
    n_events = 11
    phases = {"layer1_plan": (0, 1), "layer1_gather": (1, 2), "layer1_combine": (2, 3),
              "layer2_plan": (4, 5), "layer2_gather": (5, 6), "layer2_combine": (6, 7),
              "side_counts": (0, 8), "side_predict_home": (8, 9)}   # ev8, ev9: side stream

    def __init__(self, coact, tl: workload.TwoLayer, device, fill: bool = True, C12=None):
        self.coact, self.tl = coact, tl
        self.cfg = tl.layer1.cfg
        self.N = self.cfg.N
        E, R = self.cfg.E, self.cfg.R
        self.L1 = LayerBuffers(coact, tl.layer1, device, fill, Y_STREAM)
        self.L2 = LayerBuffers(coact, tl.layer2, device, fill, Y2_STREAM, x=self.L1.out)
        self.home = torch.empty(self.N, dtype=torch.int32, device=device)
        self.L2.src_rank = self.home
        self.pws = torch.empty(max(coact.predict_workspace_bytes(E, R), 16), dtype=torch.uint8,
                               device=device)
        self.C12_live = torch.zeros((E, E), dtype=torch.int64, device=device)
        if C12 is None:        # calibration batch (seed + 1) counted by the library
            C12 = torch.zeros((E, E), dtype=torch.int64, device=device)
            to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            coact.coact_count(to(tl.calib1), E, C12, ids2=to(tl.calib2), E2=E)
        self.C12 = C12
        self.side = torch.cuda.Stream(device=device)
        self.home_ready = torch.cuda.Event()
        # counts: 2 per layer-set + 1 cross; two plans; 2 gathers; 2 combines; predict 2
        self.kernels_per_step = 3 + 2 * plan_launches(R, self.N) + 2 + 2 + 2

    def inputs(self):
        return {"ids1": self.L1.ids, "gates1": self.L1.gates, "er1": self.L1.expert_rank,
                "rn1": self.L1.rank_node, "x1": self.L1.x, "y1": self.L1.y,
                "ids2": self.L2.ids, "gates2": self.L2.gates, "er2": self.L2.expert_rank,
                "y2": self.L2.y, "C12": self.C12}

    def outputs(self):
        return [self.L2.out, self.L2.plan.stats]

    def clone_for_copy(self, coact, device):
        return TwoLayerStep(coact, self.tl, device, fill=False, C12=torch.empty_like(self.C12))

    def step(self, ev=None):
        c, E, R = self.coact, self.cfg.E, self.cfg.R
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        if ev: ev[0].record()
        with torch.cuda.stream(self.side):
            # statistics, and the layer-2 home prediction: it needs only layer 1's picks
            # and the calibration counts, so it runs beside layer 1's dispatch and combine
            self.L1.count()
            c.coact_count(self.L1.ids, E, self.C12_live, ids2=self.L2.ids, E2=E,
                          err_flag=self.L1.err)
            self.L2.count()
            if ev: ev[8].record()
            c.predict_home(self.L1.ids, E, self.C12, self.L2.expert_rank, R, self.home,
                           workspace=self.pws, err_flag=self.L1.err)
            if ev: ev[9].record()
            self.home_ready.record(self.side)
        self.L1.plan_()
        if ev: ev[1].record()
        self.L1.gather()
        if ev: ev[2].record()
        self.L1.combine()
        if ev: ev[3].record()
        main.wait_event(self.home_ready)
        if ev: ev[4].record()
        self.L2.plan_()
        if ev: ev[5].record()
        self.L2.gather()
        if ev: ev[6].record()
        self.L2.combine()
        if ev: ev[7].record()
        main.wait_stream(self.side)
        if ev: ev[10].record()

    def roofline_parts(self):
        D1, D2 = self.L1.D(), self.L2.D()
        return [("layer1_gather", LayerBuffers.gather_kernel(), self.L1.bytes_gather(D1)),
                ("layer1_combine", "k_combine_v16", self.L1.bytes_combine()),
                ("layer2_gather", LayerBuffers.gather_kernel(), self.L2.bytes_gather(D2)),
                ("layer2_combine", "k_combine_v16", self.L2.bytes_combine())]

    def summary(self):
        nk = self.N * self.cfg.k
        st2 = self.L2.plan.stats.cpu().tolist()
        # the same layer-2 batch with contiguous home ranks, for comparison
        base = self.coact.alloc_plan(self.N, self.cfg.k, self.cfg.E, self.cfg.R, self.L2.dev)
        self.coact.plan_dispatch(self.L2.ids, self.cfg.E, self.L2.expert_rank, self.cfg.R, base,
                                 rank_node=self.L2.rank_node, n_nodes=self.cfg.n_nodes)
        stb = base.stats.cpu().tolist()
        return {"dedup_rows_over_naive": self.L2.D() / nk,
                "layer1_dedup_rows_over_naive": self.L1.D() / nk,
                "local_served_share_predicted_home": st2[5] / nk,
                "local_served_share_contiguous_home": stb[5] / nk,
                "crossnode_asg_share_predicted_home": st2[7] / nk,
                "crossnode_asg_share_contiguous_home": stb[7] / nk,
                "stats": dict(zip(self.coact.STAT_NAMES, st2)),
                "err_flag": int(self.L1.err.item()) | int(self.L2.err.item())}


class TwoHopStep(OneLayerStep):
    """One layer with the two-hop dispatch (Cobalt: fewer remote nodes): node-level plan +
    rank-level plan + forward map -> hop-1 gather into node segments (count beside it on a
    side stream) -> hop-2 forward into rank segments -> combine.  The forward runs in token
    order (forward_gather_tokens: each hop-1 row read once) unless forward = "rows"."""
    forward = "tokens"
    n_events = 6
    phases = {"coact_count": (2, 1), "plan_two_hop": (0, 2), "gather_hop1": (2, 3),
              "forward_hop2": (3, 4), "combine_scatter": (4, 5)}

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        super().__init__(coact, r, device, fill)
        c = r.cfg
        self.th = coact.alloc_two_hop(c.N, c.k, c.E, c.R, c.n_nodes, device)
        self.hop1 = torch.empty((self.th.node.row_capacity, c.H), dtype=torch.bfloat16,
                                device=device)
        # counts 1; compose 2; node plan + rank plan; forward 1; hop-1 gather; hop-2; combine
        self.kernels_per_step = 1 + 2 + plan_launches(c.n_nodes, c.N) + plan_launches(c.R, c.N) \
            + 1 + 1 + 1 + 1

    def clone_for_copy(self, coact, device):
        return TwoHopStep(coact, self.L.r, device, fill=False)

    def step(self, ev=None):
        L, c = self.L, self.cfg
        main = torch.cuda.current_stream()
        if ev: ev[0].record()
        L.coact.plan_two_hop(L.ids, c.E, L.expert_rank, c.R, L.rank_node, c.n_nodes, self.th,
                             err_flag=L.err)
        if ev: ev[2].record()
        self.count_beside(main, ev, 1)
        L.coact.dispatch_gather(L.x, self.th.node.send_row, self.hop1, err_flag=L.err,
                                tma=L.tma)
        if ev: ev[3].record()
        if self.forward == "rows":
            L.coact.forward_gather(self.hop1, self.th.fwd_src, L.send, err_flag=L.err)
        else:
            L.coact.forward_gather_tokens(self.hop1, self.th.rank.send_row, self.th.fwd_src,
                                          L.send, err_flag=L.err)
        if ev: ev[4].record()
        L.coact.combine_scatter(L.y, L.gates, self.th.rank.comb_row, L.out, err_flag=L.err)
        main.wait_stream(self.side)
        if ev: ev[5].record()

    def roofline_parts(self):
        c = self.cfg
        Dn = int(self.th.node.rank_offsets[-1].item())
        D = int(self.th.rank.rank_offsets[-1].item())
        return [("gather_hop1", LayerBuffers.gather_kernel(),
                 (c.N + Dn) * c.H * 2 + c.N * c.k * 4),
                (("forward_hop2", "k_forward_gather", 2 * D * c.H * 2 + D * 4)
                 if self.forward == "rows" else
                 ("forward_hop2", "k_forward_tokens",
                  (Dn + D) * c.H * 2 + c.N * c.k * 4 + D * 4)),
                ("combine_scatter", "k_combine_v16", self.L.bytes_combine())]

    def summary(self):
        c, nk = self.cfg, self.N * self.cfg.k
        sn = self.th.node.stats.cpu().tolist()
        sr = self.th.rank.stats.cpu().tolist()
        return {"dedup_rows_over_naive": sr[1] / nk,
                "hop1_node_rows": sn[1], "hop1_remote_node_rows": sn[2],
                "rank_rows": sr[1], "one_hop_crossnode_rows": sr[3],
                "crossnode_rows_cut_by_two_hop": 1 - sn[2] / max(sr[3], 1),
                "stats": dict(zip(self.L.coact.STAT_NAMES, sr)),
                "err_flag": int(self.L.err.item())}


def layout(coact, r: workload.Routing, kind: str, device):
    """Expert -> rank placement from the batch's own counts (library calls):
    'correlated' = rank-level co-location (Zyphra), 'two-stage' = node-level co-location
    then intra-node load rebalancing (Cobalt).  Returns (expert_rank numpy, description)."""
    c = r.cfg
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=device)
    loads = torch.zeros(c.E, dtype=torch.int64, device=device)
    coact.coact_count(to(r.ids), c.E, pair, loads)
    if kind == "correlated":
        return coact.coact_place_correlated(pair, c.R).numpy(), \
            "correlated (coact_place_correlated over this batch's pair counts)"
    if kind == "two-stage":
        return coact.coact_place_two_stage(pair, loads, torch.from_numpy(r.rank_node),
                                           c.n_nodes).numpy(), \
            "two-stage (node co-location + intra-node load rebalancing over this batch)"
    raise SystemExit(f"unknown placement {kind}")


class RebalanceStep(OneLayerStep):
    """One layer with Cobalt's two-stage layout planner: stage 1 (periodic, outside the
    step) co-locates co-activated experts on nodes from the batch's pair counts; stage 2
    runs every step on the device -- fresh loads from coact_count, rebalance_ranks inside
    each node, and the plan over that placement -- then gather and combine.  Nothing in the
    step returns to the host."""
    n_events = 6
    phases = {"coact_count": (0, 1), "rebalance_ranks": (1, 2), "plan_dispatch": (2, 3),
              "dispatch_gather": (3, 4), "combine_scatter": (4, 5)}

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        super().__init__(coact, r, device, fill)
        c = r.cfg
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=device)
        coact.coact_count(to(r.ids), c.E, pair)
        self.expert_node = to(coact.coact_place_correlated(pair, c.n_nodes).numpy())
        self.er = torch.empty(c.E, dtype=torch.int32, device=device)
        self.kernels_per_step = 1 + 1 + plan_launches(c.R, self.N) + 1 + 1
        self.step_desc = ("coact_count (fresh loads) + rebalance_ranks (per-step intra-node "
                          "rebalance on the device; node co-location from the batch's pair "
                          "counts, outside the step) + plan_dispatch + dispatch_gather + "
                          "combine_scatter (bf16 out)")

    def clone_for_copy(self, coact, device):
        return RebalanceStep(coact, self.L.r, device, fill=False)

    def step(self, ev=None):
        L, c, cfg = self.L, self.L.coact, self.cfg
        if ev: ev[0].record()
        L.pair.zero_()
        L.loads.zero_()
        L.count()
        if ev: ev[1].record()
        c.rebalance_ranks(L.loads, self.expert_node, L.rank_node, cfg.n_nodes, out=self.er,
                          err_flag=L.err)
        if ev: ev[2].record()
        c.plan_dispatch(L.ids, cfg.E, self.er, cfg.R, L.plan, rank_node=L.rank_node,
                        n_nodes=cfg.n_nodes, src_rank=L.src_rank, err_flag=L.err)
        if ev: ev[3].record()
        L.gather()
        if ev: ev[4].record()
        L.combine()
        if ev: ev[5].record()

    def summary(self):
        out = super().summary()
        loads = self.L.loads.cpu().numpy()
        er = self.er.cpu().numpy()
        rank_load = np.bincount(er, weights=loads, minlength=self.cfg.R)
        out["rank_load_max_over_mean"] = float(rank_load.max() / rank_load.mean())
        return out


class PreReducedStep(OneLayerStep):
    """One layer with the pre-reduced reverse path: count (side stream, beside the plan) ->
    plan -> gather -> combine_rows over the send rows (one bf16 partial row per (token,
    rank), D rows instead of N*k) -> dispatch_gather_backward adds each token's partial
    rows.  Here the count stays beside the plan: run beside the gather, its shared-memory
    carveout outlasted it on SMs the gather kept busy, and combine_rows, whose loads in
    flight are staged in L1, lost more than the plan gained (config 3: 6,644 vs 6,622 us)."""
    n_events = 6
    phases = {"coact_count": (0, 1), "plan_dispatch": (0, 2), "dispatch_gather": (2, 3),
              "combine_rows": (3, 4), "reduce_rows": (4, 5)}
    step_desc = ("coact_count (side stream, beside the plan) + plan_dispatch + dispatch_gather + combine_rows "
                 "(partial rows per send row) + dispatch_gather_backward (sum per token, bf16 out)")

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        super().__init__(coact, r, device, fill)
        self.pre = torch.empty((self.L.plan.row_capacity, r.cfg.H), dtype=torch.bfloat16,
                               device=device)
        self.kernels_per_step = 1 + plan_launches(r.cfg.R, self.N) + 1 + 2

    def clone_for_copy(self, coact, device):
        return PreReducedStep(coact, self.L.r, device, fill=False)

    def step(self, ev=None):
        L, c = self.L, self.L.coact
        main = torch.cuda.current_stream()
        if ev: ev[0].record()
        self.count_beside(main, ev, 1)
        L.plan_()
        if ev: ev[2].record()
        L.gather()
        if ev: ev[3].record()
        # units: the plan's send rows, as many as the device-side D = rank_offsets[R]
        c.combine_rows(L.y, L.gates, L.plan.comb_row, L.plan.row_token, L.plan.row_kmask,
                       self.pre, unit_count=L.plan.rank_offsets[self.cfg.R:], err_flag=L.err)
        if ev: ev[4].record()
        c.dispatch_gather_backward(self.pre, L.plan.send_row, L.out, err_flag=L.err)
        main.wait_stream(self.side)
        if ev: ev[5].record()

    def roofline_parts(self):
        c, D = self.cfg, self.L.D()
        return [("dispatch_gather", LayerBuffers.gather_kernel(), self.L.bytes_gather(D)),
                ("combine_rows", "k_combine_v16",
                 c.N * c.k * c.H * 2 + D * c.H * 2 + D * 5 + c.N * c.k * 8),
                ("reduce_rows", "k_combine_v16", D * c.H * 2 + c.N * c.H * 2 + c.N * c.k * 4)]


class ReplicaStep(OneLayerStep):
    """One layer over an expert layout with replicas (Cobalt: EP distributes expert
    replicas across GPUs; task assignment routes tokens to fewer remote nodes):
    assign_replicas -> plan over the chosen per-slot ranks -> gather (count beside it on a
    side stream) -> combine.  The n_hot most loaded experts of the batch have a second
    replica on another node (workload.replicate_hot)."""
    n_events = 6
    phases = {"coact_count": (3, 1), "assign_replicas": (0, 2), "plan_dispatch": (2, 3),
              "dispatch_gather": (3, 4), "combine_scatter": (4, 5)}

    layout_kind = "hot"        # "hot": workload.replicate_hot; "planned": coact_place_replicas

    def __init__(self, coact, r: workload.Routing, device, n_hot: int, fill: bool = True):
        super().__init__(coact, r, device, fill)
        c = r.cfg
        if self.layout_kind == "planned":
            # the library's planner over the batch's own counts (library calls)
            to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=device)
            loads = torch.zeros(c.E, dtype=torch.int64, device=device)
            coact.coact_count(to(r.ids), c.E, pair, loads)
            rep, nrep, _ = coact.coact_place_replicas(pair, loads, torch.from_numpy(r.expert_rank),
                                                       torch.from_numpy(r.rank_node), n_hot)
            self.rep_h, self.nrep_h = rep.numpy(), nrep.numpy()
        else:
            loads = np.bincount(r.ids.ravel(), minlength=c.E)    # the batch's expert loads
            self.rep_h, self.nrep_h = workload.replicate_hot(loads, r.expert_rank, r.rank_node,
                                                             n_hot)
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.rep, self.nrep = to(self.rep_h), to(self.nrep_h)
        self.slot = torch.empty((c.N, c.k), dtype=torch.int32, device=device)
        self.n_hot = n_hot
        self.kernels_per_step = 1 + 1 + plan_launches(c.R, self.N) + 1 + 1
        layout = ("coact_place_replicas over the batch's counts" if self.layout_kind == "planned"
                  else "the hottest experts with a second replica on another node")
        self.step_desc = (f"assign_replicas ({n_hot} replicas: {layout}) + plan_dispatch_slots + "
                          "dispatch_gather (coact_count beside it, side stream) + combine_scatter "
                          "(bf16 out)")

    def clone_for_copy(self, coact, device):
        return ReplicaStep(coact, self.L.r, device, self.n_hot, fill=False)

    def step(self, ev=None):
        L, c, cfg = self.L, self.L.coact, self.cfg
        main = torch.cuda.current_stream()
        if ev: ev[0].record()
        c.assign_replicas(L.ids, cfg.E, self.rep, self.nrep, cfg.R, self.slot, rank_node=L.rank_node,
                          n_nodes=cfg.n_nodes, err_flag=L.err)
        if ev: ev[2].record()
        c.plan_dispatch(L.ids, cfg.E, None, cfg.R, L.plan, rank_node=L.rank_node,
                        n_nodes=cfg.n_nodes, err_flag=L.err, slot_rank=self.slot)
        if ev: ev[3].record()
        self.count_beside(main, ev, 1)
        L.gather()
        if ev: ev[4].record()
        L.combine()
        main.wait_stream(self.side)
        if ev: ev[5].record()

    def roofline_parts(self):
        D = self.L.D()
        return [("dispatch_gather", LayerBuffers.gather_kernel(), self.L.bytes_gather(D)),
                ("combine_scatter", "k_combine_v16", self.L.bytes_combine())]

    def summary(self):
        L, c, cfg = self.L, self.L.coact, self.cfg
        out = super().summary()
        st = L.plan.stats.cpu().tolist()
        prim = c.alloc_plan(cfg.N, cfg.k, cfg.E, cfg.R, L.dev)
        c.plan_dispatch(L.ids, cfg.E, self.rep[:, 0].contiguous(), cfg.R, prim,
                        rank_node=L.rank_node, n_nodes=cfg.n_nodes)
        sp = prim.stats.cpu().tolist()
        load = lambda sl: np.bincount(sl.ravel(), minlength=cfg.R)
        lc = load(self.slot.cpu().numpy())
        lp = load(self.rep_h[:, 0][L.r.ids])
        out.update({
            "replicated_experts": int((self.nrep_h > 1).sum()),
            "node_remote_pairs_replica_choice": st[4], "node_remote_pairs_primary_only": sp[4],
            "local_served_asg_replica_choice": st[5], "local_served_asg_primary_only": sp[5],
            "rank_load_max_over_mean_replica_choice": float(lc.max() / lc.mean()),
            "rank_load_max_over_mean_primary_only": float(lp.max() / lp.mean())})
        return out


class BackwardStep:
    """The backward pass of one layer over the forward's plan (computed once, outside the
    timed steps): combine_scatter_backward (grad_y rows for the experts, grad_gates), then
    dispatch_gather_backward (the experts' input gradients, one row per send row, summed
    per token into grad_x).  The experts' own backward sits between the two and is not
    part of this path."""
    n_events = 3
    phases = {"combine_backward": (0, 1), "dispatch_backward": (1, 2)}
    host_inputs = ("g_out", "y", "g_send", "gates")
    step_desc = ("backward: combine_scatter_backward (grad_y bf16, grad_gates fp32) + "
                 "dispatch_gather_backward (grad_x bf16) over the forward's plan")

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        self.coact = coact
        self.L = LayerBuffers(coact, r, device, fill)
        self.cfg, self.N = r.cfg, r.cfg.N
        c = r.cfg
        self.L.plan_()
        self.D = self.L.D()
        if fill:
            self.g_out = workload.fill_bf16(c.N, c.H, r.seed, 6, device=device)
            self.g_send = workload.fill_bf16(self.L.plan.row_capacity, c.H, r.seed, 5,
                                             device=device)
        else:
            self.g_out = torch.empty((c.N, c.H), dtype=torch.bfloat16, device=device)
            self.g_send = torch.empty((self.L.plan.row_capacity, c.H), dtype=torch.bfloat16,
                                      device=device)
        self.g_y = torch.empty((c.N * c.k, c.H), dtype=torch.bfloat16, device=device)
        self.g_gates = torch.empty((c.N, c.k), dtype=torch.float32, device=device)
        self.g_x = torch.empty((c.N, c.H), dtype=torch.bfloat16, device=device)
        self.kernels_per_step = 2

    @property
    def y(self):
        return self.L.y

    @property
    def gates(self):
        return self.L.gates

    def inputs(self):
        return {n: getattr(self, n) for n in self.host_inputs}

    def outputs(self):
        return [self.g_x, self.g_gates]

    def clone_for_copy(self, coact, device):
        return BackwardStep(coact, self.L.r, device, fill=False)

    def step(self, ev=None):
        L, c = self.L, self.coact
        if ev: ev[0].record()
        c.combine_scatter_backward(L.y, L.gates, L.plan.comb_row, self.g_out, self.g_y,
                                   self.g_gates, err_flag=L.err)
        if ev: ev[1].record()
        c.dispatch_gather_backward(self.g_send, L.plan.send_row, self.g_x, err_flag=L.err)
        if ev: ev[2].record()

    def roofline_parts(self):
        c, D = self.cfg, self.D
        return [("combine_backward", "k_combine_bwd",
                 c.N * c.H * 2 + 2 * c.N * c.k * c.H * 2 + c.N * c.k * 12),
                ("dispatch_backward", "k_combine_v16", D * c.H * 2 + c.N * c.H * 2 + c.N * c.k * 4)]

    def summary(self):
        return {"dedup_rows_over_naive": self.D / (self.N * self.cfg.k),
                "err_flag": int(self.L.err.item())}


class ShuffleStep:
    """Config 4's token shuffling fused into the post-attention reduce-scatter: predict
    each token's layer-2 home rank from the calibration counts C12, plan the permutation
    (every token to its home rank alone), and reduce the R ranks' partial attention
    outputs (synthetic, bf16 [N, H] each) into the shuffled rows -- all R emulated ranks'
    segments in one launch on this GPU."""
    n_events = 4
    phases = {"predict_home": (0, 1), "shuffle_plan": (1, 2), "reduce_scatter": (2, 3)}
    step_desc = ("token shuffle: predict_home (layer-1 picks x calibration C12) + shuffle plan "
                 "(plan_dispatch, k = 1) + shuffle_reduce_scatter over R partial attention "
                 "outputs (bf16 out)")
    e2e_skip = "not measured for --shuffle: the R partial outputs are R x N x H x 2 bytes per step"

    def __init__(self, coact, tl: workload.TwoLayer, device):
        self.coact, self.tl = coact, tl
        self.cfg = c = tl.layer1.cfg
        self.N = c.N
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.ids1 = to(tl.layer1.ids)
        self.er2 = to(tl.layer2.expert_rank.astype(np.int32))
        self.C12 = torch.zeros((c.E, c.E), dtype=torch.int64, device=device)
        coact.coact_count(to(tl.calib1), c.E, self.C12, ids2=to(tl.calib2), E2=c.E)
        self.home = torch.empty(c.N, dtype=torch.int32, device=device)
        self.pws = torch.empty(max(coact.predict_workspace_bytes(c.E, c.R), 16), dtype=torch.uint8,
                               device=device)
        self.sp = coact.alloc_plan(c.N, 1, c.R, c.R, device, with_rank_mask=False,
                                   with_src_dst=False)
        self.parts = [workload.fill_bf16(c.N, c.H, tl.layer1.seed, 100 + q, device=device)
                      for q in range(c.R)]
        self.bases = torch.tensor([p.data_ptr() for p in self.parts], dtype=torch.int64,
                                  device=device)
        self.out = torch.empty((c.N, c.H), dtype=torch.bfloat16, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.kernels_per_step = 2 + plan_launches(c.R, c.N) + 1

    def step(self, ev=None):
        c, co = self.cfg, self.coact
        if ev: ev[0].record()
        co.predict_home(self.ids1, c.E, self.C12, self.er2, c.R, self.home, workspace=self.pws,
                        err_flag=self.err)
        if ev: ev[1].record()
        co.shuffle_plan(self.home, c.R, plan=self.sp, err_flag=self.err)
        if ev: ev[2].record()
        co.shuffle_reduce_scatter(self.bases, c.N, self.sp.row_token, self.out, err_flag=self.err)
        if ev: ev[3].record()

    def roofline_parts(self):
        c = self.cfg
        return [("reduce_scatter", "k_shuffle_reduce",
                 c.R * c.N * c.H * 2 + c.N * c.H * 2 + c.N * 4)]

    def summary(self):
        c, co, dev = self.cfg, self.coact, self.home.device
        nk = c.N * c.k
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        ids2, rn = to(self.tl.layer2.ids), to(self.tl.layer2.rank_node.astype(np.int32))
        share = {}
        for name, src in (("predicted_home", self.home), ("contiguous_home", None)):
            p = co.alloc_plan(c.N, c.k, c.E, c.R, dev)
            co.plan_dispatch(ids2, c.E, self.er2, c.R, p, rank_node=rn, n_nodes=c.n_nodes,
                             src_rank=src)
            share[f"local_served_share_{name}"] = int(p.stats[5].item()) / nk
        counts = self.sp.rank_counts.cpu().numpy()
        return {**share, "tokens_per_rank_max_over_mean": float(counts.max() / counts.mean()),
                "err_flag": int(self.err.item())}


def make_step(coact, cfg_index: int, seed: int, device, two_hop: bool = False,
              placement_kind: str = "auto", mode: str = "forward", tokens: Optional[int] = None):
    """The step object for a configuration, plus a description of its placement.  tokens:
    a smaller batch of the same configuration (profiling captures)."""
    cfg = workload.CONFIGS[cfg_index]
    if tokens:
        cfg = cfg.with_(N=int(tokens))
    if mode == "shuffle":
        if not cfg.two_layer:
            raise SystemExit("--shuffle needs the two-layer configuration (4)")
        return ShuffleStep(coact, workload.make_two_layer(cfg, seed=seed, N=cfg.N), device), \
            "contiguous; tokens shuffled to the predicted layer-2 home rank"
    if cfg.two_layer:
        if mode != "forward":
            raise SystemExit("--pass backward / --combine prereduced need a one-layer configuration")
        if two_hop:
            raise SystemExit("--two-hop needs a one-layer configuration with several nodes (2, 3)")
        return TwoLayerStep(coact, workload.make_two_layer(cfg, seed=seed, N=cfg.N), device), \
            "contiguous; layer 2 pre-sharded to the predicted home rank"
    r = workload.make_routing(cfg, seed=seed)
    kind = placement_kind if placement_kind != "auto" else (
        "correlated" if cfg_index == 3 else "default")
    desc = cfg.placement
    rr_D = None
    if kind != "default":
        # dedup ratio under the configuration's own placement, for comparison
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        base = coact.alloc_plan(cfg.N, cfg.k, cfg.E, cfg.R, device)
        coact.plan_dispatch(to(r.ids), cfg.E, to(r.expert_rank.astype(np.int32)), cfg.R, base,
                            rank_node=to(r.rank_node), n_nodes=cfg.n_nodes)
        rr_D = int(base.rank_offsets[-1].item()) / (cfg.N * cfg.k)
        del base
        r.expert_rank, desc = layout(coact, r, kind, device)
    if two_hop:
        if cfg.n_nodes < 2:
            raise SystemExit("--two-hop needs a one-layer configuration with several nodes (2, 3)")
        if mode != "forward":
            raise SystemExit("--two-hop runs the forward pass with the direct combine only")
        S = TwoHopStep(coact, r, device)
    elif mode.startswith("replicas:"):
        S = ReplicaStep(coact, r, device, int(mode.split(":")[1]))
    elif mode == "backward":
        S = BackwardStep(coact, r, device)
    elif mode == "prereduced":
        S = PreReducedStep(coact, r, device)
    elif mode == "rebalance":
        S = RebalanceStep(coact, r, device)
    else:
        S = OneLayerStep(coact, r, device)
    if rr_D is not None:
        S.rr_dedup = rr_D
    return S, desc


# CUDA sources of each HBM-bound kernel: a committed DRAM-traffic figure is reported only
# while these files are byte-identical to the ones the ncu capture was taken on.
KERNEL_SOURCES = {"k_gather_v16": ("gather.cu", "common.cuh"),
                  "k_shuffle_reduce": ("shuffle.cu", "common.cuh"),
                  "k_gather_bulk": ("gather.cu", "common.cuh"),
                  "k_combine_units": ("combine.cu", "common.cuh"),
                  "k_combine_bwd": ("backward.cu", "common.cuh"),
                  "k_combine_v16": ("combine.cu", "common.cuh"),
                  "k_forward_gather": ("twohop.cu", "common.cuh"),
                  "k_forward_tokens": ("twohop.cu", "common.cuh")}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for fn in KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(ROOT, "co_activation_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's sources match."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    sha = kernel_source_hash(kernel)
    for line in open(path):
        p = line.split()
        if len(p) >= 4 and not line.startswith("#") and p[0] == kernel and p[1] == workload_name:
            return int(float(p[2])) if p[3] == sha else None
    return None


# ----------------------------------------------------------------------------- GPU run


def run_gpu(args):
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    import co_activation_b200 as coact

    cfg = workload.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_(N=int(args.tokens))
    LayerBuffers.tma = args.gather == "tma"
    TwoHopStep.forward = args.forward
    ReplicaStep.layout_kind = args.replica_layout
    mode = "shuffle" if args.shuffle else f"replicas:{args.replicas}" if args.replicas else \
        "backward" if args.pass_ == "backward" else "rebalance" if args.rebalance else (
        "prereduced" if args.combine == "prereduced" else "forward")
    S, placement = make_step(coact, args.config, rank_seed(args.seed, rank), device, args.two_hop,
                             args.placement, mode, args.tokens)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 64 << 20), dtype=torch.uint8, device=device)
    flush_r = torch.zeros(max(2 * l2, 64 << 20) // 8, dtype=torch.int64, device=device)
    flush_sink = torch.empty((), dtype=torch.int64, device=device)

    def flush():
        """L2 flush between steps: write a buffer twice the L2 size, then read another
        one as large, so the step starts with a cold AND clean L2 (the dirty lines of the
        write are written back here, not inside the next timed kernel)."""
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    # warm-up (also does every lazy one-time attribute setup before graph capture)
    for _ in range(args.warmup):
        flush()
        S.step()
    torch.cuda.synchronize()
    summ = S.summary()
    assert summ["err_flag"] == 0, f"device error flags {summ['err_flag']}"

    K, NE = args.steps, S.n_events

    def capture(with_phases: bool):
        """K steps (each preceded by the L2 flush) as one CUDA graph.  Events at the step
        boundaries always; at the phase boundaries only in the breakdown pass, because
        every event node inside a graph serialises the stream (about 3 us each)."""
        ev = [[torch.cuda.Event(enable_timing=True, external=args.graph) for _ in range(NE)]
              for _ in range(K)]

        def body():
            for i in range(K):
                flush()
                if with_phases:
                    S.step(ev[i])
                else:
                    ev[i][0].record()
                    S.step()
                    ev[i][NE - 1].record()

        if not args.graph:
            return None, ev, body
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):          # captured on torch's side stream
            body()
        torch.cuda.synchronize()
        g.replay()                         # upload; these events are overwritten later
        torch.cuda.synchronize()
        return g, ev, body

    timing = ("one CUDA graph of K steps per pass; CUDA events per step (per-step times of "
              "~70 us fall on levels ~2.1 us apart on B200: value and step_us_mean are means)")
    try:
        g_main, evs, body_main = capture(False)
        g_phase, evs_phase, body_phase = capture(True)
    except RuntimeError as e:              # capture refused: time eager launches instead
        torch.cuda.synchronize()
        args.graph = False
        g_main, evs, body_main = capture(False)
        g_phase, evs_phase, body_phase = capture(True)
        timing = f"eager launches (graph capture failed: {str(e)[:80]})"
    if not args.graph and "failed" not in timing:
        timing = "eager launches; CUDA events per step"
    run = lambda g, body: g.replay() if g is not None else body()

    clocks = ClockSampler(local)
    clocks.start()
    # keep the GPU busy for a moment so the sampler sees the clocks under this load
    t_end = time.time() + args.clock_warm_s
    while time.time() < t_end:
        run(g_main, body_main)
        torch.cuda.synchronize()
    # timed region: K steps, events per step (headline)
    barrier(world)
    torch.cuda.synchronize()
    run(g_main, body_main)
    torch.cuda.synchronize()
    barrier(world)
    # breakdown passes: the same K steps with events at every phase boundary (per-kernel
    # durations for the breakdown and the roofline; slightly inflated by the event nodes
    # themselves, so the roofline fraction is a lower bound).  Replayed twice; each
    # phase keeps the lower of its two K-step means, so one disturbed replay does not
    # understate a kernel.
    phase_runs = []
    for _ in range(2):
        run(g_phase, body_phase)
        torch.cuda.synchronize()
        phase_runs.append({name: statistics.mean(evs_phase[i][a].elapsed_time(evs_phase[i][b])
                                                 for i in range(K))
                           for name, (a, b) in S.phases.items()})
        phase_runs[-1]["__step__"] = statistics.mean(
            evs_phase[i][0].elapsed_time(evs_phase[i][NE - 1]) for i in range(K))
    barrier(world)
    clk = clocks.stop()

    step_ms = [evs[i][0].elapsed_time(evs[i][NE - 1]) for i in range(K)]
    phase_ms = {name: min(pr[name] for pr in phase_runs) for name in S.phases}
    phase_pass_step_ms = min(pr["__step__"] for pr in phase_runs)
    agg = aggregate(cfg.N * K, sum(step_ms) / 1e3, world, device)
    total_s, value = agg["seconds"], agg["tokens_per_s"]
    peak, peak_kind = peaks()
    parts = [(ph, kern, byt, phase_ms[ph]) for ph, kern, byt in S.roofline_parts()]
    dc_ms = sum(p[3] for p in parts)
    dc_bytes = sum(p[2] for p in parts)
    gb_dc = dc_bytes / (dc_ms / 1e3) / 1e9
    dom = max(parts, key=lambda p: p[3])
    dom_gbs = dom[2] / (dom[3] / 1e3) / 1e9
    e2e = {"value": None, "note": S.e2e_skip} if hasattr(S, "e2e_skip") else \
        {"value": None, "note": "skipped (--no-e2e)"} if args.no_e2e else \
        run_e2e(coact, S, args, world, device)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_s * 1e3 / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded routing shaped after the pages' statistics; no router traces)",
        "config": {"workload": f"config {cfg.index}: {cfg.desc}" + (
                       f" -- reduced to N={cfg.N} for a profiling capture" if args.tokens else ""),
                   "N": cfg.N, "E": cfg.E,
                   "k": cfg.k, "H": cfg.H, "R": cfg.R, "n_nodes": cfg.n_nodes,
                   "placement": placement,
                   "pass": mode,
                   "gather": ("dispatch_gather_tma (TMA bulk copies)" if LayerBuffers.tma
                              else "dispatch_gather (vector copies, 32-byte where aligned, one "
                                   "warp per token)"),
                   "step": getattr(S, "step_desc", None) or ("two layers: counts + cross-layer counts + predict_home (side stream, "
                            "beside layer 1); plan, gather, combine of layer 1; plan, gather, "
                            "combine of layer 2"
                            if cfg.two_layer else
                            "two-hop plan (node and rank plans, forward map) + hop-1 gather "
                            f"(coact_count beside it, side stream) + hop-2 forward ({args.forward}) + "
                            "combine_scatter"
                            if args.two_hop else
                            "plan_dispatch + dispatch_gather (coact_count beside it, side "
                            "stream) + combine_scatter (bf16 out)"),
                   "l2": "flushed between timed steps (write of 2x L2, then a read of another 2x L2 "
                         "buffer so no dirty line is left), outside the step events",
                   "timing": timing,
                   "parallelism": f"{world} GPU(s), one independent batch per GPU"},
        "dispatch_combine_tokens_per_s": cfg.N / (dc_ms / 1e3),
        **{k_: v for k_, v in summ.items() if k_ != "err_flag"},
        "phase_us": {k_: v * 1e3 for k_, v in phase_ms.items()},
        "step_us_mean": statistics.mean(step_ms) * 1e3,
        "step_us_median": statistics.median(step_ms) * 1e3,
        "step_us_min": min(step_ms) * 1e3,
        "phase_pass_step_us": phase_pass_step_ms * 1e3,
        "hbm_gbs": {**{p[0]: p[2] / (p[3] / 1e3) / 1e9 for p in parts},
                    "gather+combine": gb_dc,
                    "pct_of_8tbs_gather+combine": 100 * gb_dc / 8000.0,
                    f"pct_of_{peak_kind}_{peak:.0f}": 100 * gb_dc / peak},
        "roofline": {"kernel": dom[1], "phase": dom[0], "bound": "hbm", "achieved": dom_gbs,
                     "peak": peak, "unit": "GB/s", "frac": dom_gbs / peak,
                     "peak_kind": f"of {peak_kind}", "algorithmic_bytes": dom[2],
                     "traffic": read_traffic(dom[1], f"config{cfg.index}")},
        "clocks": clk,
        "gpu_launches": K * S.kernels_per_step,
        "e2e": e2e,
    }
    if hasattr(S, "rr_dedup"):
        result["dedup_rows_over_naive_config_placement"] = S.rr_dedup
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(S, args.cpu_seconds, args.cpu_tokens)
    if world > 1:
        import torch.distributed as dist
        del g_main, g_phase
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_e2e(coact, S, args, world, device):
    """The step through the public API from pinned host buffers: every step copies its
    inputs host -> device, runs the library calls and copies its outputs (combined rows
    and statistics) device -> host.  Two device buffer sets let step i+1's input copy
    overlap step i's compute and output copy (copy engines in both directions run
    concurrently with the SMs)."""
    cfg = S.cfg

    kind = {"host": "pinned"}

    def pinned(t, fill: bool):
        try:
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        except RuntimeError:            # the host cannot pin this much: pageable buffers
            kind["host"] = "pageable (pinning failed)"
            h = torch.empty(t.shape, dtype=t.dtype)
        if fill:
            h.copy_(t)
        return h

    host = {n: pinned(t, True) for n, t in S.inputs().items()}
    bufs = [S, S.clone_for_copy(coact, device)]
    outs_h = [[pinned(t, False) for t in S.outputs()] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0])
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def run(n_steps):
        free = [None, None]
        for i in range(n_steps):
            b, slot = bufs[i % 2], i % 2
            dst = b.inputs()
            with torch.cuda.stream(s_in):
                if i == 0:
                    s_in.wait_stream(comp)
                if free[slot] is not None:
                    s_in.wait_event(free[slot])
                for n, t in host.items():
                    dst[n].copy_(t, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            comp.wait_event(ready)
            b.step()
            done = torch.cuda.Event()
            done.record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                for h, d in zip(outs_h[slot], b.outputs()):
                    h.copy_(d, non_blocking=True)
                fr = torch.cuda.Event()
                fr.record(s_out)
            free[slot] = fr
        for e in free:
            if e is not None:
                comp.wait_event(e)

    run(max(2, args.warmup))
    torch.cuda.synchronize()
    K = args.steps
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(comp)
    run(K)
    b_.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    agg = aggregate(cfg.N * K, a.elapsed_time(b_) / 1e3, world, device)
    return {"value": agg["tokens_per_s"], "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "note": f"{kind['host']} host buffers; input copy of step i+1 overlaps compute and "
                    "output copy of step i (two device buffer sets)"}


# ----------------------------------------------------------------------------- the oracle


def _oracle_layer(o, ids, gates, er, rn, n_nodes, E, R, xb, yb, src=None):
    o.count(ids, E)
    p = o.plan(ids, E, er, R, rank_node=rn, n_nodes=n_nodes, src_rank=src)
    o.gather(xb, p["row_token"], p["D"])
    return o.combine_f64(yb, gates, p["comb_row"])


def _oracle_step_fn(S, max_tokens: Optional[int] = None):
    """A closure running the oracle over the same workload as step S (host arrays); its
    `tokens` attribute is the number of tokens one call processes."""
    import oracle as o
    cfg = S.cfg
    if isinstance(S, TwoLayerStep):
        tl = S.tl
        x1, y1, y2 = o._bits(S.L1.x), o._bits(S.L1.y), o._bits(S.L2.y)
        C12 = S.C12.cpu().numpy()

        def fn():
            out1 = _oracle_layer(o, tl.layer1.ids, tl.layer1.gates, tl.layer1.expert_rank,
                                 tl.layer1.rank_node, cfg.n_nodes, cfg.E, cfg.R, x1, y1)
            o.count_cross(tl.layer1.ids, cfg.E, tl.layer2.ids, cfg.E)
            home, _ = o.predict_home(tl.layer1.ids, cfg.E, C12, tl.layer2.expert_rank, cfg.R)
            x2 = o.bf16_rne(out1.astype(np.float32))
            _oracle_layer(o, tl.layer2.ids, tl.layer2.gates, tl.layer2.expert_rank,
                          tl.layer2.rank_node, cfg.n_nodes, cfg.E, cfg.R, x2, y2, src=home)
        fn.tokens = S.N
        return fn
    if isinstance(S, ShuffleStep):
        # a bounded sample: the first 4096 tokens' predicted homes and partial rows
        tl, n = S.tl, min(S.N, 4096)
        C12 = S.C12.cpu().numpy()
        toks = np.arange(n)
        parts = np.stack([o._bits(workload.fill_bf16(n, cfg.H, tl.layer1.seed, 100 + q,
                                                    row_ids=toks)) for q in range(cfg.R)])

        def fn():
            home, _ = o.predict_home(tl.layer1.ids[:n], cfg.E, C12, tl.layer2.expert_rank, cfg.R)
            order = o.shuffle_order(home, cfg.R)
            o.shuffle_reduce_f32chain(parts, order["row_token"][:n])
        fn.tokens = n
        return fn
    L = S.L
    if isinstance(S, BackwardStep):
        yb, gob, gsb = o._bits(L.y), o._bits(S.g_out), o._bits(S.g_send)
        p = o.plan(L.r.ids, cfg.E, L.r.expert_rank, cfg.R, rank_node=L.r.rank_node,
                   n_nodes=cfg.n_nodes)

        def fn():
            o.combine_backward(yb, L.r.gates, p["comb_row"], gob)
            o.gather_backward_f32chain(gsb, p["send_row"])
        fn.tokens = S.N
        return fn
    # a bounded sample: the batch's first n tokens (their routing, x rows and as many
    # expert-output rows as n tokens have), the whole path over them
    n = S.N if not max_tokens else min(S.N, int(max_tokens))
    ids, gates = L.r.ids[:n], L.r.gates[:n]
    xb, yb = o._bits(L.x[:n]), o._bits(L.y[:n * cfg.k])
    if isinstance(S, TwoHopStep):
        def fn():
            o.count(ids, cfg.E)
            node, rank, fwd = o.plan_two_hop(ids, cfg.E, L.r.expert_rank, cfg.R,
                                             L.r.rank_node, cfg.n_nodes)
            hop1 = o.gather(xb, node["row_token"], node["D"])
            o.forward_gather(hop1, fwd)
            o.combine_f64(yb, gates, rank["comb_row"])
    elif isinstance(S, ReplicaStep):
        def fn():
            o.count(ids, cfg.E)
            slot, _ = o.assign_replicas(ids, cfg.E, S.rep_h, S.nrep_h, cfg.R,
                                        rank_node=L.r.rank_node, n_nodes=cfg.n_nodes)
            p = o.plan(ids, cfg.E, None, cfg.R, rank_node=L.r.rank_node, n_nodes=cfg.n_nodes,
                       slot_rank=slot)
            o.gather(xb, p["row_token"], p["D"])
            o.combine_f64(yb, gates, p["comb_row"])
    elif isinstance(S, RebalanceStep):
        en = S.expert_node.cpu().numpy()

        def fn():
            _, loads, _ = o.count(ids, cfg.E)
            er = o.rebalance_ranks(loads, en, L.r.rank_node)
            p = o.plan(ids, cfg.E, er, cfg.R, rank_node=L.r.rank_node, n_nodes=cfg.n_nodes)
            o.gather(xb, p["row_token"], p["D"])
            o.combine_f64(yb, gates, p["comb_row"])
    elif isinstance(S, PreReducedStep):
        def fn():
            o.count(ids, cfg.E)
            p = o.plan(ids, cfg.E, L.r.expert_rank, cfg.R, rank_node=L.r.rank_node,
                       n_nodes=cfg.n_nodes)
            o.gather(xb, p["row_token"], p["D"])
            o.combine_prereduced(yb, gates, p)
    else:
        def fn():
            _oracle_layer(o, ids, gates, L.r.expert_rank, L.r.rank_node, cfg.n_nodes, cfg.E,
                          cfg.R, xb, yb)
    fn.tokens = n
    return fn


def cpu_baseline(S, seconds: float, max_tokens: Optional[int] = None):
    """The oracle, as it stands, on this host: passes over the same workload (whole
    batches, or the batch's first max_tokens tokens when N is larger) repeated for about
    `seconds` (at least one pass)."""
    fn = _oracle_step_fn(S, max_tokens)
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    what = ("home prediction, shuffle order and the rank-order sum of the partial rows"
            if isinstance(S, ShuffleStep) else
            "both layers' count, plan, gather and float64 combine, cross-layer counts and the "
            "home prediction" if isinstance(S, TwoLayerStep) else
            "combine backward (float64 gate gradients) and transposed dispatch"
            if isinstance(S, BackwardStep) else
            "count, node and rank plans, hop-1 gather, hop-2 forward, float64 combine"
            if isinstance(S, TwoHopStep) else
            "count, replica choice, plan, gather, float64 combine"
            if isinstance(S, ReplicaStep) else
            "count, plan, gather, partial rows and their sum"
            if isinstance(S, PreReducedStep) else
            "count, intra-node rebalance, plan, gather, float64 combine"
            if isinstance(S, RebalanceStep) else
            "count, plan, gather, float64 combine")
    if fn.tokens < S.N:
        sample = (f"{n} pass(es) over the first {fn.tokens} of the {S.N} tokens of config "
                  f"{S.cfg.index} (same placement, rows of H={S.cfg.H}) through the "
                  f"single-threaded C oracle: {what}")
    else:
        sample = (f"{n} whole batch(es) of config {S.cfg.index} (N={S.N}) through the "
                  f"single-threaded C oracle: {what}")
    return {"value": fn.tokens * n / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": sample, "host_cpu": _cpu_model(), "host_nproc": os.cpu_count()}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle as o
    cfg = workload.CONFIGS[args.config]
    r = workload.make_routing(cfg, seed=args.seed)
    if args.config == 3 and args.placement in ("auto", "correlated"):
        # the timed arm's placement: correlated, from the whole batch's pair counts (built
        # once per batch, outside the timed steps in both arms)
        r.expert_rank = o.place_correlated(o.count(r.ids, cfg.E)[0], cfg.R)
    # each step: a bounded sample of the workload (the first n tokens' routing, whole
    # count/plan/gather/combine over them) sized so K + W steps end within a few minutes
    step_tokens = min(cfg.N, max(256, int(args.ref_tokens)))
    ids, gates = r.ids[:step_tokens], r.gates[:step_tokens]
    xs = o._bits(workload.fill_bf16(step_tokens, cfg.H, r.seed, X_STREAM))
    ys = o._bits(workload.fill_bf16(step_tokens * cfg.k, cfg.H, r.seed, Y_STREAM))
    for _ in range(args.warmup):
        _oracle_layer(o, ids, gates, r.expert_rank, r.rank_node, cfg.n_nodes, cfg.E, cfg.R, xs, ys)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_layer(o, ids, gates, r.expert_rank, r.rank_node, cfg.n_nodes, cfg.E, cfg.R, xs, ys)
    dt = time.perf_counter() - t0
    value = step_tokens * args.steps / dt
    sample = (f"first {step_tokens} of the {cfg.N} tokens of config {cfg.index} per step (count, "
              "plan, gather, float64 combine of one layer), single-threaded C oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"config {cfg.index}: {cfg.desc}",
                                        "tokens_per_step": step_tokens},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def run_hbm_mix(args):
    """What this GPU's HBM delivers per read/write mix, the context of the roofline
    fractions: the gather over synthetic contiguous destinations at fan-out f (f rows
    written per row read, f/(1+f) of the bytes written) and the combine over synthetic
    expert rows at k rows per output row (k/(1+k) read), in contiguous and in seeded random
    row order, beside torch's copy_ and full-tensor sum.  H = 7,168 (config 3's rows),
    ~MIX_GB per launch, L2 flushed between launches, CUDA events; one GPU, one JSON line."""
    import co_activation_b200 as coact
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    reps = max(5, min(args.steps, 20))
    total = args.mix_gb * 1e9
    H = 7168

    def timed(fn):
        for _ in range(args.warmup):
            flush_buf.zero_()
            fn()
        ts = []
        for _ in range(reps):
            flush_buf.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        return statistics.mean(ts)

    res = {}
    clk = ClockSampler(0)
    clk.start()
    n = int(total // 4)
    a = torch.empty(n, dtype=torch.bfloat16, device=dev).normal_()
    b = torch.empty_like(a)
    res["torch_copy"] = {"write_share": 0.5, "GBps": 4 * n / timed(lambda: b.copy_(a)) / 1e9}
    del b
    s = torch.empty((), dtype=torch.int64, device=dev)
    res["torch_sum"] = {"write_share": 0.0,
                        "GBps": 2 * n / timed(lambda: torch.sum(a.view(torch.int64), dim=0,
                                                                out=s)) / 1e9}
    del a
    torch.cuda.empty_cache()
    gen = torch.Generator(device=dev)
    for f in (1, 2, 4, 8):
        N = int(total / ((1 + f) * H * 2))
        x = torch.empty((N, H), dtype=torch.bfloat16, device=dev).normal_()
        send_row = (torch.arange(f, dtype=torch.int32, device=dev)[None, :] * N
                    + torch.arange(N, dtype=torch.int32, device=dev)[:, None]).contiguous()
        send = torch.empty((N * f, H), dtype=torch.bfloat16, device=dev)
        byt = (N + N * f) * H * 2 + N * f * 4
        res[f"gather_fanout{f}"] = {"write_share": round(N * f * H * 2 / byt, 4),
                                    "GBps": byt / timed(lambda: coact.dispatch_gather(
                                        x, send_row, send)) / 1e9}
        del x, send_row, send
        torch.cuda.empty_cache()
    for k in (1, 2, 4, 8):
        N = int(total / ((k + 1) * H * 2))
        y = torch.empty((N * k, H), dtype=torch.bfloat16, device=dev).normal_()
        g = torch.rand((N, k), dtype=torch.float32, device=dev)
        out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
        byt = N * k * H * 2 + N * H * 2 + N * k * 8
        share = round(N * H * 2 / byt, 4)
        rows = torch.arange(N * k, dtype=torch.int32, device=dev).view(N, k).contiguous()
        res[f"combine_k{k}"] = {"write_share": share,
                                "GBps": byt / timed(lambda: coact.combine_scatter(
                                    y, g, rows, out)) / 1e9}
        gen.manual_seed(args.seed + k)
        rows = torch.randperm(N * k, device=dev, generator=gen).to(torch.int32).view(N, k)
        res[f"combine_k{k}_random_rows"] = {"write_share": share,
                                            "GBps": byt / timed(lambda: coact.combine_scatter(
                                                y, g, rows, out)) / 1e9}
        del y, g, out, rows
        torch.cuda.empty_cache()
    clocks = clk.stop()
    peak, kind = peaks()
    for v in res.values():
        v["GBps"] = round(v["GBps"], 1)
        v["frac_of_copy_peak"] = round(v["GBps"] / peak, 4)
    print(json.dumps({"hbm_mix": res, "unit": "GB/s", "H": H, "bytes_per_launch": total,
                      "reps": reps, "warmup": args.warmup, "copy_peak": peak,
                      "copy_peak_kind": kind, "clocks": clocks}))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=3, choices=sorted(workload.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="coact", choices=["coact", "reference"])
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end pass (profiling captures of the kernels)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-tokens", type=int, default=16384,
                    help="cpu_baseline sample: the first CPU_TOKENS tokens of the batch (whole "
                         "batches when N is smaller)")
    ap.add_argument("--clock-warm-s", type=float, default=1.0)
    ap.add_argument("--ref-tokens", type=int, default=4096)
    ap.add_argument("--placement", default="auto", choices=["auto", "default", "correlated",
                                                             "two-stage"],
                    help="auto: the configuration's own (config 3: correlated)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="a smaller batch of the configuration (profiling captures); the "
                         "JSON line's config shows the N used")
    ap.add_argument("--gather", default="vector", choices=["vector", "tma"],
                    help="gather implementation: dispatch_gather or dispatch_gather_tma")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "backward"],
                    help="backward: combine_scatter_backward + dispatch_gather_backward")
    ap.add_argument("--combine", default="direct", choices=["direct", "prereduced"],
                    help="prereduced: combine_rows per send row, then the transposed dispatch")
    ap.add_argument("--replicas", type=int, default=0, metavar="N_HOT",
                    help="give the N_HOT most loaded experts a second replica on another node "
                         "and choose replicas per token (assign_replicas)")
    ap.add_argument("--replica-layout", default="hot", choices=["hot", "planned"],
                    help="which experts get the replicas: the most loaded (fixture) or "
                         "coact_place_replicas over the batch's counts")
    ap.add_argument("--shuffle", action="store_true",
                    help="config 4: token shuffling fused into the post-attention reduce-scatter")
    ap.add_argument("--forward", default="tokens", choices=["tokens", "rows"],
                    help="two-hop forward: token order, each hop-1 row read once "
                         "(forward_gather_tokens), or one read per rank row (forward_gather)")
    ap.add_argument("--rebalance", action="store_true",
                    help="Cobalt's per-step intra-node rebalance on the device inside the step "
                         "(node co-location from the batch's counts, outside the step)")
    ap.add_argument("--two-hop", action="store_true",
                    help="dispatch in two hops: to nodes, then inside the node to ranks")
    ap.add_argument("--hbm-mix", action="store_true",
                    help="instead of the step: what the HBM delivers per read/write mix (the "
                         "gather at fan-out 1-8, the combine at k = 1-8, torch copy and sum)")
    ap.add_argument("--mix-gb", type=float, default=16.0,
                    help="--hbm-mix: bytes moved per launch, in GB")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.hbm_mix:
        run_hbm_mix(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
