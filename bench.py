"""Benchmark of the co-activation dispatch/combine hot path on B200.

One step = one pass of the whole path over one batch of N tokens:
  coact_count (pair counts + loads) -> plan_dispatch (3 kernels) -> dispatch_gather
  -> combine_scatter (bf16 out)
with inputs already resident in HBM.  Default workload: config 1 (N=16384, E=64,
top-2, H=2048 bf16, 8 logical ranks of 8 experts, 16 planted pairs co-selected by 42%
of tokens, random placement), seeded synthetic routing.

Timing: W untimed warm-up steps, then EXACTLY K steps captured in one CUDA graph, each
step bracketed by CUDA events on the launching stream, with an L2 flush (a write of a
buffer twice the L2 size) between steps outside the events.  A barrier and
torch.cuda.synchronize() bracket the timed region; multi-GPU runs (torchrun, one rank
per GPU, each rank its own batch: weak scaling, no data-path collective) report the
max over ranks.  `e2e` times the same step through the public API from pinned host
buffers (H2D of the step's inputs and D2H of its outputs inside the timed region).
`--impl reference` times the CPU oracle instead (rank 0 only).

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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload  # noqa: E402

METRIC = "dispatch+combine tokens/s and HBM GB/s (% of ~8 TB/s); dedup rows/naive rows"
UNIT = "tokens/s"
X_STREAM, Y_STREAM = 1, 2
KERNELS_PER_STEP = {"coact_count": 1, "plan_dispatch": 3, "dispatch_gather": 1,
                    "combine_scatter": 1}


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


# ----------------------------------------------------------------------------- the GPU path


class GpuStep:
    """Device buffers and the four library calls of one step."""

    def __init__(self, coact, r: workload.Routing, device, fill: bool = True):
        cfg = r.cfg
        self.coact, self.r, self.cfg, self.dev = coact, r, cfg, device
        N, k, E, R, H = cfg.N, cfg.k, cfg.E, cfg.R, cfg.H
        to = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.ids = to(r.ids)
        self.gates = to(r.gates)
        self.expert_rank = to(r.expert_rank.astype(np.int32))
        self.rank_node = to(r.rank_node.astype(np.int32))
        if fill:
            self.x = workload.fill_bf16(N, H, r.seed, X_STREAM, device=device)
            self.y = workload.fill_bf16(N * k, H, r.seed, Y_STREAM, device=device)
        else:   # contents arrive by copy (end-to-end measurement)
            self.x = torch.empty((N, H), dtype=torch.bfloat16, device=device)
            self.y = torch.empty((N * k, H), dtype=torch.bfloat16, device=device)
        self.pair = torch.zeros((E, E), dtype=torch.int64, device=device)
        self.loads = torch.zeros(E, dtype=torch.int64, device=device)
        self.plan = coact.alloc_plan(N, k, E, R, device)
        self.send = torch.empty((self.plan.row_capacity, H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.side = torch.cuda.Stream(device=device)

    def count(self):
        self.coact.coact_count(self.ids, self.cfg.E, self.pair, self.loads, err_flag=self.err)

    def plan_(self):
        self.coact.plan_dispatch(self.ids, self.cfg.E, self.expert_rank, self.cfg.R, self.plan,
                                 rank_node=self.rank_node, n_nodes=self.cfg.n_nodes,
                                 err_flag=self.err)

    def gather(self):
        self.coact.dispatch_gather(self.x, self.plan.send_row, self.send, err_flag=self.err)

    def combine(self):
        self.coact.combine_scatter(self.y, self.gates, self.plan.comb_row, self.out,
                                   err_flag=self.err)

    def step(self, ev=None):
        """One pass of the path.  coact_count depends on nothing the other three calls
        produce, so it runs on a side stream, overlapped with plan_dispatch; the step
        ends when both streams have finished.  ev: optional list of 5 events for the
        phase boundaries (the count phase is then measured on the side stream)."""
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        if ev: ev[0].record()
        with torch.cuda.stream(self.side):
            self.count()
            if ev: ev[1].record()
        self.plan_()
        if ev: ev[2].record()
        self.gather()
        if ev: ev[3].record()
        self.combine()
        main.wait_stream(self.side)
        if ev: ev[4].record()

    def bytes_gather(self, D):
        c = self.cfg
        return (c.N + D) * c.H * 2 + c.N * c.k * 4

    def bytes_combine(self):
        c = self.cfg
        return c.N * c.k * c.H * 2 + c.N * c.H * 2 + c.N * c.k * 8


def read_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if its source hash matches."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for fn in sorted(os.listdir(os.path.join(ROOT, "co_activation_b200", "csrc"))):
        with open(os.path.join(ROOT, "co_activation_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    sha = h.hexdigest()[:16]
    for line in open(path):
        p = line.split()
        if len(p) >= 4 and not line.startswith("#") and p[0] == kernel and p[1] == workload_name:
            return int(float(p[2])) if p[3] == sha else None
    return None


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
    r = workload.make_routing(cfg, seed=rank_seed(args.seed, rank))
    S = GpuStep(coact, r, device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 64 << 20), dtype=torch.uint8, device=device)
    flush_r = torch.zeros(max(2 * l2, 64 << 20) // 8, dtype=torch.int64, device=device)
    flush_sink = torch.empty((), dtype=torch.int64, device=device)

    class _Flush:
        """L2 flush between steps: write a buffer twice the L2 size, then read another
        one as large, so the step starts with a cold AND clean L2 (the dirty lines of the
        write are written back here, not inside the next timed kernel)."""

        @staticmethod
        def zero_():
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=flush_sink)

    flush = _Flush()

    # warm-up (also does every lazy one-time attribute setup before graph capture)
    for _ in range(args.warmup):
        flush.zero_()
        S.step()
    torch.cuda.synchronize()
    D = int(S.plan.rank_offsets[-1].item())
    stats = S.plan.stats.cpu().tolist()
    assert S.err.item() == 0, f"device error flags {S.err.item()}"

    K = args.steps

    def capture(with_phases: bool):
        """K steps (each preceded by the L2 flush) as one CUDA graph.  Events at the step
        boundaries always; at the phase boundaries only in the breakdown pass, because
        every event node inside a graph serialises the stream (about 3 us each)."""
        ev = [[torch.cuda.Event(enable_timing=True, external=args.graph) for _ in range(5)]
              for _ in range(K)]

        def body():
            for i in range(K):
                flush.zero_()
                if with_phases:
                    S.step(ev[i])
                else:
                    ev[i][0].record()
                    S.step()
                    ev[i][4].record()

        if not args.graph:
            return None, ev, body
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):          # captured on torch's side stream
            body()
        torch.cuda.synchronize()
        g.replay()                         # upload; these events are overwritten later
        torch.cuda.synchronize()
        return g, ev, body

    timing = "one CUDA graph of K steps per pass; CUDA events per step"
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
    # second timed pass: the same K steps with events at every phase boundary
    # (per-kernel durations for the breakdown and the roofline; slightly inflated by
    # the event nodes themselves, so the roofline fraction is a lower bound)
    run(g_phase, body_phase)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()

    step_ms = [evs[i][0].elapsed_time(evs[i][4]) for i in range(K)]
    # count runs on the side stream (ev0 -> ev1); the main stream runs plan (ev0 -> ev2),
    # gather (ev2 -> ev3) and combine (ev3 -> ev4)
    spans = {"coact_count": (0, 1), "plan_dispatch": (0, 2), "dispatch_gather": (2, 3),
             "combine_scatter": (3, 4)}
    phase_ms = {name: [evs_phase[i][a].elapsed_time(evs_phase[i][b]) for i in range(K)]
                for name, (a, b) in spans.items()}
    agg = aggregate(cfg.N * K, sum(step_ms) / 1e3, world, device)
    total_s, value = agg["seconds"], agg["tokens_per_s"]
    gather_ms = statistics.mean(phase_ms["dispatch_gather"])
    combine_ms = statistics.mean(phase_ms["combine_scatter"])
    dc_tokens_s = cfg.N / ((gather_ms + combine_ms) / 1e3)
    peak, peak_kind = peaks()
    gb_g = S.bytes_gather(D) / (gather_ms / 1e3) / 1e9
    gb_c = S.bytes_combine() / (combine_ms / 1e3) / 1e9
    gb_dc = (S.bytes_gather(D) + S.bytes_combine()) / ((gather_ms + combine_ms) / 1e3) / 1e9
    dom = "combine_scatter" if combine_ms >= gather_ms else "dispatch_gather"
    dom_bytes = S.bytes_combine() if dom == "combine_scatter" else S.bytes_gather(D)
    dom_ms = combine_ms if dom == "combine_scatter" else gather_ms
    kernel_name = "k_combine_v16" if dom == "combine_scatter" else "k_gather_v16"
    wl_name = f"config{cfg.index}"
    traffic = read_traffic(kernel_name, wl_name)

    e2e = run_e2e(coact, S, args, world, device)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_s * 1e3 / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded routing shaped after the pages' statistics; no router traces)",
        "config": {"workload": f"config {cfg.index}: {cfg.desc}", "N": cfg.N, "E": cfg.E,
                   "k": cfg.k, "H": cfg.H, "R": cfg.R, "n_nodes": cfg.n_nodes,
                   "placement": cfg.placement, "step": "coact_count (side stream, overlapped "
                   "with plan) + plan_dispatch + dispatch_gather + combine_scatter (bf16 out)",
                   "l2": "flushed between timed steps (write of 2x L2, then a read of another 2x L2 "
                         "buffer so no dirty line is left), outside the step events",
                   "timing": timing,
                   "parallelism": f"{world} GPU(s), one independent batch per GPU"},
        "dispatch_combine_tokens_per_s": dc_tokens_s,
        "dedup_rows_over_naive": D / (cfg.N * cfg.k),
        "stats": dict(zip(coact.STAT_NAMES, stats)),
        "phase_us": {k_: statistics.mean(v) * 1e3 for k_, v in phase_ms.items()},
        "phase_pass_step_us": statistics.mean(
            evs_phase[i][0].elapsed_time(evs_phase[i][4]) for i in range(K)) * 1e3,
        "hbm_gbs": {"dispatch_gather": gb_g, "combine_scatter": gb_c, "gather+combine": gb_dc,
                    "pct_of_8tbs_gather+combine": 100 * gb_dc / 8000.0,
                    f"pct_of_{peak_kind}_{peak:.0f}": 100 * gb_dc / peak},
        "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": dom_bytes / (dom_ms / 1e3) / 1e9,
                     "peak": peak, "unit": "GB/s",
                     "frac": dom_bytes / (dom_ms / 1e3) / 1e9 / peak,
                     "peak_kind": f"of {peak_kind}", "algorithmic_bytes": dom_bytes,
                     "traffic": traffic},
        "clocks": clk,
        "gpu_launches": K * sum(KERNELS_PER_STEP.values()),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(S, args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        del g_main, g_phase
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


def run_e2e(coact, S: GpuStep, args, world, device):
    """The step through the public API from pinned host buffers: every step copies its
    inputs (ids, gates, placement, x and the expert outputs y) host -> device, runs the
    four calls and copies its outputs (combined rows and statistics) device -> host.
    Two device buffer sets let step i+1's input copy overlap step i's compute and
    output copy (copy engines in both directions run concurrently with the SMs)."""
    cfg = S.cfg
    names = ("ids", "gates", "expert_rank", "rank_node", "x", "y")
    host = {n: getattr(S, n).cpu().pin_memory() for n in names}
    bufs = [S, GpuStep(coact, S.r, device, fill=False)]
    out_h = [torch.empty(S.out.shape, dtype=S.out.dtype).pin_memory() for _ in range(2)]
    stats_h = [torch.empty(8, dtype=torch.int64).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size() + 8 * 8
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def run(n_steps):
        free = [None, None]
        for i in range(n_steps):
            b, slot = bufs[i % 2], i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_stream(comp) if i == 0 else None
                if free[slot] is not None:
                    s_in.wait_event(free[slot])
                for n, t in host.items():
                    getattr(b, n).copy_(t, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            comp.wait_event(ready)
            b.step()
            done = torch.cuda.Event()
            done.record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                out_h[slot].copy_(b.out, non_blocking=True)
                stats_h[slot].copy_(b.plan.stats, non_blocking=True)
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
            "note": "pinned host buffers; input copy of step i+1 overlaps compute and output "
                    "copy of step i (two device buffer sets)"}


# ----------------------------------------------------------------------------- the oracle


def _oracle_step(o, ids, gates, er, rn, n_nodes, E, R, xb, yb):
    o.count(ids, E)
    p = o.plan(ids, E, er, R, rank_node=rn, n_nodes=n_nodes)
    o.gather(xb, p["row_token"], p["D"])
    o.combine_f64(yb, gates, p["comb_row"])


def cpu_baseline(S: GpuStep, seconds: float):
    """The oracle, as it stands, on this host: whole batches of the same workload
    repeated for about `seconds` (at least one)."""
    import oracle as o
    from oracle import _bits
    r, cfg = S.r, S.cfg
    xb, yb = _bits(S.x), _bits(S.y)
    n, t0 = 0, time.perf_counter()
    while True:
        _oracle_step(o, r.ids, r.gates, r.expert_rank, r.rank_node, cfg.n_nodes, cfg.E, cfg.R, xb, yb)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": cfg.N * n / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} whole batches of config {cfg.index} (N={cfg.N}) through the "
                      "single-threaded C oracle: count, plan, gather, float64 combine",
            "host_cpu": _cpu_model(), "host_nproc": os.cpu_count()}


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
    xb = o._bits(workload.fill_bf16(cfg.N, cfg.H, r.seed, X_STREAM))
    yb = o._bits(workload.fill_bf16(cfg.N * cfg.k, cfg.H, r.seed, Y_STREAM))
    # each step: a bounded sample of the workload (the first n tokens' routing, whole
    # plan/gather/combine over them) sized so K + W steps end within a few minutes
    step_tokens = min(cfg.N, max(256, int(args.ref_tokens)))
    ids, gates = r.ids[:step_tokens], r.gates[:step_tokens]
    xs, ys = xb[:step_tokens], yb[:step_tokens * cfg.k]
    for _ in range(args.warmup):
        _oracle_step(o, ids, gates, r.expert_rank, r.rank_node, cfg.n_nodes, cfg.E, cfg.R, xs, ys)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(o, ids, gates, r.expert_rank, r.rank_node, cfg.n_nodes, cfg.E, cfg.R, xs, ys)
    dt = time.perf_counter() - t0
    value = step_tokens * args.steps / dt
    sample = (f"first {step_tokens} tokens of config {cfg.index} per step (count, plan, gather, "
              "float64 combine), single-threaded C oracle")
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


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1, choices=sorted(workload.CONFIGS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="coact", choices=["coact", "reference"])
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--clock-warm-s", type=float, default=1.0)
    ap.add_argument("--ref-tokens", type=int, default=4096)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
