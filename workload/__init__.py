"""Seeded synthetic MoE routing workloads for the co-activation dispatch/combine path.

This module is the one input generator that both the CUDA library's tests/bench and
the CPU oracle consume.  It holds none of the method's arithmetic: it draws router
logits, takes the router's top-k and softmax gates (the *model's* routing, which the
co-activation method leaves unchanged), and builds expert->rank and rank->node maps.
It counts no pairs, plans no dispatch, gathers and combines nothing.

Workloads follow the shapes and routing statistics of the pages:
  * "Cobalt: efficient distributed MoE training using expert co-activation",
    English abstract: EP over 32 B200 GPUs, expert pairs frequently co-activated by
    single tokens, cross-node token traffic.
  * Zyphra correlated expert placement / token shuffling, English abstract: top-2 and
    top-6 routing, EP 8-64 on 8-GPU nodes, "0.8% of the expert pairs ... selected
    together by 42% of tokens", layer-to-layer expert prediction, 12.5% -> 59% locally
    served assignments on one node.
The pages ship no router traces; these seeded configurations stand in for them.

Randomness:
  * routing (logits, planting, placements, layer-2 transitions) uses numpy PCG64
    streams keyed by (seed, config, purpose);
  * bulk bf16 tensors (hidden rows x, expert outputs y) use a counter-based hash
    (splitmix64 finaliser of a per-element counter) mapped to an Irwin-Hall(3)
    approximation of N(0,1) with exact integer/power-of-two arithmetic, so that any
    element can be regenerated on the host for sampled checks and the bulk can be
    filled on the GPU with bit-identical results (`fill_bf16`).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Config", "CONFIGS", "Routing", "TwoLayer", "make_routing", "make_two_layer",
    "contiguous_src_rank", "fill_bf16", "bf16_bits_to_float", "placement",
]

# ----------------------------------------------------------------------------- configs


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic workload.

    N tokens, E experts, top-k routing, hidden size H (bf16), R logical EP ranks of
    `epr` experts each, spread over `n_nodes` nodes of R // n_nodes ranks.
    """
    index: int
    N: int
    E: int
    k: int
    H: int
    R: int
    n_nodes: int
    zipf_s: Optional[float]          # Zipf(s) expert popularity prior, None = flat
    group_size: int                  # experts per planted co-activation group
    n_groups: int                    # number of planted groups
    fixed_groups: Optional[tuple]    # explicit groups (config 0), else drawn
    bias: float                      # logit bias added to a planted token's group
    plant_prob: float                # probability that a token is planted
    placement: str                   # contiguous | random | planted | roundrobin
    two_layer: bool = False
    desc: str = ""

    @property
    def epr(self) -> int:
        return self.E // self.R

    @property
    def ranks_per_node(self) -> int:
        return self.R // self.n_nodes

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# Planting probability of config 1.  The pages' statistic is a *realised*
# co-selection share (42% of tokens pick one of the 0.8% planted pairs, Zyphra
# abstract); a planted token misses its pair when an unbiased logit beats one of the
# two biased ones, so the planting probability sits above 0.42.  Calibrated once with
# this generator (seed 0) so that the realised share lands on 42%.
C1_PLANT_PROB = 0.47

CONFIGS = {
    0: Config(0, N=4096, E=8, k=2, H=256, R=4, n_nodes=1, zipf_s=None,
              group_size=2, n_groups=1, fixed_groups=((0, 5),), bias=3.0,
              plant_prob=0.40, placement="contiguous",
              desc="N=4096 E=8 top-2 H=256; 4 ranks x2 experts, 1 node; pair (0,5) +3.0 for 40%"),
    1: Config(1, N=16384, E=64, k=2, H=2048, R=8, n_nodes=1, zipf_s=None,
              group_size=2, n_groups=16, fixed_groups=None, bias=4.0,
              plant_prob=C1_PLANT_PROB, placement="random",
              desc="N=16384 E=64 top-2 H=2048; 8 ranks x8 experts, 1 node; 16 planted pairs +4 "
                   "(co-selected by ~42% of tokens); random placement"),
    2: Config(2, N=65536, E=64, k=6, H=4096, R=32, n_nodes=4, zipf_s=1.1,
              group_size=4, n_groups=8, fixed_groups=None, bias=2.5,
              plant_prob=0.30, placement="contiguous",
              desc="N=65536 E=64 top-6 H=4096; 32 ranks x2 experts in 4 nodes; Zipf(1.1); "
                   "8 planted groups of 4 (+2.5, 30%)"),
    3: Config(3, N=131072, E=256, k=8, H=7168, R=64, n_nodes=8, zipf_s=1.2,
              group_size=2, n_groups=32, fixed_groups=None, bias=3.0,
              plant_prob=0.35, placement="roundrobin",
              desc="N=131072 E=256 top-8 H=7168; 64 ranks x4 experts in 8 nodes; Zipf(1.2); "
                   "32 planted pairs (+3, 35%); round-robin placement, and the correlated "
                   "placement built from the batch's pair counts"),
    4: Config(4, N=65536, E=128, k=2, H=4096, R=16, n_nodes=2, zipf_s=None,
              group_size=2, n_groups=0, fixed_groups=None, bias=0.0,
              plant_prob=0.0, placement="contiguous", two_layer=True,
              desc="two MoE layers N=65536 E=128 top-2 H=4096; 16 ranks x8 experts in 2 nodes; "
                   "layer-2 experts from a sparse transition matrix; tokens pre-sharded to the "
                   "predicted layer-2 rank"),
}

_PURPOSE = {"routing": 1, "planting": 2, "zipf": 3, "placement": 4, "groups": 5,
            "transition": 6, "layer2": 7, "layer2_gates": 8}


def _rng(seed: int, cfg: int, purpose: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [int(seed) & 0xFFFFFFFF, int(cfg), _PURPOSE[purpose]])))


# ----------------------------------------------------------------------------- routing


@dataclasses.dataclass
class Routing:
    """Router output and EP layout for one MoE layer (host numpy arrays)."""
    cfg: Config
    ids: np.ndarray          # int32 [N, k]; slot order = descending logit
    gates: np.ndarray        # float32 [N, k]; softmax over the k selected logits
    expert_rank: np.ndarray  # int32 [E]
    rank_node: np.ndarray    # int32 [R]
    src_rank: np.ndarray     # int32 [N]; contiguous sequence-parallel shards
    groups: np.ndarray       # int32 [n_groups, group_size] planted groups
    planted: np.ndarray      # bool [N] token was planted
    seed: int

    @property
    def N(self): return self.ids.shape[0]

    @property
    def k(self): return self.ids.shape[1]


def contiguous_src_rank(N: int, R: int) -> np.ndarray:
    """Home rank of token t when sequence parallelism shards tokens contiguously."""
    return ((np.arange(N, dtype=np.int64) * R) // N).astype(np.int32)


def _topk_sorted(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, by descending logit, ties -> lower id."""
    part = np.argpartition(-logits, k - 1, axis=1)[:, :k]
    vals = np.take_along_axis(logits, part, axis=1)
    # lexsort: last key is primary -> (-value) primary, id secondary
    order = np.lexsort((part, -vals), axis=1)
    return np.take_along_axis(part, order, axis=1)


def _softmax_rows(v: np.ndarray) -> np.ndarray:
    m = v.max(axis=1, keepdims=True)
    e = np.exp(v - m)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _draw_groups(cfg: Config, seed: int) -> np.ndarray:
    if cfg.fixed_groups is not None:
        return np.asarray(cfg.fixed_groups, dtype=np.int32)
    if cfg.n_groups == 0:
        return np.zeros((0, cfg.group_size), dtype=np.int32)
    perm = _rng(seed, cfg.index, "groups").permutation(cfg.E)
    need = cfg.n_groups * cfg.group_size
    return perm[:need].reshape(cfg.n_groups, cfg.group_size).astype(np.int32)


def placement(cfg: Config, kind: str, groups: Optional[np.ndarray] = None,
              seed: int = 0) -> np.ndarray:
    """Expert -> rank map (int32 [E]), each rank holding exactly E/R experts.

    contiguous : expert e -> rank e // epr
    random     : a seeded permutation perm; expert perm[i] -> rank i // epr
    roundrobin : expert e -> rank e mod R
    planted    : co-locates the planted co-activation groups: groups in order go to
                 the lowest-index rank with room for the whole group, then the other
                 experts, ascending id, to the lowest rank with a free slot (uses the
                 generator's ground-truth groups; the placement built from *measured*
                 counts is the library's coact_place_correlated).
    identity   : E == R, expert e -> rank e (every expert alone on its rank)
    """
    E, R, epr = cfg.E, cfg.R, cfg.epr
    if kind == "contiguous":
        return (np.arange(E) // epr).astype(np.int32)
    if kind == "roundrobin":
        return (np.arange(E) % R).astype(np.int32)
    if kind == "identity":
        if E != R:
            raise ValueError("identity placement needs E == R")
        return np.arange(E, dtype=np.int32)
    if kind == "random":
        perm = _rng(seed, cfg.index, "placement").permutation(E)
        out = np.empty(E, dtype=np.int32)
        out[perm] = np.arange(E) // epr
        return out
    if kind == "planted":
        if groups is None:
            raise ValueError("planted placement needs the planted groups")
        out = np.full(E, -1, dtype=np.int32)
        free = np.full(R, epr, dtype=np.int64)
        for g in groups:
            g = [int(e) for e in g if out[e] < 0]
            if not g:
                continue
            for r in range(R):
                if free[r] >= len(g):
                    out[g] = r
                    free[r] -= len(g)
                    break
        for e in range(E):
            if out[e] < 0:
                r = int(np.nonzero(free > 0)[0][0])
                out[e] = r
                free[r] -= 1
        return out
    raise ValueError(f"unknown placement {kind!r}")


def make_routing(cfg: Config | int, seed: int = 0, placement_kind: Optional[str] = None,
                 N: Optional[int] = None) -> Routing:
    """Router top-k ids and gates plus the EP layout for one layer of `cfg`.

    logit[t, e] = N(0,1) + ln p(e) + bias * [t planted and e in t's group]
    where ln p(e) = -s ln(pi(e)+1) for a seeded permutation pi (Zipf(s) popularity,
    hot experts scattered over ranks) or 0 for a flat prior.  A token is planted
    with probability `plant_prob` and then gets one group uniformly.  ids are the
    top-k by descending logit (ties -> lower id); gates the softmax of those k logits
    computed in float64 and rounded to float32.
    """
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    if N is not None:
        cfg = cfg.with_(N=int(N))
    N, E, k = cfg.N, cfg.E, cfg.k
    rng = _rng(seed, cfg.index, "routing")
    logits = rng.standard_normal((N, E))
    if cfg.zipf_s:
        pi = _rng(seed, cfg.index, "zipf").permutation(E)
        logits += (-cfg.zipf_s * np.log(pi + 1.0))[None, :]
    groups = _draw_groups(cfg, seed)
    planted = np.zeros(N, dtype=bool)
    if cfg.n_groups > 0 and cfg.plant_prob > 0:
        prng = _rng(seed, cfg.index, "planting")
        planted = prng.random(N) < cfg.plant_prob
        which = prng.integers(0, len(groups), N)
        rows = np.nonzero(planted)[0]
        for c in range(groups.shape[1]):
            logits[rows, groups[which[rows], c]] += cfg.bias
    ids = _topk_sorted(logits, k).astype(np.int32)
    gates = _softmax_rows(np.take_along_axis(logits, ids.astype(np.int64), axis=1))
    kind = placement_kind or cfg.placement
    er = placement(cfg, kind, groups=groups, seed=seed)
    rank_node = (np.arange(cfg.R) // cfg.ranks_per_node).astype(np.int32)
    return Routing(cfg=cfg, ids=np.ascontiguousarray(ids), gates=np.ascontiguousarray(gates),
                   expert_rank=er, rank_node=rank_node,
                   src_rank=contiguous_src_rank(N, cfg.R), groups=groups,
                   planted=planted, seed=seed)


# ----------------------------------------------------------------------------- two layers


@dataclasses.dataclass
class TwoLayer:
    """Two consecutive MoE layers whose layer-2 picks follow layer-1 picks."""
    layer1: Routing
    layer2: Routing           # ids/gates of layer 2; src_rank = contiguous baseline
    succ: np.ndarray          # int32 [E, 4] the heavy successors of each expert
    calib1: np.ndarray        # int32 [N, k] calibration batch, layer-1 ids
    calib2: np.ndarray        # int32 [N, k] calibration batch, layer-2 ids


def _transition(E: int, rng: np.random.Generator):
    """Sparse transition: 4 distinct successors at 0.175 each, 0.30 over the rest."""
    succ = np.empty((E, 4), dtype=np.int64)
    others = np.empty((E, E - 4), dtype=np.int64)
    for a in range(E):
        s = rng.choice(E, size=4, replace=False)
        succ[a] = s
        mask = np.ones(E, dtype=bool)
        mask[s] = False
        others[a] = np.nonzero(mask)[0]
    return succ, others


def _draw_successor(a: np.ndarray, succ, others, rng) -> np.ndarray:
    u = rng.random(a.shape)
    heavy = u < 0.7
    out = np.empty(a.shape, dtype=np.int64)
    hi = np.minimum((u[heavy] / 0.175).astype(np.int64), 3)
    out[heavy] = succ[a[heavy], hi]
    n_other = others.shape[1]
    lo = np.minimum(((u[~heavy] - 0.7) / 0.3 * n_other).astype(np.int64), n_other - 1)
    out[~heavy] = others[a[~heavy], lo]
    return out


def _layer2_ids(ids1: np.ndarray, succ, others, rng) -> np.ndarray:
    N, k = ids1.shape
    out = np.empty((N, k), dtype=np.int64)
    for j in range(k):
        out[:, j] = _draw_successor(ids1[:, j].astype(np.int64), succ, others, rng)
        # a token picks k distinct experts: redraw slot j while it repeats an earlier slot
        for _ in range(64):
            clash = np.zeros(N, dtype=bool)
            for jj in range(j):
                clash |= out[:, j] == out[:, jj]
            rows = np.nonzero(clash)[0]
            if rows.size == 0:
                break
            out[rows, j] = _draw_successor(ids1[rows, j].astype(np.int64), succ, others, rng)
        else:
            for t in rows:
                used = set(out[t, :j].tolist())
                out[t, j] = min(e for e in range(others.shape[0]) if e not in used)
    return out.astype(np.int32)


def make_two_layer(cfg: Config | int = 4, seed: int = 0, N: Optional[int] = None) -> TwoLayer:
    """Config 4: layer-1 routing (flat N(0,1) logits, top-k), layer-2 experts drawn
    from a seeded sparse E x E transition of the layer-1 picks (70% of the mass on 4
    successors), layer-2 gates = softmax of k fresh N(0,1) logits, and a separate
    calibration batch (seed + 1) from which the layer-1 -> layer-2 counts are taken."""
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    if N is not None:
        cfg = cfg.with_(N=int(N))
    l1 = make_routing(cfg, seed=seed)
    succ, others = _transition(cfg.E, _rng(seed, cfg.index, "transition"))
    ids2 = _layer2_ids(l1.ids, succ, others, _rng(seed, cfg.index, "layer2"))
    g2 = _softmax_rows(_rng(seed, cfg.index, "layer2_gates").standard_normal((cfg.N, cfg.k)))
    l2 = dataclasses.replace(l1, ids=ids2, gates=g2)
    cal1 = make_routing(cfg, seed=seed + 1).ids
    cal2 = _layer2_ids(cal1, succ, others, _rng(seed + 1, cfg.index, "layer2"))
    return TwoLayer(layer1=l1, layer2=l2, succ=succ.astype(np.int32), calib1=cal1, calib2=cal2)


# ----------------------------------------------------------------------------- bf16 bulk fill

_GOLDEN = -7046029254386353131    # 0x9E3779B97F4A7C15 as int64
_MIX1 = -4658895280553007687      # 0xBF58476D1CE4E5B9
_MIX2 = -7723592293110705685      # 0x94D049BB133111EB


def _srl(z, s: int):
    """Logical right shift of an int64 tensor."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _splitmix(z):
    z = z + _GOLDEN
    z = (z ^ _srl(z, 30)) * _MIX1
    z = (z ^ _srl(z, 27)) * _MIX2
    return z ^ _srl(z, 31)


def _stream_key(seed: int, stream: int) -> int:
    v = ((int(seed) & 0xFFFFFFFF) << 20) ^ (int(stream) & 0xFFFFF)
    v = (v * 0x9E3779B97F4A7C15 + 0x632BE59BD9B4E019) & 0xFFFFFFFFFFFFFFFF
    return v - (1 << 64) if v >= (1 << 63) else v


def fill_bf16(rows: int, H: int, seed: int, stream: int, device="cpu", row0: int = 0,
              row_ids=None, chunk_rows: Optional[int] = None):
    """bf16 tensor [rows, H] whose element (i, h) is a pure function of
    (seed, stream, row0 + i, h) -- or of (row_ids[i], h) when `row_ids` is given.

    value = (2*(u0+u1+u2) - 196605) * 2^-16 with u0..u2 the three low 16-bit words of
    splitmix64(key + row*H + h): an Irwin-Hall(3) approximation of N(0,1) (mean 0,
    variance 1) that is exact in fp32, rounded to bf16 nearest-even with integer ops.
    Same value on CPU and GPU.  Returns a torch.bfloat16 tensor on `device`.
    """
    import torch
    dev = torch.device(device)
    key = _stream_key(seed, stream)
    out = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
    if rows == 0:
        return out
    if chunk_rows is None:
        chunk_rows = max(1, (1 << 26) // max(H, 1))
    cols = torch.arange(H, dtype=torch.int64, device=dev)
    ids_t = None
    if row_ids is not None:
        ids_t = torch.as_tensor(np.asarray(row_ids, dtype=np.int64), device=dev)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        if ids_t is None:
            rr = torch.arange(row0 + r0, row0 + r1, dtype=torch.int64, device=dev)
        else:
            rr = ids_t[r0:r1]
        z = _splitmix(rr[:, None] * H + cols[None, :] + key)
        s = (z & 0xFFFF) + (_srl(z, 16) & 0xFFFF) + (_srl(z, 32) & 0xFFFF)
        f = (2 * s - 196605).to(torch.float32) * (2.0 ** -16)   # exact in fp32
        u = f.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
        u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16               # nearest-even to bf16
        out[r0:r1] = (u & 0xFFFF).to(torch.int32).to(torch.int16).view(torch.bfloat16)
    return out


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def pages_stats(r: Routing) -> dict:
    """Routing statistics the pages quote, measured on a generated workload:
    share of tokens whose top-k contains a whole planted group, max/mean expert load."""
    cfg = r.cfg
    ids = r.ids
    share = 0.0
    if len(r.groups):
        hit = np.zeros(r.N, dtype=bool)
        for g in r.groups:
            has = np.ones(r.N, dtype=bool)
            for e in g:
                has &= (ids == e).any(axis=1)
            hit |= has
        share = float(hit.mean())
    load = np.bincount(ids.ravel(), minlength=cfg.E)
    return {"group_coselect_share": share,
            "load_max_over_mean": float(load.max() / max(load.mean(), 1e-9))}


# ----------------------------------------------------------------------------- replicas


def replicate_hot(loads, expert_rank, rank_node, n_hot: int, max_rep: int = 2):
    """Replica layout fixture (the pages give none; Cobalt says only that EP distributes
    expert replicas across GPUs): every expert keeps its rank as replica 0; the n_hot most
    loaded experts (ties: lower id) each get one more replica, heaviest first, on the
    rank with the least current load among the ranks of other nodes (ties: lower rank),
    counting half of the expert's load as moved there.  Returns (rep_rank int32
    [E, max_rep] with -1 padding, n_rep int32 [E])."""
    loads = np.asarray(loads, dtype=np.int64)
    er = np.asarray(expert_rank, dtype=np.int64)
    rn = np.asarray(rank_node, dtype=np.int64)
    E, R = len(loads), len(rn)
    rep = np.full((E, max_rep), -1, np.int32)
    rep[:, 0] = er
    n_rep = np.ones(E, np.int32)
    rank_load = np.zeros(R, np.float64)
    np.add.at(rank_load, er, loads.astype(np.float64))
    hot = sorted(range(E), key=lambda e: (-loads[e], e))[:n_hot]
    for e in hot:
        if max_rep < 2:
            break
        cand = [r for r in range(R) if rn[r] != rn[er[e]]]
        if not cand:
            continue
        r = min(cand, key=lambda q: (rank_load[q], q))
        rep[e, 1] = r
        n_rep[e] = 2
        rank_load[er[e]] -= loads[e] / 2
        rank_load[r] += loads[e] / 2
    return rep, n_rep
