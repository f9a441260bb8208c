"""CPU oracle for the co-activation dispatch/combine path (numpy front end).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg -- never by the library.  The arithmetic lives in
`coact_oracle.c` (plain single-threaded C, compiled here with gcc); this module only
allocates numpy arrays and marshals them.  It shares no code with the CUDA library.

Parity pins: see tests/test_oracle_pins.py.  Each function below names the page
passage its definition follows (in the C source).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "coact_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FLAG_ID_RANGE, FLAG_DUP_ID, FLAG_CAPACITY, FLAG_SRC_RANK = 1, 2, 4, 8
N_STATS = 8
STAT_NAMES = ("naive_rows", "dedup_rows", "remote_rows", "crossnode_rows",
              "node_dedup_crossnode_rows", "local_served_asg", "remote_asg", "crossnode_asg")


def build(force: bool = False) -> str:
    """Compile coact_oracle.c into liboracle.so (plain gcc, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off",
                               "-fno-fast-math", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32 = ctypes.c_int64, ctypes.c_int
            _lib.oracle_count.argtypes = [P, I64, I32, I32, P, P]
            _lib.oracle_count_cross.argtypes = [P, I32, I32, P, I32, I32, I64, P, P]
            _lib.oracle_plan.argtypes = [P, I64, I32, I32, P, I32, P, I32, P, P, P, P, P, P, P,
                                         I64, P, P, P, P]
            _lib.oracle_plan_slots.argtypes = _lib.oracle_plan.argtypes
            _lib.oracle_assign_replicas.argtypes = [P, I64, I32, I32, P, I32, P, I32, P, I32, P, P]
            _lib.oracle_place_replicas.argtypes = [P, P, P, I32, P, I32, I32, I32, P, P]
            _lib.oracle_gather.argtypes = [P, I64, P, I64, P]
            _lib.oracle_gather.restype = None
            _lib.oracle_combine_f64.argtypes = [P, I64, P, P, I64, I32, I64, P]
            _lib.oracle_combine_f64.restype = None
            _lib.oracle_combine_f32chain.argtypes = [P, I64, P, P, I64, I32, I64, P]
            _lib.oracle_combine_f32chain.restype = None
            _lib.oracle_bf16_rne_array.argtypes = [P, P, I64]
            _lib.oracle_bf16_rne_array.restype = None
            _lib.oracle_expand_identity.argtypes = [P, I64, P, P, I64, P]
            _lib.oracle_expand_identity.restype = I64
            _lib.oracle_naive_combine_identity_f32.argtypes = [P, P, I64, I32, I64, P]
            _lib.oracle_naive_combine_identity_f32.restype = None
            _lib.oracle_predict_home.argtypes = [P, I64, I32, I32, P, I32, P, I32, P]
            _lib.oracle_place_correlated.argtypes = [P, I32, I32, P]
            _lib.oracle_rebalance_ranks.argtypes = [P, P, I32, P, I32, P]
            _lib.oracle_forward_src.argtypes = [P, P, I32, P, P, P, I32, I64, I64, P]
            _lib.oracle_forward_src.restype = None
            _lib.oracle_forward_gather.argtypes = [P, I64, P, I64, P]
            _lib.oracle_forward_gather.restype = None
            _lib.oracle_gather_backward_f32chain.argtypes = [P, I64, P, I64, I32, I64, P]
            _lib.oracle_gather_backward_f32chain.restype = None
            _lib.oracle_combine_units_f32chain.argtypes = [P, I64, P, P, I32, P, P, I64, I64, P]
            _lib.oracle_combine_units_f32chain.restype = None
            _lib.oracle_combine_backward.argtypes = [P, I64, P, P, I32, P, P, I64, I64, P, P, P, P]
            _lib.oracle_combine_backward.restype = None
            _lib.oracle_shuffle_reduce_f32chain.argtypes = [P, I32, I64, I64, P, I64, P]
            _lib.oracle_shuffle_reduce_f32chain.restype = None
            _lib.oracle_row_meta.argtypes = [P, P, I64, P, I32, P, P, P, I64, I32, P, P, P, P]
            _lib.oracle_gather_row_slots.argtypes = [P, I64, P, P, I64, I32, P]
        return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _bits(a) -> np.ndarray:
    """bf16 data as uint16 bit patterns (accepts uint16/int16 numpy or a torch bf16 tensor)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.asarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.uint16)


# ----------------------------------------------------------------------------- counting


def count(ids, E: int, pair=None, loads=None):
    """Co-activation pair counts [E,E] and loads [E] (int64, accumulated).  Returns
    (pair, loads, flags)."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    pair = np.zeros((E, E), np.int64) if pair is None else pair
    loads = np.zeros(E, np.int64) if loads is None else loads
    f = _get().oracle_count(_p(ids), N, k, E, _p(pair), _p(loads))
    return pair, loads, f


def count_cross(ids1, E1: int, ids2, E2: int, C12=None, loads1=None):
    """Cross-layer counts C12 [E1,E2] and layer-1 loads (int64, accumulated)."""
    ids1, ids2 = _c(ids1, np.int32), _c(ids2, np.int32)
    N, k1 = ids1.shape
    k2 = ids2.shape[1]
    C12 = np.zeros((E1, E2), np.int64) if C12 is None else C12
    loads1 = np.zeros(E1, np.int64) if loads1 is None else loads1
    f = _get().oracle_count_cross(_p(ids1), k1, E1, _p(ids2), k2, E2, N, _p(C12), _p(loads1))
    return C12, loads1, f


# ----------------------------------------------------------------------------- plan


def plan(ids, E: int, expert_rank, R: int, rank_node=None, n_nodes: int = 1, src_rank=None,
         row_capacity: Optional[int] = None, slot_rank=None) -> dict:
    """Deduplicated dispatch plan; returns a dict of numpy arrays plus 'flags' and 'D'.
    With slot_rank (int32 [N, k]) every slot goes to its own rank and expert_rank is not
    used (expert replicas)."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    er = _c(expert_rank if slot_rank is None else slot_rank, np.int32)
    rn = None if rank_node is None else _c(rank_node, np.int32)
    sr = None if src_rank is None else _c(src_rank, np.int32)
    cap = N * min(k, R) if row_capacity is None else int(row_capacity)
    out = {
        "rank_counts": np.zeros(R, np.int32),
        "rank_offsets": np.zeros(R + 1, np.int32),
        "asg_offsets": np.zeros(R + 1, np.int32),
        "rank_mask": np.zeros(N, np.uint64),
        "row_token": np.full(max(cap, 0), -1, np.int32),
        "row_kmask": np.zeros(max(cap, 0), np.uint8),
        "send_row": np.zeros((N, k), np.int32),
        "comb_row": np.zeros((N, k), np.int32),
        "stats": np.zeros(N_STATS, np.int64),
        "src_dst": np.zeros((R, R), np.int32),
    }
    fn = _get().oracle_plan if slot_rank is None else _get().oracle_plan_slots
    f = fn(_p(ids), N, k, E, _p(er), R, _p(rn), n_nodes, _p(sr),
                           _p(out["rank_counts"]), _p(out["rank_offsets"]),
                           _p(out["asg_offsets"]), _p(out["rank_mask"]), _p(out["row_token"]),
                           _p(out["row_kmask"]), cap, _p(out["send_row"]), _p(out["comb_row"]),
                           _p(out["stats"]), _p(out["src_dst"]))
    out["flags"] = f
    out["D"] = int(out["rank_offsets"][R])
    out["row_capacity"] = cap
    return out


# ----------------------------------------------------------------------------- rows


def gather(x, row_token, D: int) -> np.ndarray:
    """send[d] = x[row_token[d]] for d < D (uint16 bf16 bits [D, H])."""
    xb = _bits(x)
    H = xb.shape[1]
    rt = _c(row_token, np.int32)
    send = np.zeros((D, H), np.uint16)
    _get().oracle_gather(_p(xb), H, _p(rt), D, _p(send))
    return send


def combine_f64(y, gates, comb_row) -> np.ndarray:
    """out[t] = sum_j gate[t,j] * y[comb_row[t,j]] in float64 ([N, H])."""
    yb = _bits(y)
    g = _c(gates, np.float32)
    cr = _c(comb_row, np.int32)
    N, k = g.shape
    H = yb.shape[1]
    out = np.zeros((N, H), np.float64)
    _get().oracle_combine_f64(_p(yb), yb.shape[0], _p(g), _p(cr), N, k, H, _p(out))
    return out


def combine_f32chain(y, gates, comb_row) -> np.ndarray:
    """The fixed-order fp32 fma chain (ascending j from +0) ([N, H] float32)."""
    yb = _bits(y)
    g = _c(gates, np.float32)
    cr = _c(comb_row, np.int32)
    N, k = g.shape
    H = yb.shape[1]
    out = np.zeros((N, H), np.float32)
    _get().oracle_combine_f32chain(_p(yb), yb.shape[0], _p(g), _p(cr), N, k, H, _p(out))
    return out


def bf16_rne(a) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (the oracle's own definition)."""
    a = _c(a, np.float32)
    out = np.zeros(a.shape, np.uint16)
    _get().oracle_bf16_rne_array(_p(a), _p(out), a.size)
    return out


def expand_identity(x, row_token, row_kmask, D: int) -> np.ndarray:
    """Identity-expert outputs in expanded receive order ([sum popcount(row_kmask[:D]), H])."""
    xb = _bits(x)
    H = xb.shape[1]
    rt = _c(row_token, np.int32)
    km = _c(row_kmask, np.uint8)
    n = int(sum(bin(int(v)).count("1") for v in km[:D]))
    y = np.zeros((n, H), np.uint16)
    got = _get().oracle_expand_identity(_p(xb), H, _p(rt), _p(km), D, _p(y))
    assert got == n
    return y


def naive_combine_identity_f32(x, gates) -> np.ndarray:
    """Non-deduplicated combine with identity experts (fp32 chain), [N, H] float32."""
    xb = _bits(x)
    g = _c(gates, np.float32)
    N, k = g.shape
    H = xb.shape[1]
    out = np.zeros((N, H), np.float32)
    _get().oracle_naive_combine_identity_f32(_p(xb), _p(g), N, k, H, _p(out))
    return out


def predict_home(ids1, E1: int, C12, expert_rank2, R: int):
    """Predicted layer-2 home rank per token (int32 [N]) and flags."""
    ids1 = _c(ids1, np.int32)
    N, k1 = ids1.shape
    C = _c(C12, np.int64)
    E2 = C.shape[1]
    er2 = _c(expert_rank2, np.int32)
    home = np.zeros(N, np.int32)
    f = _get().oracle_predict_home(_p(ids1), N, k1, E1, _p(C), E2, _p(er2), R, _p(home))
    return home, f


def place_correlated(pair, R: int) -> np.ndarray:
    """Greedy correlated placement from pair counts (int32 expert -> rank, [E])."""
    pr = _c(pair, np.int64)
    E = pr.shape[0]
    out = np.zeros(E, np.int32)
    if _get().oracle_place_correlated(_p(pr), E, R, _p(out)) != 0:
        raise ValueError("E must be a multiple of R")
    return out


def node_maps(expert_rank, rank_node, src_rank=None, N=None, R=None):
    """expert -> node and token -> home node maps for the node-level (hop-1) plan."""
    er = np.asarray(expert_rank, np.int64)
    rn = np.asarray(rank_node, np.int64)
    expert_node = rn[er].astype(np.int32)
    if src_rank is None:
        src_rank = (np.arange(N, dtype=np.int64) * R) // N
    src_node = rn[np.asarray(src_rank, np.int64)].astype(np.int32)
    return expert_node, src_node


def plan_two_hop(ids, E: int, expert_rank, R: int, rank_node, n_nodes: int, src_rank=None):
    """(node-level plan, rank-level plan, fwd_src): hop 1 sends each token once per node,
    hop 2 forwards each node-level row to the token's ranks in that node."""
    ids = _c(ids, np.int32)
    N = ids.shape[0]
    en, sn = node_maps(expert_rank, rank_node, src_rank, N, R)
    node = plan(ids, E, en, n_nodes, rank_node=np.arange(n_nodes, dtype=np.int32),
                n_nodes=n_nodes, src_rank=sn)
    rank = plan(ids, E, expert_rank, R, rank_node=rank_node, n_nodes=n_nodes, src_rank=src_rank)
    fwd = forward_src(rank, rank_node, node, n_nodes)
    return node, rank, fwd


def forward_src(rank_plan: dict, rank_node, node_plan: dict, n_nodes: int) -> np.ndarray:
    rt = _c(rank_plan["row_token"], np.int32)
    ro = _c(rank_plan["rank_offsets"], np.int32)
    R = ro.shape[0] - 1
    rn = _c(rank_node, np.int32)
    nrt = _c(node_plan["row_token"], np.int32)
    no = _c(node_plan["rank_offsets"], np.int32)
    N = rank_plan["send_row"].shape[0]
    cap = rt.shape[0]
    out = np.zeros(cap, np.int32)
    _get().oracle_forward_src(_p(rt), _p(ro), R, _p(rn), _p(nrt), _p(no), n_nodes, N, cap, _p(out))
    return out


def forward_gather(src, fwd_src, cap=None) -> np.ndarray:
    """dst[d] = src[fwd_src[d]] where fwd_src[d] >= 0 (zeros elsewhere)."""
    sb = _bits(src)
    H = sb.shape[1]
    f = _c(fwd_src, np.int32)
    cap = f.shape[0] if cap is None else cap
    dst = np.zeros((cap, H), np.uint16)
    _get().oracle_forward_gather(_p(sb), H, _p(f), cap, _p(dst))
    return dst


def rebalance_ranks(loads, expert_node, rank_node) -> np.ndarray:
    """Longest-first intra-node rebalancing (expert -> rank, int32 [E])."""
    ld = _c(loads, np.int64)
    en = _c(expert_node, np.int32)
    rn = _c(rank_node, np.int32)
    E, R = ld.shape[0], rn.shape[0]
    out = np.zeros(E, np.int32)
    if _get().oracle_rebalance_ranks(_p(ld), _p(en), E, _p(rn), R, _p(out)) != 0:
        raise ValueError("a node's expert count does not match its slots")
    return out


def place_two_stage(pair, loads, rank_node, n_nodes: int) -> np.ndarray:
    """Stage 1: correlated placement at node granularity; stage 2: rebalance in nodes."""
    expert_node = place_correlated(pair, n_nodes)
    return rebalance_ranks(loads, expert_node, rank_node)


# ----------------------------------------------------------------------------- backward


def gather_backward_f32chain(g_send, send_row) -> np.ndarray:
    """Transpose of the dispatch: grad_x[t] = sum of grad_send[send_row[t,j]] over the
    token's send rows (ascending j, fp32 add chain from +0) ([N, H] float32)."""
    gb = _bits(g_send)
    sr = _c(send_row, np.int32)
    N, k = sr.shape
    H = gb.shape[1]
    out = np.zeros((N, H), np.float32)
    _get().oracle_gather_backward_f32chain(_p(gb), gb.shape[0], _p(sr), N, k, H, _p(out))
    return out


def _units(row_token, row_kmask, n_units, N):
    if row_token is None:
        return None, None, N
    rt = _c(row_token, np.int32)
    km = _c(row_kmask, np.uint8)
    n = len(rt) if n_units is None else int(n_units)
    return rt[:n].copy(), km[:n].copy(), n


def combine_units_f32chain(y, gates, comb_row, row_token=None, row_kmask=None,
                           n_units=None) -> np.ndarray:
    """Combine over units: unit u is token row_token[u] restricted to the slots of
    row_kmask[u] (or token u, all slots, without row_token) ([n_units, H] float32)."""
    yb = _bits(y)
    g = _c(gates, np.float32)
    cr = _c(comb_row, np.int32)
    N, k = g.shape
    rt, km, n = _units(row_token, row_kmask, n_units, N)
    H = yb.shape[1]
    out = np.zeros((n, H), np.float32)
    _get().oracle_combine_units_f32chain(_p(yb), yb.shape[0], _p(g), _p(cr), k, _p(rt), _p(km),
                                         n, H, _p(out))
    return out


def combine_backward(y, gates, comb_row, g_out, row_token=None, row_kmask=None, n_units=None,
                     g_y=None):
    """Backward of the combine.  Returns (g_y bf16 bits [n_rows, H] -- rows no slot names
    keep the contents of the g_y passed in (zeros by default) --, g_gates float64 [N, k],
    g_gates_abs float64 [N, k]); slots no unit covers are 0 in both."""
    yb = _bits(y)
    g = _c(gates, np.float32)
    cr = _c(comb_row, np.int32)
    N, k = g.shape
    rt, km, n = _units(row_token, row_kmask, n_units, N)
    H = yb.shape[1]
    gob = _bits(g_out)
    assert gob.shape == (n, H)
    gy = np.zeros(yb.shape, np.uint16) if g_y is None else _bits(g_y).copy()
    gg = np.zeros((N, k), np.float64)
    ga = np.zeros((N, k), np.float64)
    _get().oracle_combine_backward(_p(yb), yb.shape[0], _p(g), _p(cr), k, _p(rt), _p(km), n, H,
                                   _p(gob), _p(gy), _p(gg), _p(ga))
    return gy, gg, ga


def combine_prereduced(y, gates, plan_: dict):
    """The pre-reduced reverse path over a plan: one partial row per send row (bf16), then
    the transposed dispatch adds each token's partial rows.  Returns (pre bf16 bits [D, H],
    out float32 [N, H] before the final rounding)."""
    D = plan_["D"]
    pre = bf16_rne(combine_units_f32chain(y, gates, plan_["comb_row"], plan_["row_token"],
                                          plan_["row_kmask"], D))
    return pre, gather_backward_f32chain(pre, plan_["send_row"])


# ----------------------------------------------------------------------------- token shuffling


def shuffle_order(home, R: int) -> dict:
    """The shuffle's permutation: the dispatch plan of every token to its predicted home
    rank alone (k = 1, identity expert -> rank map): row_token lists the tokens grouped by
    home rank in ascending token order, rank_offsets delimits the ranks' segments."""
    if R < 1:
        raise ValueError("token shuffling needs at least one rank")
    home = _c(home, np.int32)
    E = max(R, 2)                  # the plan takes E >= 2; with one rank both map to it
    return plan(home.reshape(-1, 1), E, np.minimum(np.arange(E, dtype=np.int32), R - 1), R)


def shuffle_reduce_f32chain(parts, row_token) -> np.ndarray:
    """out[i] = sum over q of parts[q][row_token[i]], fp32 add chain in rank order
    ([n_out, H] float32); parts: bf16 bits [P, N, H]."""
    pb = _bits(parts)
    Pn, N, H = pb.shape
    rt = _c(row_token, np.int32)
    out = np.zeros((len(rt), H), np.float32)
    _get().oracle_shuffle_reduce_f32chain(_p(pb), Pn, N, H, _p(rt), len(rt), _p(out))
    return out


# ----------------------------------------------------------------------------- replicas


def assign_replicas(ids, E: int, rep_rank, n_rep, R: int, rank_node=None, n_nodes: int = 1,
                    src_rank=None):
    """Replica choice per (token, slot) (int32 [N, k], -1 for invalid tokens) and flags;
    rep_rank: int32 [E, max_rep], n_rep: int32 [E]."""
    ids = _c(ids, np.int32)
    N, k = ids.shape
    rr = _c(rep_rank, np.int32)
    nr = _c(n_rep, np.int32)
    rn = None if rank_node is None else _c(rank_node, np.int32)
    sr = None if src_rank is None else _c(src_rank, np.int32)
    out = np.zeros((N, k), np.int32)
    f = _get().oracle_assign_replicas(_p(ids), N, k, E, _p(rr), rr.shape[1], _p(nr), R, _p(rn),
                                      n_nodes, _p(sr), _p(out))
    return out, f


def place_replicas(pair, loads, expert_rank, rank_node, budget: int, max_rep: int = 2):
    """Replica layout from co-activation and load statistics: (rep_rank int32 [E, max_rep]
    with -1 padding, n_rep int32 [E], replicas added)."""
    pr = _c(pair, np.int64)
    ld = _c(loads, np.int64)
    er = _c(expert_rank, np.int32)
    rn = _c(rank_node, np.int32)
    E, R = len(ld), len(rn)
    rep = np.zeros((E, max_rep), np.int32)
    nrep = np.zeros(E, np.int32)
    added = _get().oracle_place_replicas(_p(pr), _p(ld), _p(er), E, _p(rn), R, budget, max_rep,
                                         _p(rep), _p(nrep))
    return rep, nrep, added


# ----------------------------------------------------------------------------- EP row metadata


def row_meta(plan_: dict, ids, gates, slot_base=None, n_rows=None):
    """Per send row of a plan, one entry per slot: (expert ids int32 [n, k], gates fp32
    [n, k], expert-output slots int32 [n, k], flags) -- -1 / 0 / -1 where the row does not
    serve the slot; slots are comb_row + slot_base[rank of the row] (slot_base None: 0).
    n_rows defaults to the plan's D."""
    ids = _c(ids, np.int32)
    g = _c(gates, np.float32)
    N, k = ids.shape
    n = plan_["D"] if n_rows is None else int(n_rows)
    ro = _c(plan_["rank_offsets"], np.int32)
    sb = None if slot_base is None else _c(slot_base, np.int32)
    # sentinels, so that every entry must be written by the C code
    ex = np.full((n, k), -7, np.int32)
    go = np.full((n, k), np.nan, np.float32)
    sl = np.full((n, k), -7, np.int32)
    f = _get().oracle_row_meta(_p(_c(plan_["row_token"], np.int32)),
                               _p(_c(plan_["row_kmask"], np.uint8)), n, _p(ro), len(ro) - 1,
                               _p(ids), _p(g), _p(_c(plan_["comb_row"], np.int32)), N, k, _p(sb),
                               _p(ex), _p(go), _p(sl))
    return ex, go, sl, f


def gather_row_slots(vals, send_row, row_kmask):
    """out[t, j] = vals[d, j] for the send row d of token t that holds slot j (0 where none
    does); vals fp32 [n_rows, k].  Returns (out fp32 [N, k], flags)."""
    v = _c(vals, np.float32)
    sr = _c(send_row, np.int32)
    km = _c(row_kmask, np.uint8)
    N, k = sr.shape
    out = np.full((N, k), np.nan, np.float32)     # every entry must be written by the C code
    f = _get().oracle_gather_row_slots(_p(v), v.shape[0], _p(sr), _p(km), N, k, _p(out))
    return out, f
