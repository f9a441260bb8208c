"""Python binding of libcoact.so, the B200 co-activation dispatch/combine library.

Thin marshalling only: every entry point takes torch CUDA tensors, checks dtype /
shape / contiguity, and passes data pointers and the current CUDA stream to the C ABI
declared in include/coact.h.  All computation happens in the library's CUDA kernels;
there is no CPU fallback, and importing this module fails loudly if the library has
not been built (python co_activation_b200/build.py).

Entry points (same names as the C ABI):
  coact_count, plan_dispatch, dispatch_gather, combine_scatter, predict_home
plus allocation helpers (`alloc_plan`, `plan_workspace`) that only create torch tensors.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("COACT_LIB", os.path.join(_PKG, "libcoact.so"))

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libcoact.so not found at {LIB_PATH}: build it first with "
        "`python co_activation_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
EFLAG_ID_RANGE, EFLAG_DUP_ID, EFLAG_CAPACITY, EFLAG_SRC_RANK, EFLAG_ROW_RANGE, EFLAG_TIMEOUT = (
    1, 2, 4, 8, 16, 32)
NUM_STATS = 8
STAT_NAMES = ("naive_rows", "dedup_rows", "remote_rows", "crossnode_rows",
              "node_dedup_crossnode_rows", "local_served_asg", "remote_asg", "crossnode_asg")
MAX_K, MAX_E, MAX_R, MAX_REPLICAS = 8, 1024, 64, 8

_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_lib.coact_strerror.argtypes = [_I32]
_lib.coact_strerror.restype = ctypes.c_char_p
_lib.coact_abi_version.restype = _I32
_lib.coact_last_cuda_error.restype = _I32
_lib.coact_count.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P]
_lib.plan_dispatch_workspace_bytes.argtypes = [_I64, _I32, _I32, _I32]
_lib.plan_dispatch_workspace_bytes.restype = _SZ
_lib.plan_dispatch.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _I32, _P, _P, _P, _P, _P, _P,
                               _P, _I64, _P, _P, _P, _P, _P, _SZ, _P, _P]
_lib.plan_dispatch_slots.argtypes = _lib.plan_dispatch.argtypes
_lib.assign_replicas.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _I32, _P, _I32, _P, _P, _P, _P]
_lib.dispatch_gather.argtypes = [_P, _I64, _I64, _P, _I32, _P, _I64, _P, _P]
_lib.dispatch_gather_tma.argtypes = [_P, _I64, _I64, _P, _I32, _P, _I64, _P, _P]
_lib.combine_scatter.argtypes = [_P, _I64, _P, _P, _I64, _I32, _I64, _P, _I32, _P, _P]
_lib.combine_rows.argtypes = [_P, _I64, _P, _P, _I64, _I32, _P, _P, _I64, _P, _I64, _P, _I32, _P,
                              _P]
_lib.dispatch_gather_backward.argtypes = [_P, _I64, _P, _I64, _I32, _I64, _P, _I32, _P, _P]
_lib.shuffle_reduce_scatter.argtypes = [_P, _I32, _I64, _I64, _P, _I64, _P, _I32, _P, _P]
_lib.combine_scatter_backward.argtypes = [_P, _I64, _P, _P, _I64, _I32, _P, _P, _I64, _P, _P,
                                          _I64, _P, _P, _P, _P]
_lib.predict_home_workspace_bytes.argtypes = [_I32, _I32]
_lib.predict_home_workspace_bytes.restype = _SZ
_lib.predict_home.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _I32, _P, _P, _SZ, _P, _P]
_lib.coact_place_correlated.argtypes = [_P, _I32, _I32, _P]
_lib.coact_rebalance_ranks.argtypes = [_P, _P, _I32, _P, _I32, _P]
_lib.coact_place_replicas.argtypes = [_P, _P, _P, _I32, _P, _I32, _I32, _I32, _P, _P]
_lib.dispatch_gather_peer.argtypes = [_P, _I64, _I64, _P, _I32, _P, _I32, _P, _P, _P, _P, _P]
_lib.combine_scatter_peer.argtypes = [_P, _P, _P, _P, _I32, _P, _P, _I64, _I32, _I64, _P, _I32,
                                      _P, _P]
_lib.coact_compose_map.argtypes = [_P, _I64, _P, _I64, _P, _P, _P]
_lib.plan_forward.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _I32, _P, _P, _P, _P, _I64, _P, _P]
_lib.forward_gather.argtypes = [_P, _I64, _I64, _P, _I64, _P, _P, _P]
_lib.forward_gather_tokens.argtypes = [_P, _I64, _I64, _P, _I64, _I32, _P, _I64, _P, _P, _P]
_lib.plan_row_meta.argtypes = [_P, _P, _I64, _P, _I32, _P, _P, _P, _I64, _I32, _P, _P, _P, _P, _P,
                               _P]
_lib.gather_row_slots.argtypes = [_P, _I64, _P, _P, _I64, _I32, _P, _P, _P]
_lib.rebalance_ranks.argtypes = [_P, _P, _I32, _P, _I32, _I32, _P, _P, _P]
_lib.plan_dispatch_noalloc.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _I32, _P, _P, _P, _P,
                                       _P, _P, _P, _I64, _P, _P, _P, _P, _P, _P]
for _f in ("coact_count", "plan_dispatch", "dispatch_gather", "dispatch_gather_tma",
           "combine_scatter", "combine_rows", "dispatch_gather_backward",
           "combine_scatter_backward", "shuffle_reduce_scatter", "plan_dispatch_slots",
           "assign_replicas", "predict_home",
           "coact_place_correlated", "plan_dispatch_noalloc", "coact_compose_map", "plan_forward",
           "forward_gather", "forward_gather_tokens", "coact_rebalance_ranks",
           "coact_place_replicas", "dispatch_gather_peer",
           "combine_scatter_peer", "plan_row_meta", "gather_row_slots", "rebalance_ranks"):
    getattr(_lib, _f).restype = _I32

ABI_SYMBOLS = ("coact_strerror", "coact_abi_version", "coact_last_cuda_error", "coact_count", "plan_dispatch_workspace_bytes",
               "plan_dispatch", "dispatch_gather", "dispatch_gather_tma", "combine_scatter",
               "predict_home_workspace_bytes", "predict_home", "coact_place_correlated",
               "plan_dispatch_noalloc", "coact_compose_map", "plan_forward", "forward_gather",
               "coact_rebalance_ranks", "dispatch_gather_peer", "combine_scatter_peer",
               "combine_rows", "dispatch_gather_backward", "combine_scatter_backward",
               "shuffle_reduce_scatter", "plan_dispatch_slots", "assign_replicas",
               "forward_gather_tokens", "coact_place_replicas", "plan_row_meta",
               "gather_row_slots", "rebalance_ranks")
NOALLOC_MAX_TOKENS = 262144


class CoactError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {_lib.coact_strerror(status).decode()} (status {status})"
        self.cuda_error = _lib.coact_last_cuda_error() if status == ERR_CUDA else 0
        if self.cuda_error:
            msg += f"; cudaError_t {self.cuda_error}"
        super().__init__(msg)
        self.status = status


def abi_version() -> int:
    return _lib.coact_abi_version()


def strerror(status: int) -> str:
    return _lib.coact_strerror(status).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise CoactError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: Optional[torch.Tensor], name: str, dtype, shape=None, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _bits16(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensors are passed by bit pattern (uint16 in the ABI)."""
    if t.dtype != torch.bfloat16:
        raise ValueError(f"expected a bfloat16 tensor, got {t.dtype}")
    return t


# ----------------------------------------------------------------------------- entry points


def coact_count(ids: torch.Tensor, E: int, pair: torch.Tensor, loads: Optional[torch.Tensor] = None,
                ids2: Optional[torch.Tensor] = None, E2: Optional[int] = None,
                err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """pair[a,b] += tokens selecting both a and b (a != b); loads[e] += selections of e.
    Cross mode (ids2 given): pair[a,b] += slot pairs with ids[t,.] == a, ids2[t,.] == b."""
    N, k = ids.shape
    _need(ids, "ids", torch.int32)
    if ids2 is None:
        _need(pair, "pair", torch.int64, (E, E))
        k2, E2_ = 0, 0
    else:
        if E2 is None:
            raise ValueError("E2 is required with ids2")
        _need(ids2, "ids2", torch.int32)
        if ids2.shape[0] != N:
            raise ValueError("ids and ids2 must have the same number of tokens")
        _need(pair, "pair", torch.int64, (E, E2))
        k2, E2_ = ids2.shape[1], E2
    _need(loads, "loads", torch.int64, (E,), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.coact_count(_ptr(ids), N, k, E, _ptr(ids2), k2, E2_, _ptr(pair), _ptr(loads),
                            _ptr(err_flag), _stream(stream)), "coact_count")


def plan_workspace_bytes(N: int, k: int, E: int, R: int) -> int:
    return int(_lib.plan_dispatch_workspace_bytes(N, k, E, R))


@dataclasses.dataclass
class Plan:
    """Output buffers of plan_dispatch (torch CUDA tensors)."""
    rank_counts: torch.Tensor
    rank_offsets: torch.Tensor
    asg_offsets: torch.Tensor
    rank_mask: Optional[torch.Tensor]
    row_token: torch.Tensor
    row_kmask: torch.Tensor
    send_row: torch.Tensor
    comb_row: torch.Tensor
    stats: torch.Tensor
    src_dst: Optional[torch.Tensor]
    workspace: torch.Tensor

    @property
    def row_capacity(self) -> int:
        return self.row_token.shape[0]


def alloc_plan(N: int, k: int, E: int, R: int, device="cuda", row_capacity: Optional[int] = None,
               with_rank_mask: bool = True, with_src_dst: bool = True) -> Plan:
    """Allocates plan_dispatch's outputs and workspace.  row_capacity defaults to
    N*min(k, R), the size that can never overflow."""
    cap = N * min(k, R) if row_capacity is None else int(row_capacity)
    dev = torch.device(device)
    i32 = dict(dtype=torch.int32, device=dev)
    ws = torch.empty(max(plan_workspace_bytes(N, k, E, R), 16), dtype=torch.uint8, device=dev)
    return Plan(rank_counts=torch.empty(R, **i32), rank_offsets=torch.empty(R + 1, **i32),
                asg_offsets=torch.empty(R + 1, **i32),
                rank_mask=torch.empty(N, dtype=torch.int64, device=dev) if with_rank_mask else None,
                row_token=torch.empty(cap, **i32),
                row_kmask=torch.empty(cap, dtype=torch.uint8, device=dev),
                send_row=torch.empty((N, k), **i32), comb_row=torch.empty((N, k), **i32),
                stats=torch.empty(NUM_STATS, dtype=torch.int64, device=dev),
                src_dst=torch.empty((R, R), **i32) if with_src_dst else None, workspace=ws)


def plan_dispatch(ids: torch.Tensor, E: int, expert_rank: Optional[torch.Tensor], R: int,
                  plan: Plan, rank_node: Optional[torch.Tensor] = None, n_nodes: int = 1,
                  src_rank: Optional[torch.Tensor] = None,
                  err_flag: Optional[torch.Tensor] = None, stream=None,
                  slot_rank: Optional[torch.Tensor] = None) -> Plan:
    """Deduplicated dispatch layout into `plan`'s buffers (see include/coact.h).  With
    slot_rank (int32 [N, k], e.g. from assign_replicas) every slot goes to its own rank
    (plan_dispatch_slots) and expert_rank is not used."""
    N, k = ids.shape
    _need(ids, "ids", torch.int32)
    if slot_rank is None:
        _need(expert_rank, "expert_rank", torch.int32, (E,))
    else:
        _need(slot_rank, "slot_rank", torch.int32, (N, k))
    _need(rank_node, "rank_node", torch.int32, (R,), optional=True)
    _need(src_rank, "src_rank", torch.int32, (N,), optional=True)
    _need(plan.rank_counts, "rank_counts", torch.int32, (R,))
    _need(plan.rank_offsets, "rank_offsets", torch.int32, (R + 1,))
    _need(plan.asg_offsets, "asg_offsets", torch.int32, (R + 1,))
    _need(plan.rank_mask, "rank_mask", torch.int64, (N,), optional=True)
    _need(plan.row_token, "row_token", torch.int32)
    _need(plan.row_kmask, "row_kmask", torch.uint8, (plan.row_token.shape[0],))
    _need(plan.send_row, "send_row", torch.int32, (N, k))
    _need(plan.comb_row, "comb_row", torch.int32, (N, k))
    _need(plan.stats, "stats", torch.int64, (NUM_STATS,))
    _need(plan.src_dst, "src_dst", torch.int32, (R, R), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    ws = plan.workspace
    fn = _lib.plan_dispatch if slot_rank is None else _lib.plan_dispatch_slots
    _check(fn(
        _ptr(ids), N, k, E, _ptr(expert_rank if slot_rank is None else slot_rank), R,
        _ptr(rank_node), n_nodes, _ptr(src_rank),
        _ptr(plan.rank_counts), _ptr(plan.rank_offsets), _ptr(plan.asg_offsets),
        _ptr(plan.rank_mask), _ptr(plan.row_token), _ptr(plan.row_kmask), plan.row_capacity,
        _ptr(plan.send_row), _ptr(plan.comb_row), _ptr(plan.stats), _ptr(plan.src_dst),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(err_flag), _stream(stream)),
        "plan_dispatch" if slot_rank is None else "plan_dispatch_slots")
    return plan


def assign_replicas(ids: torch.Tensor, E: int, rep_rank: torch.Tensor, n_rep: torch.Tensor, R: int,
                    slot_rank: torch.Tensor, rank_node: Optional[torch.Tensor] = None,
                    n_nodes: int = 1, src_rank: Optional[torch.Tensor] = None,
                    err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The replica serving each (token, slot) into slot_rank (int32 [N, k]); rep_rank:
    int32 [E, max_rep] replica ranks, n_rep: int32 [E] replicas per expert."""
    N, k = ids.shape
    _need(ids, "ids", torch.int32)
    _need(rep_rank, "rep_rank", torch.int32)
    if rep_rank.dim() != 2 or rep_rank.shape[0] != E:
        raise ValueError("rep_rank must be [E, max_rep]")
    _need(n_rep, "n_rep", torch.int32, (E,))
    _need(slot_rank, "slot_rank", torch.int32, (N, k))
    _need(rank_node, "rank_node", torch.int32, (R,), optional=True)
    _need(src_rank, "src_rank", torch.int32, (N,), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.assign_replicas(_ptr(ids), N, k, E, _ptr(rep_rank), rep_rank.shape[1], _ptr(n_rep),
                                R, _ptr(rank_node), n_nodes, _ptr(src_rank), _ptr(slot_rank),
                                _ptr(err_flag), _stream(stream)), "assign_replicas")
    return slot_rank


def dispatch_gather(x: torch.Tensor, send_row: torch.Tensor, send: torch.Tensor,
                    err_flag: Optional[torch.Tensor] = None, stream=None,
                    tma: bool = False) -> torch.Tensor:
    """send[send_row[t, j]] = x[t] for every send_row entry >= 0 (bf16 rows).
    tma=True uses the TMA bulk-copy implementation (dispatch_gather_tma)."""
    N, H = x.shape
    _need(_bits16(x), "x", torch.bfloat16)
    _need(send_row, "send_row", torch.int32)
    if send_row.shape[0] != N:
        raise ValueError("send_row must have one row per token")
    _need(_bits16(send), "send", torch.bfloat16)
    if send.shape[1] != H:
        raise ValueError("send rows must have x's hidden size")
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    fn = _lib.dispatch_gather_tma if tma else _lib.dispatch_gather
    _check(fn(_ptr(x), N, H, _ptr(send_row), send_row.shape[1], _ptr(send), send.shape[0],
              _ptr(err_flag), _stream(stream)), "dispatch_gather_tma" if tma else "dispatch_gather")
    return send


def combine_scatter(y: torch.Tensor, gates: torch.Tensor, comb_row: torch.Tensor,
                    out: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """out[t] = sum_j gates[t,j] * y[comb_row[t,j]] (fp32 fma chain in ascending j;
    out is bf16 or fp32)."""
    N, k = gates.shape
    _need(_bits16(y), "y", torch.bfloat16)
    H = y.shape[1]
    _need(gates, "gates", torch.float32)
    _need(comb_row, "comb_row", torch.int32, (N, k))
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (N, H))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.combine_scatter(_ptr(y), y.shape[0], _ptr(gates), _ptr(comb_row), N, k, H,
                                _ptr(out), 1 if out.dtype == torch.float32 else 0,
                                _ptr(err_flag), _stream(stream)), "combine_scatter")
    return out


def _out_dtype(out: torch.Tensor) -> int:
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bfloat16 or float32")
    return 1 if out.dtype == torch.float32 else 0


def combine_rows(y: torch.Tensor, gates: torch.Tensor, comb_row: torch.Tensor,
                 row_token: torch.Tensor, row_kmask: torch.Tensor, out: torch.Tensor,
                 n_units: Optional[int] = None, unit_count: Optional[torch.Tensor] = None,
                 err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[u] = sum over the slots j of row_kmask[u] (ascending) of
    gates[t,j] * y[comb_row[t,j]], t = row_token[u] -- over the plan's send rows, the
    partial rows of the pre-reduced reverse path.  n_units defaults to out.shape[0];
    unit_count: optional device int32 [1] further bounding it (e.g. the plan's
    rank_offsets[R:], i.e. D), read by the kernel."""
    N, k = gates.shape
    _need(_bits16(y), "y", torch.bfloat16)
    H = y.shape[1]
    n = out.shape[0] if n_units is None else int(n_units)
    _need(gates, "gates", torch.float32)
    _need(comb_row, "comb_row", torch.int32, (N, k))
    _need(row_token, "row_token", torch.int32)
    _need(row_kmask, "row_kmask", torch.uint8)
    if row_token.numel() < n or row_kmask.numel() < n or out.shape[0] < n or out.shape[1] != H:
        raise ValueError("row_token, row_kmask and out need n_units rows")
    _need(out, "out", out.dtype)
    _need(unit_count, "unit_count", torch.int32, (1,), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.combine_rows(_ptr(y), y.shape[0], _ptr(gates), _ptr(comb_row), N, k, _ptr(row_token),
                             _ptr(row_kmask), n, _ptr(unit_count), H, _ptr(out), _out_dtype(out),
                             _ptr(err_flag), _stream(stream)), "combine_rows")
    return out


def dispatch_gather_backward(grad_send: torch.Tensor, send_row: torch.Tensor, grad_x: torch.Tensor,
                             err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grad_x[t] = sum over the token's send rows (send_row[t,j] >= 0, ascending j) of
    grad_send[send_row[t,j]] (fp32 add chain; grad_x bf16 or fp32)."""
    N, k = send_row.shape
    _need(_bits16(grad_send), "grad_send", torch.bfloat16)
    H = grad_send.shape[1]
    _need(send_row, "send_row", torch.int32, (N, k))
    _need(grad_x, "grad_x", grad_x.dtype, (N, H))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.dispatch_gather_backward(_ptr(grad_send), grad_send.shape[0], _ptr(send_row), N, k, H,
                                         _ptr(grad_x), _out_dtype(grad_x), _ptr(err_flag),
                                         _stream(stream)), "dispatch_gather_backward")
    return grad_x


def combine_scatter_backward(y: torch.Tensor, gates: torch.Tensor, comb_row: torch.Tensor,
                             grad_out: torch.Tensor, grad_y: torch.Tensor, grad_gates: torch.Tensor,
                             row_token: Optional[torch.Tensor] = None,
                             row_kmask: Optional[torch.Tensor] = None,
                             unit_count: Optional[torch.Tensor] = None,
                             err_flag: Optional[torch.Tensor] = None, stream=None):
    """Gradients of the combine: grad_y[comb_row[t,j]] = bf16(gates[t,j] * grad_out[u]) and
    grad_gates[t,j] = <grad_out[u], y[comb_row[t,j]]>, u = token t (row_token None) or the
    units row_token / row_kmask with one grad_out row each (optionally bounded by the
    device int32 [1] unit_count)."""
    N, k = gates.shape
    _need(_bits16(y), "y", torch.bfloat16)
    H = y.shape[1]
    _need(gates, "gates", torch.float32)
    _need(comb_row, "comb_row", torch.int32, (N, k))
    n = N
    if row_token is not None:
        n = grad_out.shape[0]
        _need(row_token, "row_token", torch.int32)
        _need(row_kmask, "row_kmask", torch.uint8)
        if row_token.numel() < n or row_kmask.numel() < n:
            raise ValueError("row_token and row_kmask need one entry per grad_out row")
    _need(_bits16(grad_out), "grad_out", torch.bfloat16, (n, H))
    _need(_bits16(grad_y), "grad_y", torch.bfloat16, tuple(y.shape))
    _need(grad_gates, "grad_gates", torch.float32, (N, k))
    _need(unit_count, "unit_count", torch.int32, (1,), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.combine_scatter_backward(_ptr(y), y.shape[0], _ptr(gates), _ptr(comb_row), N, k,
                                         _ptr(row_token), _ptr(row_kmask), n, _ptr(unit_count),
                                         _ptr(grad_out), H,
                                         _ptr(grad_y), _ptr(grad_gates), _ptr(err_flag),
                                         _stream(stream)), "combine_scatter_backward")
    return grad_y, grad_gates


def shuffle_plan(home: torch.Tensor, R: int, plan: Optional["Plan"] = None,
                 err_flag: Optional[torch.Tensor] = None, stream=None) -> "Plan":
    """The token shuffle's permutation: plan_dispatch of every token to its predicted home
    rank alone (ids = home [N, 1], E = R, identity expert -> rank map).  plan.row_token
    lists the tokens grouped by home rank in ascending token order; rank r's output rows
    are [rank_offsets[r], rank_offsets[r+1])."""
    if R < 1:
        raise ValueError("token shuffling needs at least one rank")
    _need(home, "home", torch.int32)
    N = home.shape[0]
    E = max(R, 2)                  # the planner takes E >= 2; with one rank both map to it
    if plan is None:
        plan = alloc_plan(N, 1, E, R, home.device, with_rank_mask=False, with_src_dst=False)
    ident = torch.arange(E, dtype=torch.int32, device=home.device).clamp_(max=R - 1)
    return plan_dispatch(home.view(N, 1), E, ident, R, plan, err_flag=err_flag, stream=stream)


def shuffle_reduce_scatter(part_bases: torch.Tensor, N: int, row_token: torch.Tensor,
                           out: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """out[i] = sum over q of part_q[row_token[i]] (fp32 adds in rank order); part_bases:
    device int64 [P] addresses of the P bf16 [N, H] partial outputs; H = out.shape[1]."""
    _need(part_bases, "part_bases", torch.int64)
    P = part_bases.shape[0]
    _need(row_token, "row_token", torch.int32)
    n_out, H = out.shape
    if row_token.numel() < n_out:
        raise ValueError("row_token needs one entry per output row")
    _need(out, "out", out.dtype)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.shuffle_reduce_scatter(_ptr(part_bases), P, N, H, _ptr(row_token), n_out, _ptr(out),
                                       _out_dtype(out), _ptr(err_flag), _stream(stream)),
           "shuffle_reduce_scatter")
    return out


def predict_workspace_bytes(E1: int, R: int) -> int:
    return int(_lib.predict_home_workspace_bytes(E1, R))


def predict_home(ids1: torch.Tensor, E1: int, C12: torch.Tensor, expert_rank2: torch.Tensor, R: int,
                 home: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                 err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """home[t] = argmax_r sum_j sum_{b on r} C12[ids1[t,j], b] (ties -> lowest r)."""
    N, k1 = ids1.shape
    _need(ids1, "ids1", torch.int32)
    _need(C12, "C12", torch.int64)
    E2 = C12.shape[1]
    if C12.shape[0] != E1:
        raise ValueError("C12 must be [E1, E2]")
    _need(expert_rank2, "expert_rank2", torch.int32, (E2,))
    _need(home, "home", torch.int32, (N,))
    if workspace is None:
        workspace = torch.empty(max(predict_workspace_bytes(E1, R), 16), dtype=torch.uint8,
                                device=ids1.device)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.predict_home(_ptr(ids1), N, k1, E1, _ptr(C12), E2, _ptr(expert_rank2), R,
                             _ptr(home), _ptr(workspace), workspace.numel(), _ptr(err_flag),
                             _stream(stream)), "predict_home")
    return home


def coact_place_correlated(pair, R: int):
    """Correlated expert placement from co-activation counts (host computation in the
    library).  `pair`: int64 [E, E] counts (any device; copied to host).  Returns an
    int32 CPU tensor expert -> rank with E/R experts per rank."""
    p = pair.detach().to("cpu", torch.int64).contiguous()
    E = p.shape[0]
    if tuple(p.shape) != (E, E):
        raise ValueError("pair must be [E, E]")
    out = torch.empty(E, dtype=torch.int32)
    _check(_lib.coact_place_correlated(_ptr(p), E, R, _ptr(out)), "coact_place_correlated")
    return out


def plan_dispatch_noalloc(ids: torch.Tensor, E: int, expert_rank: torch.Tensor, R: int, plan: Plan,
                          rank_node: Optional[torch.Tensor] = None, n_nodes: int = 1,
                          src_rank: Optional[torch.Tensor] = None,
                          err_flag: Optional[torch.Tensor] = None, stream=None) -> Plan:
    """plan_dispatch for callers that cannot allocate device memory (a runtime that owns
    all device memory through its own pool or fixed memory plan, or a caller that cannot
    afford cudaMalloc's device-wide synchronisation): the library's own file-scope device
    scratch replaces the workspace (plan.workspace is not used).  Batches of at most
    NOALLOC_MAX_TOKENS tokens; calls that overlap on the GPU share that scratch and race,
    so keep them on one stream.  The first call on a device, and the first after a device
    reset, must come before any stream capture (it looks up the scratch address)."""
    N, k = ids.shape
    if N > NOALLOC_MAX_TOKENS:
        raise ValueError(f"plan_dispatch_noalloc handles at most {NOALLOC_MAX_TOKENS} tokens "
                         f"(got {N}); use plan_dispatch with a workspace")
    _need(ids, "ids", torch.int32)
    _need(expert_rank, "expert_rank", torch.int32, (E,))
    _need(rank_node, "rank_node", torch.int32, (R,), optional=True)
    _need(src_rank, "src_rank", torch.int32, (N,), optional=True)
    _need(plan.rank_counts, "rank_counts", torch.int32, (R,))
    _need(plan.rank_offsets, "rank_offsets", torch.int32, (R + 1,))
    _need(plan.asg_offsets, "asg_offsets", torch.int32, (R + 1,))
    _need(plan.rank_mask, "rank_mask", torch.int64, (N,), optional=True)
    _need(plan.row_token, "row_token", torch.int32)
    _need(plan.row_kmask, "row_kmask", torch.uint8, (plan.row_token.shape[0],))
    _need(plan.send_row, "send_row", torch.int32, (N, k))
    _need(plan.comb_row, "comb_row", torch.int32, (N, k))
    _need(plan.stats, "stats", torch.int64, (NUM_STATS,))
    _need(plan.src_dst, "src_dst", torch.int32, (R, R), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.plan_dispatch_noalloc(
        _ptr(ids), N, k, E, _ptr(expert_rank), R, _ptr(rank_node), n_nodes, _ptr(src_rank),
        _ptr(plan.rank_counts), _ptr(plan.rank_offsets), _ptr(plan.asg_offsets),
        _ptr(plan.rank_mask), _ptr(plan.row_token), _ptr(plan.row_kmask), plan.row_capacity,
        _ptr(plan.send_row), _ptr(plan.comb_row), _ptr(plan.stats), _ptr(plan.src_dst),
        _ptr(err_flag), _stream(stream)), "plan_dispatch_noalloc")
    return plan


# ----------------------------------------------------------------------------- EP row metadata


def plan_row_meta(plan: "Plan", ids: Optional[torch.Tensor] = None,
                  gates: Optional[torch.Tensor] = None, slot_base: Optional[torch.Tensor] = None,
                  experts: bool = True, with_slots: bool = True,
                  err_flag: Optional[torch.Tensor] = None, stream=None):
    """Per send row of `plan` (rows < rank_offsets[R], read on the device), one entry per
    slot: the expert id (ids given), the gate (gates given) and the expert-output position
    comb_row + slot_base[rank of the row] (with_slots); -1 / 0 / -1 where the row does not
    serve the slot.  Returns (row_experts int32, row_gates fp32, row_slots int32), each
    [row_capacity, k] or None; rows past D are left uninitialised."""
    N, k = plan.send_row.shape
    R = plan.rank_counts.shape[0]
    cap = plan.row_capacity
    dev = plan.send_row.device
    _need(ids, "ids", torch.int32, (N, k), optional=True)
    _need(gates, "gates", torch.float32, (N, k), optional=True)
    _need(slot_base, "slot_base", torch.int32, (R,), optional=True)
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    ex = torch.empty((cap, k), dtype=torch.int32, device=dev) if (experts and ids is not None) else None
    gt = torch.empty((cap, k), dtype=torch.float32, device=dev) if gates is not None else None
    sl = torch.empty((cap, k), dtype=torch.int32, device=dev) if with_slots else None
    _check(_lib.plan_row_meta(_ptr(plan.row_token), _ptr(plan.row_kmask), cap,
                              _ptr(plan.rank_offsets), R, _ptr(ids), _ptr(gates),
                              _ptr(plan.comb_row), N, k, _ptr(slot_base), _ptr(ex), _ptr(gt),
                              _ptr(sl), _ptr(err_flag), _stream(stream)), "plan_row_meta")
    return ex, gt, sl


def gather_row_slots(vals: torch.Tensor, send_row: torch.Tensor, row_kmask: torch.Tensor,
                     out: Optional[torch.Tensor] = None, err_flag: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """out[t, j] = vals[d, j] for the send row d of token t that holds slot j (0 where
    none does); vals fp32 [n_rows, k] in send-row order."""
    N, k = send_row.shape
    _need(vals, "vals", torch.float32)
    if vals.dim() != 2 or vals.shape[1] != k:
        raise ValueError("vals must be [n_rows, k]")
    _need(send_row, "send_row", torch.int32, (N, k))
    _need(row_kmask, "row_kmask", torch.uint8)
    if row_kmask.numel() < vals.shape[0]:
        raise ValueError("row_kmask needs an entry per row of vals")
    if out is None:
        out = torch.empty((N, k), dtype=torch.float32, device=send_row.device)
    _need(out, "out", torch.float32, (N, k))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.gather_row_slots(_ptr(vals), vals.shape[0], _ptr(send_row), _ptr(row_kmask), N, k,
                                 _ptr(out), _ptr(err_flag), _stream(stream)), "gather_row_slots")
    return out


# ----------------------------------------------------------------------------- two-hop dispatch


def coact_compose_map(a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor] = None,
                      err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[i] = b[a[i]] on the device (int32)."""
    _need(a, "a", torch.int32)
    _need(b, "b", torch.int32)
    if out is None:
        out = torch.empty_like(a)
    _need(out, "out", torch.int32, tuple(a.shape))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.coact_compose_map(_ptr(a), a.numel(), _ptr(b), b.numel(), _ptr(out),
                                  _ptr(err_flag), _stream(stream)), "coact_compose_map")
    return out


def plan_forward(ids: torch.Tensor, E: int, expert_rank: torch.Tensor, R: int, rank_plan: Plan,
                 node_plan: Plan, fwd_src: torch.Tensor, rank_node: Optional[torch.Tensor] = None,
                 n_nodes: int = 1, err_flag: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """fwd_src[d] = the node-level (hop-1) row feeding rank-level row d; -1 past D."""
    N, k = ids.shape
    _need(ids, "ids", torch.int32)
    _need(expert_rank, "expert_rank", torch.int32, (E,))
    _need(rank_node, "rank_node", torch.int32, (R,), optional=True)
    _need(fwd_src, "fwd_src", torch.int32, (rank_plan.row_capacity,))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.plan_forward(_ptr(ids), N, k, E, _ptr(expert_rank), R, _ptr(rank_node), n_nodes,
                             _ptr(rank_plan.send_row), _ptr(rank_plan.rank_offsets),
                             _ptr(node_plan.send_row), _ptr(fwd_src), rank_plan.row_capacity,
                             _ptr(err_flag), _stream(stream)), "plan_forward")
    return fwd_src


def forward_gather(src: torch.Tensor, fwd_src: torch.Tensor, dst: torch.Tensor,
                   err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dst[d] = src[fwd_src[d]] for fwd_src[d] >= 0 (bf16 rows)."""
    _need(_bits16(src), "src", torch.bfloat16)
    _need(_bits16(dst), "dst", torch.bfloat16)
    if src.shape[1] != dst.shape[1]:
        raise ValueError("src and dst rows must have the same width")
    _need(fwd_src, "fwd_src", torch.int32, (dst.shape[0],))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.forward_gather(_ptr(src), src.shape[0], src.shape[1], _ptr(fwd_src), dst.shape[0],
                               _ptr(dst), _ptr(err_flag), _stream(stream)), "forward_gather")
    return dst


def forward_gather_tokens(src: torch.Tensor, send_row: torch.Tensor, fwd_src: torch.Tensor,
                          dst: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """forward_gather in token order: each hop-1 row read once and written to every rank
    row it feeds (send_row: the rank plan's [N, k])."""
    _need(_bits16(src), "src", torch.bfloat16)
    _need(_bits16(dst), "dst", torch.bfloat16)
    if src.shape[1] != dst.shape[1]:
        raise ValueError("src and dst rows must have the same width")
    _need(send_row, "send_row", torch.int32)
    N, k = send_row.shape
    _need(fwd_src, "fwd_src", torch.int32, (dst.shape[0],))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.forward_gather_tokens(_ptr(src), src.shape[0], src.shape[1], _ptr(send_row), N, k,
                                      _ptr(fwd_src), dst.shape[0], _ptr(dst), _ptr(err_flag),
                                      _stream(stream)), "forward_gather_tokens")
    return dst


@dataclasses.dataclass
class TwoHopPlan:
    """Plans of a two-hop dispatch: node level (hop 1), rank level (hop 2) and the map
    between them.  expert_node / src_node are the device maps the node plan used;
    node_ids (0..n_nodes-1) and contiguous_src (floor(t*R/N), the default home ranks)
    are constant inputs made once here."""
    node: Plan
    rank: Plan
    fwd_src: torch.Tensor
    expert_node: torch.Tensor
    src_node: torch.Tensor
    node_ids: torch.Tensor
    contiguous_src: torch.Tensor


def alloc_two_hop(N: int, k: int, E: int, R: int, n_nodes: int, device="cuda") -> TwoHopPlan:
    dev = torch.device(device)
    rank = alloc_plan(N, k, E, R, dev)
    t = torch.arange(N, dtype=torch.int64, device=dev)
    return TwoHopPlan(node=alloc_plan(N, k, E, n_nodes, dev), rank=rank,
                      fwd_src=torch.empty(rank.row_capacity, dtype=torch.int32, device=dev),
                      expert_node=torch.empty(E, dtype=torch.int32, device=dev),
                      src_node=torch.empty(N, dtype=torch.int32, device=dev),
                      node_ids=torch.arange(n_nodes, dtype=torch.int32, device=dev),
                      contiguous_src=(t * R // max(N, 1)).to(torch.int32))


def plan_two_hop(ids: torch.Tensor, E: int, expert_rank: torch.Tensor, R: int,
                 rank_node: torch.Tensor, n_nodes: int, th: TwoHopPlan,
                 src_rank: Optional[torch.Tensor] = None, err_flag: Optional[torch.Tensor] = None,
                 stream=None) -> TwoHopPlan:
    """Both plans and the forward map, all in library kernels: expert -> node and token
    -> home node maps (coact_compose_map), the node-level plan_dispatch, the rank-level
    plan_dispatch and plan_forward."""
    N = ids.shape[0]
    coact_compose_map(expert_rank, rank_node, th.expert_node, err_flag, stream)
    src = th.contiguous_src if src_rank is None else src_rank
    if N:
        coact_compose_map(src, rank_node, th.src_node, err_flag, stream)
    plan_dispatch(ids, E, th.expert_node, n_nodes, th.node, rank_node=th.node_ids,
                  n_nodes=n_nodes, src_rank=th.src_node if N else None, err_flag=err_flag,
                  stream=stream)
    plan_dispatch(ids, E, expert_rank, R, th.rank, rank_node=rank_node, n_nodes=n_nodes,
                  src_rank=src_rank, err_flag=err_flag, stream=stream)
    plan_forward(ids, E, expert_rank, R, th.rank, th.node, th.fwd_src, rank_node=rank_node,
                 n_nodes=n_nodes, err_flag=err_flag, stream=stream)
    return th


def coact_rebalance_ranks(loads, expert_node, rank_node):
    """Cobalt's intra-node rebalancing (host computation in the library): each node's
    experts, heaviest first, to the least-loaded rank of that node with a free slot.
    Returns an int32 CPU tensor expert -> rank."""
    ld = loads.detach().to("cpu", torch.int64).contiguous()
    en = expert_node.detach().to("cpu", torch.int32).contiguous()
    rn = rank_node.detach().to("cpu", torch.int32).contiguous()
    out = torch.empty(ld.shape[0], dtype=torch.int32)
    _check(_lib.coact_rebalance_ranks(_ptr(ld), _ptr(en), ld.shape[0], _ptr(rn), rn.shape[0],
                                      _ptr(out)), "coact_rebalance_ranks")
    return out


def rebalance_ranks(loads: torch.Tensor, expert_node: torch.Tensor, rank_node: torch.Tensor,
                    n_nodes: int, out: Optional[torch.Tensor] = None,
                    err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """coact_rebalance_ranks on the device (Cobalt's per-step intra-node adjustment): the
    node's experts by load descending, each to the node's least loaded rank with a free
    slot.  loads: device int64 [E]; expert_node: int32 [E]; rank_node: int32 [R].
    Returns the int32 [E] expert -> rank map (-1 and a flag where the layout does not
    fit)."""
    E, R = loads.shape[0], rank_node.shape[0]
    _need(loads, "loads", torch.int64, (E,))
    _need(expert_node, "expert_node", torch.int32, (E,))
    _need(rank_node, "rank_node", torch.int32, (R,))
    if out is None:
        out = torch.empty(E, dtype=torch.int32, device=loads.device)
    _need(out, "out", torch.int32, (E,))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.rebalance_ranks(_ptr(loads), _ptr(expert_node), E, _ptr(rank_node), R, n_nodes,
                                _ptr(out), _ptr(err_flag), _stream(stream)), "rebalance_ranks")
    return out


def coact_place_two_stage(pair, loads, rank_node, n_nodes: int):
    """Cobalt's two-stage layout: co-activated experts co-located per node
    (coact_place_correlated at node granularity), then per-rank loads balanced inside
    each node (coact_rebalance_ranks).  Returns expert -> rank (int32 CPU tensor)."""
    expert_node = coact_place_correlated(pair, n_nodes)
    return coact_rebalance_ranks(loads, expert_node, rank_node)


# ----------------------------------------------------------------------------- across GPUs


def dispatch_gather_peer(x: torch.Tensor, send_row: torch.Tensor, rank_offsets: torch.Tensor,
                         dst_bases: torch.Tensor, dst_row_offset: torch.Tensor,
                         dst_capacity: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                         stream=None) -> None:
    """Rows of rank r's segment of this source's plan go straight into the destination
    buffer dst_bases[r] (a device address, e.g. a peer GPU's symmetric buffer) at
    dst_row_offset[r] + (row - rank_offsets[r])."""
    N, H = x.shape
    R = rank_offsets.shape[0] - 1
    _need(_bits16(x), "x", torch.bfloat16)
    _need(send_row, "send_row", torch.int32)
    _need(rank_offsets, "rank_offsets", torch.int32)
    _need(dst_bases, "dst_bases", torch.int64, (R,))
    _need(dst_row_offset, "dst_row_offset", torch.int32, (R,))
    _need(dst_capacity, "dst_capacity", torch.int32, (R,))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.dispatch_gather_peer(_ptr(x), N, H, _ptr(send_row), send_row.shape[1],
                                     _ptr(rank_offsets), R, _ptr(dst_bases), _ptr(dst_row_offset),
                                     _ptr(dst_capacity), _ptr(err_flag), _stream(stream)),
           "dispatch_gather_peer")


def combine_scatter_peer(y_bases: torch.Tensor, y_row_offset: torch.Tensor,
                         y_capacity: torch.Tensor, asg_offsets: torch.Tensor,
                         gates: Optional[torch.Tensor], comb_row: torch.Tensor, out: torch.Tensor,
                         H: int, err_flag: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """combine_scatter with each expert output read from the rank that computed it.  With
    gates None (unit weights), send_row and rank_offsets: the transposed dispatch reading
    each row from the rank that holds it."""
    N, k = comb_row.shape
    R = asg_offsets.shape[0] - 1
    _need(y_bases, "y_bases", torch.int64, (R,))
    _need(y_row_offset, "y_row_offset", torch.int32, (R,))
    _need(y_capacity, "y_capacity", torch.int32, (R,))
    _need(asg_offsets, "asg_offsets", torch.int32)
    _need(gates, "gates", torch.float32, (N, k), optional=True)
    _need(comb_row, "comb_row", torch.int32, (N, k))
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bfloat16 or float32")
    _need(out, "out", out.dtype, (N, H))
    _need(err_flag, "err_flag", torch.int32, (1,), optional=True)
    _check(_lib.combine_scatter_peer(_ptr(y_bases), _ptr(y_row_offset), _ptr(y_capacity),
                                     _ptr(asg_offsets), R, _ptr(gates), _ptr(comb_row), N, k, H,
                                     _ptr(out), 1 if out.dtype == torch.float32 else 0,
                                     _ptr(err_flag), _stream(stream)), "combine_scatter_peer")
    return out


def coact_place_replicas(pair: torch.Tensor, loads: torch.Tensor, expert_rank: torch.Tensor,
                         rank_node: torch.Tensor, budget: int, max_rep: int = 2):
    """Replica layout from co-activation counts and loads (host code; CPU tensors or
    copies of device ones): (rep_rank int32 [E, max_rep] with -1 padding, n_rep int32
    [E], replicas added)."""
    pr = pair.detach().to("cpu", torch.int64).contiguous()
    ld = loads.detach().to("cpu", torch.int64).contiguous()
    er = expert_rank.detach().to("cpu", torch.int32).contiguous()
    rn = rank_node.detach().to("cpu", torch.int32).contiguous()
    E, R = ld.shape[0], rn.shape[0]
    if pr.shape != (E, E) or er.shape != (E,):
        raise ValueError("pair must be [E, E] and expert_rank [E]")
    rep = torch.empty((E, max_rep), dtype=torch.int32)
    nrep = torch.empty(E, dtype=torch.int32)
    added = _lib.coact_place_replicas(pr.data_ptr(), ld.data_ptr(), er.data_ptr(), E, rn.data_ptr(),
                                      R, budget, max_rep, rep.data_ptr(), nrep.data_ptr())
    if added < 0:
        raise CoactError(added, "coact_place_replicas")
    return rep, nrep, added
