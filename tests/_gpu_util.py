"""Helpers for the GPU parity tests: move generated workloads to the device, run the
library's path, and compare with the oracle (bit-exact integers and rows; combine
within the stated floating-point tolerance)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workload

DEV = torch.device("cuda:0")
X_STREAM, Y_STREAM = 1, 2       # fill_bf16 streams of the hidden rows and expert outputs


def cuda(a, dtype=None):
    """numpy array -> device tensor (dtype: an optional numpy dtype to convert to first)."""
    a = np.asarray(a) if dtype is None else np.asarray(a, dtype=dtype)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def run_plan(coact, r, E=None, expert_rank=None, R=None, rank_node=None, n_nodes=None,
             src_rank=None, row_capacity=None, sentinel=True):
    """GPU plan for routing r; returns (plan, err_flag) with buffers on the device."""
    cfg = r.cfg
    E = cfg.E if E is None else E
    R = cfg.R if R is None else R
    er = r.expert_rank if expert_rank is None else expert_rank
    rn = r.rank_node if rank_node is None else rank_node
    nn = cfg.n_nodes if n_nodes is None else n_nodes
    N, k = r.ids.shape
    plan = coact.alloc_plan(N, k, E, R, DEV, row_capacity=row_capacity)
    if sentinel:   # detect writes outside the documented ranges
        plan.row_token.fill_(-7)
        plan.row_kmask.fill_(0xEE)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    coact.plan_dispatch(cuda(r.ids), E, cuda(er, np.int32), R, plan,
                        rank_node=None if rn is None else cuda(rn, np.int32), n_nodes=nn,
                        src_rank=None if src_rank is None else cuda(src_rank, np.int32),
                        err_flag=err)
    torch.cuda.synchronize()
    return plan, err


def plan_to_host(plan) -> dict:
    out = {k: getattr(plan, k).cpu().numpy() for k in
           ("rank_counts", "rank_offsets", "asg_offsets", "row_token", "row_kmask", "send_row",
            "comb_row", "stats")}
    if plan.src_dst is not None:
        out["src_dst"] = plan.src_dst.cpu().numpy()
    if plan.rank_mask is not None:
        out["rank_mask"] = plan.rank_mask.cpu().numpy().view(np.uint64)
    return out


def assert_plan_equal(g: dict, o: dict, sentinel=True):
    D = int(o["rank_offsets"][-1])
    for key in ("rank_counts", "rank_offsets", "asg_offsets", "send_row", "comb_row", "stats"):
        assert np.array_equal(g[key], o[key]), key
    if "src_dst" in g:
        assert np.array_equal(g["src_dst"], o["src_dst"]), "src_dst"
    if "rank_mask" in g:
        assert np.array_equal(g["rank_mask"], o["rank_mask"]), "rank_mask"
    cap = len(o["row_token"])
    n = min(D, cap)
    assert np.array_equal(g["row_token"][:n], o["row_token"][:n]), "row_token"
    assert np.array_equal(g["row_kmask"][:n], o["row_kmask"][:n]), "row_kmask"
    if sentinel and n < len(g["row_token"]):
        assert (g["row_token"][n:] == -7).all(), "row_token written beyond D"
        assert (g["row_kmask"][n:] == 0xEE).all(), "row_kmask written beyond D"


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits); min normal spacing at 0."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check_combine(out_gpu: torch.Tensor, y_bits: np.ndarray, gates: np.ndarray,
                  comb_row: np.ndarray, tokens=None):
    """out_gpu rows (all, or `tokens`) against the oracle.  y_bits holds the rows that
    comb_row (already restricted to `tokens`) indexes."""
    got = out_gpu if tokens is None else out_gpu[torch.as_tensor(tokens, device=out_gpu.device)]
    got = got.cpu().numpy() if got.dtype == torch.float32 else host_bits(got)
    check_combine_host(got, y_bits, gates, comb_row)


def check_combine_host(got: np.ndarray, y_bits: np.ndarray, gates: np.ndarray,
                       comb_row: np.ndarray):
    """Combined rows already on the host (float32, or uint16 bf16 bit patterns) against
    the oracle.

    Tolerance (stated for floating point): fp32 output within 1e-5 of the magnitude
    sum_j |g_j y_j| of the float64 reference (fp32 accumulation error is defined relative
    to that scale: k fma roundings of 2^-24 each), and bit-identical to the fixed-order
    fp32 fma chain; bf16 output within 1 bf16 ulp of the float64 reference (+ the same
    fp32 term) and bit-identical to the chain rounded to nearest-even."""
    ref64 = oracle.combine_f64(y_bits, gates, comb_row)
    chain = oracle.combine_f32chain(y_bits, gates, comb_row)
    yf = workload.bf16_bits_to_float(y_bits).astype(np.float64)
    mag = np.zeros_like(ref64)
    for j in range(gates.shape[1]):
        valid = (comb_row[:, j] >= 0) & (comb_row[:, j] < y_bits.shape[0])
        mag[valid] += np.abs(gates[valid, j, None].astype(np.float64) * yf[comb_row[valid, j]])
    if got.dtype == np.float32:
        assert (np.abs(got.astype(np.float64) - ref64) <= 1e-5 * mag + 1e-30).all()
        assert np.array_equal(got.view(np.uint32), chain.view(np.uint32))
    else:
        gf = workload.bf16_bits_to_float(got).astype(np.float64)
        assert (np.abs(gf - ref64) <= ulp_bf16(ref64) + 1e-5 * mag).all()
        assert np.array_equal(got, oracle.bf16_rne(chain))


def _first_bad_row(got: np.ndarray, want: np.ndarray) -> int:
    return int(np.nonzero((got != want).reshape(len(got), -1).any(axis=1))[0][0])


def check_gather_complete(send: torch.Tensor, x_bits: np.ndarray, row_token: np.ndarray,
                          D: int, chunk: int = 1 << 15):
    """Every one of the D gathered rows against the oracle's gather of the host copy of x,
    streamed in chunks of rows (no sampling)."""
    for d0 in range(0, D, chunk):
        d1 = min(D, d0 + chunk)
        got = host_bits(send[d0:d1])
        want = oracle.gather(x_bits, row_token[d0:d1], d1 - d0)
        if not np.array_equal(got, want):
            raise AssertionError(f"gathered row {d0 + _first_bad_row(got, want)} differs")


def for_chunks(n: int, chunk: int, prepare, workers: int = 0):
    """Runs a check over [0, n) in chunks: prepare(c0, c1) does the device work in this
    thread (selecting and copying the chunk's rows to the host) and returns a callable
    that checks them on a worker thread (the oracle's C calls release the GIL).  At most
    2 x workers chunks are in flight, which bounds host memory."""
    import concurrent.futures as cf
    import os
    workers = workers or max(1, min(16, os.cpu_count() or 1))
    pending = []
    with cf.ThreadPoolExecutor(workers) as ex:
        for c0 in range(0, n, chunk):
            pending.append(ex.submit(prepare(c0, min(n, c0 + chunk))))
            if len(pending) >= 2 * workers:
                pending.pop(0).result()
        for f in pending:
            f.result()


def rows_of(t: torch.Tensor, idx: np.ndarray) -> np.ndarray:
    """Host bf16 bits of the device rows t[idx] (idx: any shape of non-negative ints)."""
    return host_bits(t.index_select(0, torch.as_tensor(np.ravel(idx).astype(np.int64),
                                                       device=t.device)))


def check_combine_complete(out: torch.Tensor, y: torch.Tensor, gates: np.ndarray,
                           comb_row: np.ndarray, chunk: int = 512, workers: int = 0):
    """Every combined row against the oracle (check_combine_host), in chunks of tokens:
    per chunk, the expert-output rows that the ORACLE's comb_row names are copied from
    the device (the generated inputs, selected by the oracle's indices)."""
    def prepare(t0, t1):
        rows = comb_row[t0:t1]
        valid = rows >= 0
        yh = rows_of(y, rows[valid])
        local = np.full(rows.shape, -1, np.int32)
        local[valid] = np.arange(int(valid.sum()), dtype=np.int32)
        o = out[t0:t1]
        got = o.cpu().numpy() if o.dtype == torch.float32 else host_bits(o)
        g = gates[t0:t1]

        def job():
            try:
                check_combine_host(got, yh, g, local)
            except AssertionError as e:
                raise AssertionError(f"combined rows of tokens [{t0}, {t1}): {e}") from None
        return job

    for_chunks(len(gates), chunk, prepare, workers)
