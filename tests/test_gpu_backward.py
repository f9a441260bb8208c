"""GPU parity of the backward pass and the pre-reduced reverse path, through the C ABI,
against the CPU oracle on the same seeded inputs.

  dispatch_gather_backward   bit-exact with the oracle's fp32 add chain (fp32 out) and its
                             round-to-nearest-even (bf16 out)
  combine_rows               bit-exact with the oracle's unit combine (fp32 fma chain)
  pre-reduced combine        combine_rows over the plan's send rows (bf16 partial rows), then
                             dispatch_gather_backward: bit-exact with the oracle's
  combine_scatter_backward   grad_y bit-exact (fp32 product rounded to bf16); grad_gates
                             within the stated bound of the float64 dot product:
                             (m + 5) * 2^-24 * sum_h |grad_out * y|, m the terms per lane
                             (max(8*ceil(H/256), 16*ceil(H/512)))
Full-size configurations are checked in full (every row and every gate gradient, streamed
in chunks against the oracle), with the launch configuration the benchmark uses."""
import math

import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, Y_STREAM, cuda, for_chunks, host_bits, rows_of, run_plan

pytestmark = pytest.mark.gpu

G_STREAM, GO_STREAM = 5, 6       # fill_bf16 streams: gradient rows of the dispatch / the combine


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def zero_flag():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def oracle_plan_for(r):
    c = r.cfg
    return oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)


def check_grad_x(got: torch.Tensor, g_bits: np.ndarray, send_row: np.ndarray, tokens=None):
    """got rows (all, or `tokens`) against the oracle's chain over g_bits (the rows
    send_row indexes)."""
    chain = oracle.gather_backward_f32chain(g_bits, send_row)
    if tokens is not None:
        got = got[torch.as_tensor(tokens, device=got.device)]
    if got.dtype == torch.float32:
        assert np.array_equal(got.cpu().numpy().view(np.uint32), chain.view(np.uint32))
    else:
        assert np.array_equal(host_bits(got), oracle.bf16_rne(chain))


def grad_gates_bound(H: int, mag: np.ndarray) -> np.ndarray:
    # terms per lane: 8 * ceil(H/256) with 16-byte chunks, 16 * ceil(H/512) with 32-byte ones
    m = max(8 * math.ceil(H / 256), 16 * math.ceil(H / 512))
    return 1.01 * (m + 5) * 2.0 ** -24 * mag + 1e-30


def check_combine_backward(gy_dev, gg_dev, y_bits, gates, comb_row, go_bits, gy_rows=None,
                           gg_tokens=None):
    """Oracle on the local arrays; gy_rows: device rows of grad_y that local row i stands
    for (default: all); gg_tokens: device tokens of grad_gates (default: all)."""
    gy_o, gg_o, ga_o = oracle.combine_backward(y_bits, gates, comb_row, go_bits)
    valid = comb_row.ravel()
    valid = np.unique(valid[valid >= 0])
    rows = valid if gy_rows is None else np.asarray(gy_rows)[valid]
    got_rows = host_bits(gy_dev[torch.as_tensor(rows, device=gy_dev.device)])
    assert np.array_equal(got_rows, gy_o[valid])
    gg = gg_dev.cpu().numpy() if gg_tokens is None else gg_dev[
        torch.as_tensor(gg_tokens, device=gg_dev.device)].cpu().numpy()
    assert (np.abs(gg.astype(np.float64) - gg_o) <= grad_gates_bound(y_bits.shape[1], ga_o)).all()


# ----------------------------------------------------------------------------- transposed dispatch


@pytest.mark.parametrize("cfg", [0, 1])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gather_backward_full(coact, cfg, out_dtype):
    r = workload.make_routing(cfg)
    H = r.cfg.H
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    cap = plan.row_capacity
    g_send = workload.fill_bf16(cap, H, r.seed, G_STREAM, device=DEV)
    gx = torch.empty((r.N, H), dtype=out_dtype, device=DEV)
    err = zero_flag()
    coact.dispatch_gather_backward(g_send, plan.send_row, gx, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    check_grad_x(gx, host_bits(g_send), o["send_row"])


@pytest.mark.parametrize("cfg", [2, 3])
def test_gather_backward_full_size_complete(coact, cfg):
    """Configs 2 and 3 at full size: every token's gradient row against the oracle's fp32
    add chain over the rows the oracle's send_row names, in chunks of tokens."""
    r = workload.make_routing(cfg)
    H = r.cfg.H
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    g_send = workload.fill_bf16(plan.row_capacity, H, r.seed, G_STREAM, device=DEV)
    gx = torch.empty((r.N, H), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.dispatch_gather_backward(g_send, plan.send_row, gx, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0

    def prepare(t0, t1):
        sr = o["send_row"][t0:t1]
        valid = sr >= 0
        g_local = rows_of(g_send, sr[valid])
        local = np.full(sr.shape, -1, np.int32)
        local[valid] = np.arange(int(valid.sum()), dtype=np.int32)
        got = host_bits(gx[t0:t1])
        return lambda: np.testing.assert_array_equal(
            got, oracle.bf16_rne(oracle.gather_backward_f32chain(g_local, local)),
            err_msg=f"tokens [{t0}, {t1})")

    for_chunks(r.N, 1024, prepare)


@pytest.mark.parametrize("k", [1, 3, 8])
@pytest.mark.parametrize("H", [8, 1000])
def test_gather_backward_shapes(coact, k, H):
    r = workload.make_routing(0)
    rng = np.random.default_rng(k * 10 + H)
    N, E, R = 777, 16, 4
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(N)]).astype(np.int32)
    er = rng.permutation(np.repeat(np.arange(R), E // R)).astype(np.int32)
    o = oracle.plan(ids, E, er, R)
    g = workload.fill_bf16(o["row_capacity"], H, k, 7, device=DEV)
    for dt in (torch.bfloat16, torch.float32):
        gx = torch.empty((N, H), dtype=dt, device=DEV)
        coact.dispatch_gather_backward(g, cuda(o["send_row"]), gx)
        check_grad_x(gx, host_bits(g), o["send_row"])
    del r


def test_gather_backward_row_range_flag(coact):
    N, k, H = 50, 2, 16
    send_row = np.full((N, k), -1, np.int32)
    send_row[:, 0] = np.arange(N)
    send_row[3, 1] = N + 4                     # outside the gradient rows: skipped, flagged
    send_row[7, 1] = -3                        # below -1: skipped, flagged
    g = workload.fill_bf16(N, H, 1, 8, device=DEV)
    gx = torch.empty((N, H), dtype=torch.float32, device=DEV)
    err = zero_flag()
    coact.dispatch_gather_backward(g, cuda(send_row), gx, err_flag=err)
    assert err.item() == coact.EFLAG_ROW_RANGE
    check_grad_x(gx, host_bits(g), send_row)


# ----------------------------------------------------------------------------- pre-reduced combine


@pytest.mark.parametrize("cfg", [0, 1])
def test_prereduced_combine_full(coact, cfg):
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    D = o["D"]
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    gates = cuda(r.gates)
    pre = torch.empty((D, H), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.combine_rows(y, gates, plan.comb_row, plan.row_token, plan.row_kmask, pre, err_flag=err)
    out = torch.empty((r.N, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather_backward(pre, plan.send_row, out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    pre_o, out_o = oracle.combine_prereduced(host_bits(y), r.gates, o)
    assert np.array_equal(host_bits(pre), pre_o)
    assert np.array_equal(host_bits(out), oracle.bf16_rne(out_o))


def test_combine_rows_device_unit_count(coact):
    """n_units = the plan's row capacity, bounded on the device by rank_offsets[R] = D: rows
    past D (row_token sentinel -7 from the test plan) are neither read nor written."""
    r = workload.make_routing(1)
    H, nk, R = 256, r.N * r.k, r.cfg.R
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    D, cap = o["D"], plan.row_capacity
    assert D < cap
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    gates = cuda(r.gates)
    pre = torch.full((cap, H), float("nan"), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.combine_rows(y, gates, plan.comb_row, plan.row_token, plan.row_kmask, pre,
                       unit_count=plan.rank_offsets[R:], err_flag=err)
    g_out = workload.fill_bf16(cap, H, r.seed, GO_STREAM, device=DEV)
    gy = torch.empty((nk, H), dtype=torch.bfloat16, device=DEV)
    gg = torch.empty((r.N, r.k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(y, gates, plan.comb_row, g_out, gy, gg,
                                   row_token=plan.row_token, row_kmask=plan.row_kmask,
                                   unit_count=plan.rank_offsets[R:], err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    pre_o, _ = oracle.combine_prereduced(host_bits(y), r.gates, o)
    assert np.array_equal(host_bits(pre[:D]), pre_o)
    assert torch.isnan(pre[D:].float()).all()
    gy_o, gg_o, ga_o = oracle.combine_backward(host_bits(y), r.gates, o["comb_row"],
                                               host_bits(g_out[:D]), o["row_token"], o["row_kmask"], D)
    assert np.array_equal(host_bits(gy), gy_o)
    assert (np.abs(gg.cpu().numpy().astype(np.float64) - gg_o) <= grad_gates_bound(H, ga_o)).all()


@pytest.mark.parametrize("cfg", [2, 3])
def test_combine_rows_full_size_complete(coact, cfg):
    """Configs 2 and 3 at full size: every partial row (one per send row) against the
    oracle's fp32 chain over the unit's slots, in chunks of send rows."""
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    D = o["D"]
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    pre = torch.empty((D, H), dtype=torch.float32, device=DEV)
    coact.combine_rows(y, cuda(r.gates), plan.comb_row, plan.row_token, plan.row_kmask, pre)
    torch.cuda.synchronize()

    def prepare(u0, u1):
        toks = o["row_token"][u0:u1]
        cr = o["comb_row"][toks]
        y_local = rows_of(y, cr)
        local = np.arange(cr.size, dtype=np.int32).reshape(cr.shape)
        got = pre[u0:u1].cpu().numpy()
        g, km = r.gates[toks], o["row_kmask"][u0:u1]

        def job():
            want = oracle.combine_units_f32chain(y_local, g, local,
                                                 np.arange(u1 - u0, dtype=np.int32), km)
            np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32),
                                          err_msg=f"units [{u0}, {u1})")
        return job

    for_chunks(D, 1024, prepare)


# ----------------------------------------------------------------------------- combine backward


@pytest.mark.parametrize("cfg", [0, 1])
def test_combine_backward_full(coact, cfg):
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    g_out = workload.fill_bf16(r.N, H, r.seed, GO_STREAM, device=DEV)
    gy = torch.empty((nk, H), dtype=torch.bfloat16, device=DEV)
    gg = torch.empty((r.N, r.k), dtype=torch.float32, device=DEV)
    err = zero_flag()
    coact.combine_scatter_backward(y, cuda(r.gates), plan.comb_row, g_out, gy, gg, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    check_combine_backward(gy, gg, host_bits(y), r.gates, o["comb_row"], host_bits(g_out))


@pytest.mark.parametrize("cfg", [2, 3])
def test_combine_backward_full_size_complete(coact, cfg):
    """Configs 2 and 3 at full size: every grad_y row bit for bit and every gate gradient
    within its bound, in chunks of tokens (each chunk's y rows and grad_y rows are the
    ones the oracle's comb_row names)."""
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    g_out = workload.fill_bf16(r.N, H, r.seed, GO_STREAM, device=DEV)
    gy = torch.empty((nk, H), dtype=torch.bfloat16, device=DEV)
    gg = torch.empty((r.N, r.k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(y, cuda(r.gates), plan.comb_row, g_out, gy, gg)
    torch.cuda.synchronize()
    gg_h = gg.cpu().numpy().astype(np.float64)

    def prepare(t0, t1):
        cr = o["comb_row"][t0:t1]
        y_local, gy_got = rows_of(y, cr), rows_of(gy, cr)
        go_local = host_bits(g_out[t0:t1])
        local = np.arange(cr.size, dtype=np.int32).reshape(cr.shape)
        g = r.gates[t0:t1]

        def job():
            gy_o, gg_o, ga_o = oracle.combine_backward(y_local, g, local, go_local)
            np.testing.assert_array_equal(gy_got, gy_o, err_msg=f"grad_y, tokens [{t0}, {t1})")
            assert (np.abs(gg_h[t0:t1] - gg_o) <= grad_gates_bound(H, ga_o)).all(), (t0, t1)
        return job

    for_chunks(r.N, 512, prepare)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_combine_backward_over_plan_rows_equals_tokens(coact, cfg):
    """Units = the plan's send rows with the token's gradient row dispatched to each (the
    gather of grad_out): the slot masks partition each token's slots, and a unit's dot
    products run in the same order as the token's, so both results are bit-identical."""
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    if cfg == 2:
        H = 512
    plan, _ = run_plan(coact, r)
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    g_out = workload.fill_bf16(r.N, H, r.seed, GO_STREAM, device=DEV)
    gates = cuda(r.gates)
    gy_t = torch.empty((nk, H), dtype=torch.bfloat16, device=DEV)
    gg_t = torch.empty((r.N, r.k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(y, gates, plan.comb_row, g_out, gy_t, gg_t)
    D = int(plan.rank_offsets[-1].item())
    g_rows = torch.empty((plan.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather(g_out, plan.send_row, g_rows)
    gy_u = torch.empty_like(gy_t)
    gg_u = torch.full_like(gg_t, float("nan"))
    err = zero_flag()
    coact.combine_scatter_backward(y, gates, plan.comb_row, g_rows[:D], gy_u, gg_u,
                                   row_token=plan.row_token, row_kmask=plan.row_kmask, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(gy_t.view(torch.int16), gy_u.view(torch.int16))
    assert torch.equal(gg_t.view(torch.int32), gg_u.view(torch.int32))


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("H", [8, 1000, 2056])
def test_combine_backward_k_and_h(coact, k, H):
    rng = np.random.default_rng(k * 1000 + H)
    N = 555
    gates = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    y = workload.fill_bf16(N * k, H, k, 9, device=DEV)
    g_out = workload.fill_bf16(N, H, k, 10, device=DEV)
    gy = torch.empty_like(y)
    gg = torch.empty((N, k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(y, cuda(gates), cuda(comb), g_out, gy, gg)
    check_combine_backward(gy, gg, host_bits(y), gates, comb, host_bits(g_out))


def test_combine_backward_invalid_slots(coact):
    N, k, H = 64, 3, 24
    rng = np.random.default_rng(2)
    gates = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    freed = [int(comb[4, 1]), int(comb[9, 2])]
    comb[4, 1] = -1                           # slot of an invalid token: no row, gate grad 0
    comb[9, 2] = N * k + 5                    # out of range: skipped and flagged
    y = workload.fill_bf16(N * k, H, 0, 11, device=DEV)
    g_out = workload.fill_bf16(N, H, 0, 12, device=DEV)
    gy = torch.full_like(y, float("nan"))
    gg = torch.empty((N, k), dtype=torch.float32, device=DEV)
    err = zero_flag()
    coact.combine_scatter_backward(y, cuda(gates), cuda(comb), g_out, gy, gg, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == coact.EFLAG_ROW_RANGE
    assert gg[4, 1].item() == 0.0 and gg[9, 2].item() == 0.0
    assert torch.isnan(gy[freed].float()).all()       # rows no slot names: not written
    comb_o = comb.copy()
    comb_o[9, 2] = -1
    check_combine_backward(gy, gg, host_bits(y), gates, comb_o, host_bits(g_out))


def test_backward_empty(coact):
    H = 16
    y = torch.empty((0, H), dtype=torch.bfloat16, device=DEV)
    g = torch.empty((0, H), dtype=torch.bfloat16, device=DEV)
    gates = torch.empty((0, 2), dtype=torch.float32, device=DEV)
    comb = torch.empty((0, 2), dtype=torch.int32, device=DEV)
    coact.combine_scatter_backward(y, gates, comb, g, torch.empty_like(y), torch.empty_like(gates))
    coact.dispatch_gather_backward(g, comb, torch.empty((0, H), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()


@pytest.mark.parametrize("k", [3, 8])
def test_gather_backward_slot_order_of_the_sum(coact, k):
    """Rows 1, 2^24, -2^24 on a token's first three send rows: 0 when added in slot order,
    1 in reverse -- the kernel (also its sparse-slot form for k >= 3) adds in slot order."""
    H = 64
    send_row = np.full((2, k), -1, np.int32)
    send_row[0, :3] = [0, 1, 2]
    send_row[1, :3] = [2, 1, 0]
    g = torch.tensor([[1.0], [2.0 ** 24], [-(2.0 ** 24)]], dtype=torch.float32).expand(3, H)
    g = g.contiguous().to(torch.bfloat16).to(DEV)
    gx = torch.empty((2, H), dtype=torch.float32, device=DEV)
    coact.dispatch_gather_backward(g, cuda(send_row), gx)
    torch.cuda.synchronize()
    assert (gx[0] == 0.0).all() and (gx[1] == 1.0).all()
