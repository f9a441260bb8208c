"""Seeded random shapes through the whole path, enqueued back to back on one stream (the
calls' kernels chained by programmatic dependent launch exactly as in a step), against the
oracle: counts, every plan output, the gathered rows and the combine.

Three call orders per case:
  0  count -> plan -> gather -> combine               (the step)
  1  plan -> combine -> gather                        (a combine right after the plan)
  2  plan(batch A) -> plan(batch B) -> gather -> combine   (the same plan buffers and
                                                       workspace reused by the next call
                                                       on the stream)
"""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import DEV, assert_plan_equal, check_combine, cuda, host_bits, plan_to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def rand_ids(rng, N, E, k):
    """N tokens' k distinct expert ids in random slot order."""
    out = np.empty((N, k), np.int32)
    for i0 in range(0, N, 8192):
        n = min(8192, N - i0)
        top = np.argpartition(rng.random((n, E)), k - 1, axis=1)[:, :k] if k < E else \
            np.tile(np.arange(E), (n, 1))
        out[i0:i0 + n] = np.take_along_axis(top, np.argsort(rng.random((n, k)), axis=1), 1)
    return out


def draw_case(seed):
    rng = np.random.default_rng(1000 + seed)
    N = int(rng.choice([0, 1, 257, 4097, int(rng.integers(1, 30000)), int(rng.integers(1, 30000)),
                        int(rng.integers(30000, 70000)), int(rng.integers(30000, 70000))]))
    E = int(rng.choice([2, 8, 64, 256, int(rng.integers(2, 300)), 1024]))
    k = int(rng.integers(1, min(8, E) + 1))
    R = int(rng.integers(1, 65))
    nodes = int(rng.integers(1, min(R, 8) + 1))
    H = 8 * int(rng.choice([1, 3, 32, 33, 256, int(rng.integers(1, 300))]))
    while N * k * H > (1 << 25) and H > 8:
        H = max(8, H // 16 * 8)
    N = min(N, (1 << 25) // (k * H))
    return rng, N, E, k, R, nodes, H, seed % 3


@pytest.mark.parametrize("seed", range(30))
def test_random_chain(coact, seed):
    rng, N, E, k, R, nodes, H, order = draw_case(seed)
    ids = rand_ids(rng, N, E, k)
    er = rng.integers(0, R, E).astype(np.int32)
    rn = np.sort(rng.integers(0, nodes, R)).astype(np.int32)
    src = rng.integers(0, R, N).astype(np.int32) if seed % 2 else None
    gates = rng.standard_normal((N, k)).astype(np.float32)
    g = torch.Generator(device=DEV).manual_seed(seed)
    x = torch.randn(N, H, device=DEV, generator=g).to(torch.bfloat16)
    y = torch.randn(N * k, H, device=DEV, generator=g).to(torch.bfloat16)
    pair = torch.zeros(E, E, dtype=torch.int64, device=DEV)
    loads = torch.zeros(E, dtype=torch.int64, device=DEV)
    plan = coact.alloc_plan(N, k, E, R, DEV)
    plan.row_token.fill_(-7)
    plan.row_kmask.fill_(0xEE)
    cap = plan.row_token.numel()
    send = torch.zeros(cap, H, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(N, H, dtype=torch.float32 if seed % 4 == 1 else torch.bfloat16, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    d_er, d_rn = cuda(er), cuda(rn)
    d_src = None if src is None else cuda(src)
    d_g = cuda(gates)

    def plan_of(i):
        coact.plan_dispatch(i, E, d_er, R, plan, rank_node=d_rn, n_nodes=nodes, src_rank=d_src,
                            err_flag=err)

    ids_a = rand_ids(rng, N, E, k)
    torch.cuda.synchronize()
    if order == 0:
        coact.coact_count(cuda(ids), E, pair, loads, err_flag=err)
        plan_of(cuda(ids))
        coact.dispatch_gather(x, plan.send_row, send, err_flag=err)
        coact.combine_scatter(y, d_g, plan.comb_row, out, err_flag=err)
    elif order == 1:
        plan_of(cuda(ids))
        coact.combine_scatter(y, d_g, plan.comb_row, out, err_flag=err)
        coact.dispatch_gather(x, plan.send_row, send, err_flag=err)
    else:
        plan_of(cuda(ids_a))
        plan_of(cuda(ids))
        coact.dispatch_gather(x, plan.send_row, send, err_flag=err)
        coact.combine_scatter(y, d_g, plan.comb_row, out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0

    o = oracle.plan(ids, E, er, R, rank_node=rn, n_nodes=nodes, src_rank=src)
    got = plan_to_host(plan)
    assert_plan_equal(got, o, sentinel=order != 2)
    D = int(o["rank_offsets"][-1])
    if order == 2:   # rows past D: untouched by the second plan (the first plan's, or -7)
        oa = oracle.plan(ids_a, E, er, R, rank_node=rn, n_nodes=nodes, src_rank=src)
        want = np.full(cap - D, -7, np.int32)
        m = max(0, min(int(oa["rank_offsets"][-1]), cap) - D)
        want[:m] = oa["row_token"][D:D + m]
        assert np.array_equal(got["row_token"][D:], want)
    if order == 0:
        po, lo, _ = oracle.count(ids, E)
        assert np.array_equal(pair.cpu().numpy(), po)
        assert np.array_equal(loads.cpu().numpy(), lo)
    if D:
        assert np.array_equal(host_bits(send[:D]), host_bits(x)[o["row_token"][:D]])
    if N:
        check_combine(out, host_bits(y), gates, o["comb_row"])
