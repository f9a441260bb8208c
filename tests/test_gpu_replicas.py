"""GPU parity of expert replicas, through the C ABI, against the CPU oracle: the replica
choice (assign_replicas) and the plan over per-slot ranks (plan_dispatch_slots) bit-exact
on full-size configurations and random replica tables, and the whole path with identity
experts equal to the naive combine."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import (DEV, X_STREAM, assert_plan_equal, check_combine, cuda, host_bits,
                       plan_to_host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def zero_flag():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def gpu_assign(coact, ids, E, rep, n_rep, R, rank_node, n_nodes, src=None):
    N, k = ids.shape
    slot = torch.full((N, k), -9, dtype=torch.int32, device=DEV)
    err = zero_flag()
    coact.assign_replicas(cuda(ids), E, cuda(rep), cuda(n_rep), R, slot,
                          rank_node=None if rank_node is None else cuda(rank_node, np.int32),
                          n_nodes=n_nodes, src_rank=None if src is None else cuda(src, np.int32),
                          err_flag=err)
    torch.cuda.synchronize()
    return slot, err.item()


@pytest.mark.parametrize("cfg", [2, 3])
def test_full_size_choice_and_plan(coact, cfg):
    r = workload.make_routing(cfg)
    c = r.cfg
    _, loads, _ = oracle.count(r.ids, c.E)
    rep, n_rep = workload.replicate_hot(loads, r.expert_rank, r.rank_node, c.E // 8)
    slot, err = gpu_assign(coact, r.ids, c.E, rep, n_rep, c.R, r.rank_node, c.n_nodes)
    want, f = oracle.assign_replicas(r.ids, c.E, rep, n_rep, c.R, rank_node=r.rank_node,
                                     n_nodes=c.n_nodes)
    assert err == f == 0
    assert np.array_equal(slot.cpu().numpy(), want)
    plan = coact.alloc_plan(c.N, c.k, c.E, c.R, DEV)
    plan.row_token.fill_(-7)
    plan.row_kmask.fill_(0xEE)
    coact.plan_dispatch(cuda(r.ids), c.E, None, c.R, plan, rank_node=cuda(r.rank_node, np.int32),
                        n_nodes=c.n_nodes, err_flag=(e2 := zero_flag()), slot_rank=slot)
    torch.cuda.synchronize()
    assert e2.item() == 0
    o = oracle.plan(r.ids, c.E, None, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes, slot_rank=want)
    assert_plan_equal(plan_to_host(plan), o)
    # the choice opens fewer (token, remote node) pairs than serving every slot on replica 0
    prim = oracle.plan(r.ids, c.E, rep[:, 0], c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    assert o["stats"][4] < prim["stats"][4]


@pytest.mark.parametrize("seed", range(6))
def test_random_tables(coact, seed):
    rng = np.random.default_rng(900 + seed)
    N = int(rng.integers(1, 5000))
    k = int(rng.integers(1, 9))
    R = int(rng.choice([2, 5, 16, 64]))
    E = max(k + 1, int(rng.integers(8, 200)))
    max_rep = int(rng.integers(1, 9))
    n_nodes = int(rng.integers(1, min(R, 8) + 1))
    rank_node = np.sort(rng.integers(0, n_nodes, R)).astype(np.int32)
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    n_rep = rng.integers(1, max_rep + 1, E).astype(np.int32)
    rep = np.full((E, max_rep), -1, np.int32)
    for e in range(E):
        rep[e, :n_rep[e]] = rng.choice(R, n_rep[e], replace=n_rep[e] > R)
    src = rng.integers(0, R, N).astype(np.int32)
    slot, err = gpu_assign(coact, ids, E, rep, n_rep, R, rank_node, n_nodes, src)
    want, f = oracle.assign_replicas(ids, E, rep, n_rep, R, rank_node=rank_node, n_nodes=n_nodes,
                                     src_rank=src)
    assert err == f == 0
    assert np.array_equal(slot.cpu().numpy(), want)
    plan = coact.alloc_plan(N, k, E, R, DEV)
    coact.plan_dispatch(cuda(ids), E, None, R, plan, rank_node=cuda(rank_node), n_nodes=n_nodes,
                        src_rank=cuda(src), slot_rank=slot)
    torch.cuda.synchronize()
    o = oracle.plan(ids, E, None, R, rank_node=rank_node, n_nodes=n_nodes, src_rank=src,
                    slot_rank=want)
    assert_plan_equal(plan_to_host(plan), o, sentinel=False)


def test_invalid_tables_and_tokens(coact):
    N, k, E, R = 6, 2, 4, 4
    ids = np.array([[0, 1], [1, 2], [2, 3], [3, 0], [0, 0], [9, 1]], np.int32)
    rep = np.array([[0, 1], [2, -1], [3, 7], [1, 2]], np.int32)
    n_rep = np.array([2, 1, 2, 2], np.int32)          # expert 2 has a replica on rank 7
    slot, err = gpu_assign(coact, ids, E, rep, n_rep, R, None, 1)
    want, f = oracle.assign_replicas(ids, E, rep, n_rep, R)
    assert err == f and f & coact.EFLAG_ID_RANGE and f & coact.EFLAG_DUP_ID
    assert np.array_equal(slot.cpu().numpy(), want)
    assert (want[1] == -1).all() and (want[2] == -1).all() and (want[0] >= 0).all()


@pytest.mark.parametrize("cfg", [1, 2])
def test_identity_experts_through_the_slot_plan(coact, cfg):
    """Gather and combine over the replica plan: with identity experts the combined rows
    equal x[t] * sum_j gates[t,j] through the fixed fp32 chain, whatever replica serves
    each slot (routing decisions unchanged)."""
    r = workload.make_routing(cfg)
    c = r.cfg
    H = 512
    _, loads, _ = oracle.count(r.ids, c.E)
    rep, n_rep = workload.replicate_hot(loads, r.expert_rank, r.rank_node, c.E // 8)
    slot, _ = gpu_assign(coact, r.ids, c.E, rep, n_rep, c.R, r.rank_node, c.n_nodes)
    plan = coact.alloc_plan(c.N, c.k, c.E, c.R, DEV)
    coact.plan_dispatch(cuda(r.ids), c.E, None, c.R, plan, rank_node=cuda(r.rank_node, np.int32),
                        n_nodes=c.n_nodes, slot_rank=slot)
    x = workload.fill_bf16(c.N, H, r.seed, X_STREAM, device=DEV)
    send = torch.empty((plan.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather(x, plan.send_row, send)
    torch.cuda.synchronize()
    o = oracle.plan(r.ids, c.E, None, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes,
                    slot_rank=slot.cpu().numpy())
    y_h = oracle.expand_identity(host_bits(x), o["row_token"], o["row_kmask"], o["D"])
    out = torch.empty((c.N, H), dtype=torch.float32, device=DEV)
    coact.combine_scatter(cuda(y_h.view(np.int16)).view(torch.bfloat16), cuda(r.gates),
                          plan.comb_row, out)
    torch.cuda.synchronize()
    naive = oracle.naive_combine_identity_f32(host_bits(x), r.gates)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), naive.view(np.uint32))
    check_combine(out, y_h, r.gates, o["comb_row"])
