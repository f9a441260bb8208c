"""rebalance_ranks (Cobalt's per-step intra-node adjustment on the device) against the
oracle's longest-first greedy, bit for bit: random loads with many ties over random node
layouts, the configurations' two-stage layouts with loads counted on the GPU, layouts
that do not fit, and the per-step chain count -> rebalance -> plan enqueued with no host
synchronisation."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, assert_plan_equal, cuda, plan_to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def _layout(rng, R, n_nodes, slots):
    """rank -> node (every node at least one rank) and expert -> node filling each node's
    slots exactly, both shuffled."""
    rn = np.concatenate([np.arange(n_nodes), rng.integers(0, n_nodes, R - n_nodes)])
    rn = rng.permutation(rn).astype(np.int32)
    en = rng.permutation(np.repeat(rn, slots)).astype(np.int32)
    return rn, en


@pytest.mark.parametrize("seed", range(16))
def test_rebalance_random_layouts(coact, seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 65))
    n_nodes = int(rng.integers(1, min(R, 16) + 1))
    slots = int(rng.integers(1, max(2, 1024 // R) + 1))
    slots = max(slots, 2 if R == 1 else 1)
    E = R * slots
    rn, en = _layout(rng, R, n_nodes, slots)
    loads = rng.integers(0, 6 if seed % 2 else 10 ** 9, E).astype(np.int64)   # ties or not
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = coact.rebalance_ranks(cuda(loads), cuda(en), cuda(rn), n_nodes, err_flag=err)
    want = oracle.rebalance_ranks(loads, en, rn)
    assert err.item() == 0
    assert np.array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("cfg", [2, 3])
def test_rebalance_two_stage_config(coact, cfg):
    """Stage 1 (host, periodic): node co-location from the pair counts; stage 2 (device,
    per step): the intra-node rebalance over the loads the GPU counted."""
    r = workload.make_routing(cfg)
    c = r.cfg
    pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=DEV)
    loads = torch.zeros(c.E, dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(r.ids), c.E, pair, loads)
    op, ol, _ = oracle.count(r.ids, c.E)
    en = oracle.place_correlated(op, c.n_nodes)
    got = coact.rebalance_ranks(loads, cuda(en), cuda(r.rank_node, np.int32), c.n_nodes)
    want = oracle.rebalance_ranks(ol, en, r.rank_node)
    assert np.array_equal(got.cpu().numpy(), want)
    # the host planner agrees too
    host = coact.coact_rebalance_ranks(torch.from_numpy(ol), torch.from_numpy(en),
                                       torch.from_numpy(r.rank_node.astype(np.int32)))
    assert np.array_equal(host.numpy(), want)


def test_rebalance_layouts_that_do_not_fit(coact):
    # 2 nodes of 2 ranks, 2 slots per rank: 8 experts
    rn = np.array([0, 0, 1, 1], np.int32)
    loads = np.arange(8, 0, -1).astype(np.int64)        # expert e has load 8 - e
    # node 0 asked to hold 5 experts in its 4 slots: the lightest of them finds no slot
    en = np.array([0, 0, 0, 1, 1, 1, 0, 0], np.int32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    got = coact.rebalance_ranks(cuda(loads), cuda(en), cuda(rn), 2, err_flag=err).cpu().numpy()
    assert err.item() == coact.EFLAG_ID_RANGE
    # by hand, node 0 (experts 0, 1, 2, 6, 7 with loads 8, 7, 6, 2, 1): 0 -> rank 0 (tie:
    # lower rank), 1 -> rank 1 (0 < 8), 2 -> rank 1 (7 < 8; rank 1 now full), 6 -> rank 0
    # (the only free slot; now full), 7 -> no slot left: -1.  Node 1 (experts 3, 4, 5 with
    # loads 5, 4, 3): 3 -> rank 2, 4 -> rank 3 (0 < 5), 5 -> rank 3 (4 < 5).
    assert got.tolist() == [0, 1, 1, 2, 3, 3, 0, -1]
    # an expert on a node outside the layout, and a rank on one
    en2 = np.array([0, 0, 0, 0, 1, 1, 1, 5], np.int32)
    err.zero_()
    got = coact.rebalance_ranks(cuda(loads), cuda(en2), cuda(rn), 2, err_flag=err).cpu().numpy()
    assert err.item() == coact.EFLAG_ID_RANGE and got[7] == -1
    err.zero_()
    got = coact.rebalance_ranks(cuda(loads), cuda(en), cuda(np.array([0, 0, 1, 9], np.int32)), 2,
                                err_flag=err).cpu().numpy()
    assert err.item() == coact.EFLAG_ID_RANGE and 3 not in got.tolist()


@pytest.mark.parametrize("cfg", [1, 2])
def test_per_step_chain_count_rebalance_plan(coact, cfg):
    """count (fresh loads) -> rebalance -> plan, enqueued back to back on one stream with no
    host synchronisation: the plan over the rebalanced placement equals the oracle's."""
    r = workload.make_routing(cfg)
    c = r.cfg
    op, ol, _ = oracle.count(r.ids, c.E)
    en = oracle.place_correlated(op, c.n_nodes) if c.n_nodes > 1 else np.zeros(c.E, np.int32)
    ids, rn, en_d = cuda(r.ids), cuda(r.rank_node, np.int32), cuda(en)
    loads = torch.empty(c.E, dtype=torch.int64, device=DEV)
    pair = torch.empty((c.E, c.E), dtype=torch.int64, device=DEV)
    er = torch.empty(c.E, dtype=torch.int32, device=DEV)
    plan = coact.alloc_plan(r.N, r.k, c.E, c.R, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):                                  # twice: the loads start from zero
        loads.zero_()
        pair.zero_()
        coact.coact_count(ids, c.E, pair, loads, err_flag=err)
        coact.rebalance_ranks(loads, en_d, rn, c.n_nodes, out=er, err_flag=err)
        coact.plan_dispatch(ids, c.E, er, c.R, plan, rank_node=rn, n_nodes=c.n_nodes,
                            err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    want_er = oracle.rebalance_ranks(ol, en, r.rank_node)
    assert np.array_equal(er.cpu().numpy(), want_er)
    o = oracle.plan(r.ids, c.E, want_er, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    assert_plan_equal(plan_to_host(plan), o, sentinel=False)
