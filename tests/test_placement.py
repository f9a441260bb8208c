"""Correlated expert placement (Zyphra English abstract: experts often selected together
go on the same GPU).  The oracle's greedy is pinned by hand-worked cases; the library's
host implementation must match it exactly.  Both are host code, so this runs on CPU."""
import numpy as np
import pytest

import oracle
import workload


def sym(E, weights):
    p = np.zeros((E, E), np.int64)
    for (a, b), w in weights.items():
        p[a, b] = p[b, a] = w
    return p


def test_hand_worked_pairs():
    # heaviest pair (0,3) takes rank 0, next (1,2) takes rank 1
    assert oracle.place_correlated(sym(4, {(0, 3): 5, (1, 2): 4}), 2).tolist() == [0, 1, 1, 0]


def test_hand_worked_chain():
    # 3 slots per rank: (0,1) -> rank 0; 2 joins its partner 1 on rank 0 (now full);
    # (2,3) cannot join; (3,4) opens rank 1; 5 joins 4
    w = {(0, 1): 10, (1, 2): 9, (2, 3): 8, (3, 4): 7, (4, 5): 6}
    assert oracle.place_correlated(sym(6, w), 2).tolist() == [0, 0, 0, 1, 1, 1]


def test_hand_worked_ties_and_leftovers():
    # equal weights: (1,4) before (2,3) (smaller a first); experts 0 and 5 are never
    # paired and fill the remaining slots in ascending id
    p = sym(6, {(2, 3): 3, (1, 4): 3})
    assert oracle.place_correlated(p, 3).tolist() == [2, 0, 1, 1, 0, 2]
    # no co-activation at all: ascending id fills ranks in order
    assert oracle.place_correlated(np.zeros((6, 6), np.int64), 3).tolist() == [0, 0, 1, 1, 2, 2]


def test_asymmetric_counts_use_both_halves():
    p = np.zeros((4, 4), np.int64)
    p[3, 0] = 5          # only the lower half holds the (0,3) weight
    p[1, 2] = 4
    assert oracle.place_correlated(p, 2).tolist() == [0, 1, 1, 0]


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_library_matches_oracle_on_config_counts(cfg):
    import co_activation_b200 as coact
    import torch
    r = workload.make_routing(cfg)
    pair, _, _ = oracle.count(r.ids, r.cfg.E)
    want = oracle.place_correlated(pair, r.cfg.R)
    got = coact.coact_place_correlated(torch.from_numpy(pair), r.cfg.R).numpy()
    assert np.array_equal(got, want)
    assert np.bincount(got, minlength=r.cfg.R).tolist() == [r.cfg.epr] * r.cfg.R
    # co-locating co-activated experts sends fewer rows than the config's own placement
    d_corr = oracle.plan(r.ids, r.cfg.E, want, r.cfg.R)["D"]
    d_base = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)["D"]
    assert d_corr < d_base


@pytest.mark.parametrize("seed", range(10))
def test_library_matches_oracle_random(seed):
    import co_activation_b200 as coact
    import torch
    rng = np.random.default_rng(seed)
    R = int(rng.choice([1, 2, 4, 8]))
    E = R * int(rng.integers(1, 9))
    if E < 2:
        E = 2 * R
    p = rng.integers(0, 4, (E, E)).astype(np.int64)          # many ties, asymmetric
    np.fill_diagonal(p, 0)
    want = oracle.place_correlated(p, R)
    got = coact.coact_place_correlated(torch.from_numpy(p), R).numpy()
    assert np.array_equal(got, want)


def test_library_rejects_bad_sizes():
    import co_activation_b200 as coact
    import torch
    with pytest.raises(coact.CoactError):
        coact.coact_place_correlated(torch.zeros((6, 6), dtype=torch.int64), 4)   # 6 % 4 != 0


# ----------------------------------------------------------------------------- two-stage planner


def test_rebalance_hand_worked():
    # one node, two ranks of two slots; heaviest first: e0 (10) -> r0, e2 (7) -> r1,
    # e3 (5) -> r1 (7 < 10), r1 full, e1 (1) -> r0: loads 11 / 12
    got = oracle.rebalance_ranks([10, 1, 7, 5], [0, 0, 0, 0], [0, 0])
    assert got.tolist() == [0, 0, 1, 1]


def test_rebalance_two_nodes_stays_in_node():
    loads = [5, 9, 2, 2, 8, 1, 3, 7]
    expert_node = [0, 1, 0, 1, 0, 1, 0, 1]
    # node 0 (ranks 0, 1): e4 (8) r0, e0 (5) r1, e6 (3) r1, e2 (2) r0
    # node 1 (ranks 2, 3): e1 (9) r2, e7 (7) r3, e3 (2) r3, e5 (1) r2
    got = oracle.rebalance_ranks(loads, expert_node, [0, 0, 1, 1])
    assert got.tolist() == [1, 2, 0, 3, 0, 2, 1, 3]


def test_rebalance_rejects_mismatched_node_sizes():
    with pytest.raises(ValueError):
        oracle.rebalance_ranks([1, 2, 3, 4], [0, 0, 0, 1], [0, 1])


@pytest.mark.parametrize("seed", range(8))
def test_rebalance_library_matches_oracle(seed):
    import co_activation_b200 as coact
    import torch
    rng = np.random.default_rng(300 + seed)
    n_nodes = int(rng.choice([1, 2, 4]))
    R = n_nodes * int(rng.integers(1, 5))
    E = R * int(rng.integers(1, 5))
    loads = rng.integers(0, 6, E).astype(np.int64)          # many equal loads
    rank_node = (np.arange(R) // (R // n_nodes)).astype(np.int32)
    expert_node = rng.permutation(np.repeat(np.arange(n_nodes), E // n_nodes)).astype(np.int32)
    want = oracle.rebalance_ranks(loads, expert_node, rank_node)
    got = coact.coact_rebalance_ranks(torch.from_numpy(loads), torch.from_numpy(expert_node),
                                      torch.from_numpy(rank_node)).numpy()
    assert np.array_equal(got, want)
    assert np.bincount(got, minlength=R).tolist() == [E // R] * R
    assert (rank_node[got] == expert_node).all()


@pytest.mark.parametrize("cfg", [2, 3])
def test_two_stage_layout_on_configs(cfg):
    """Stage 1 cuts cross-node traffic, stage 2 keeps it and evens the rank loads."""
    import co_activation_b200 as coact
    import torch
    r = workload.make_routing(cfg)
    c = r.cfg
    pair, loads, _ = oracle.count(r.ids, c.E)
    two = oracle.place_two_stage(pair, loads, r.rank_node, c.n_nodes)
    got = coact.coact_place_two_stage(torch.from_numpy(pair), torch.from_numpy(loads),
                                      torch.from_numpy(r.rank_node), c.n_nodes).numpy()
    assert np.array_equal(got, two)
    base = oracle.plan(r.ids, c.E, r.expert_rank, c.R, r.rank_node, c.n_nodes)
    p2 = oracle.plan(r.ids, c.E, two, c.R, r.rank_node, c.n_nodes)
    assert p2["stats"][4] < base["stats"][4]            # fewer (token, remote node) pairs
    rank_load = lambda er: np.bincount(er[r.ids.ravel()], minlength=c.R)
    corr = oracle.place_correlated(pair, c.R)
    assert rank_load(two).max() < rank_load(corr).max()  # better balanced than rank-level co-location
