"""Pins for the oracle's replica choice and per-slot plan (Cobalt, arxivdaily 2609.36959,
English abstract: EP distributes expert replicas across GPUs; a communication-aware task
assignment routes tokens to fewer remote nodes under the current layout).  The greedy is
the reading stated in the oracle; it is pinned by hand-worked cases for each of its
classes, by the single-replica case reducing to the plain plan, by invariants the
reading guarantees, and the per-slot plan by brute force (sorting)."""
import numpy as np
import pytest

import oracle
from test_oracle_pins import brute_plan, rand_ids

NODES6 = [0, 0, 1, 1, 2, 2]          # six ranks on three nodes


def assign(ids, rep, R=6, rank_node=NODES6, src=None):
    E = len(rep)
    max_rep = max(len(r) for r in rep)
    rr = np.full((E, max_rep), -1, np.int32)
    for e, r in enumerate(rep):
        rr[e, :len(r)] = r
    nr = np.array([len(r) for r in rep], np.int32)
    return oracle.assign_replicas(np.array(ids, np.int32), E, rr, nr, R, rank_node=rank_node,
                                  n_nodes=max(rank_node) + 1, src_rank=src)


def test_hand_worked_each_class():
    # experts: 0 single on rank 2 (node 1); 1 on [3, 2]; 2 on [2, 1]; 3 on [4, 3]; 4 on [4, 5];
    # 5 on [5, 0]
    rep = [[2], [3, 2], [2, 1], [4, 3], [4, 5], [5, 0]]
    ids = [[1, 0],     # t0 home 0: slot 1 forced to 2; slot 0: (b) rank 2 already used -> 2
           [2, 5],     # t1 home 0: slot 0: (c) home node 0 -> rank 1; slot 1: (a) home rank 0 -> 0
           [0, 3],     # t2 home 0: slot 0 forced 2 (node 1); slot 1: (d) node 1 in use -> 3
           [4, 5],     # t3 home 0: slot 0: no class -> (t + j) % 2 = 1 -> rank 5; slot 1: (a) 0
           [4, 2]]     # t4 home 0: slot 0: no class -> (4 + 0) % 2 = 0 -> rank 4; slot 1: (c) 1
    got, f = assign(ids, rep, src=[0, 0, 0, 0, 0])
    assert f == 0
    assert got.tolist() == [[2, 2], [1, 0], [2, 3], [5, 0], [4, 1]]


def test_home_rank_beats_used_rank_and_primary():
    rep = [[1], [1, 4]]
    # home 4: expert 0 forced to rank 1; expert 1 has replicas on 1 (used) and 4 (home):
    # the home rank comes first
    got, _ = assign([[0, 1]], rep, src=[4])
    assert got.tolist() == [[1, 4]]


def test_single_replicas_reduce_to_the_plain_plan():
    rng = np.random.default_rng(5)
    N, E, k, R = 300, 16, 3, 4
    ids = rand_ids(rng, N, E, k)
    er = rng.integers(0, R, E).astype(np.int32)
    rn = np.array([0, 0, 1, 1], np.int32)
    src = rng.integers(0, R, N).astype(np.int32)
    slot, f = oracle.assign_replicas(ids, E, er[:, None], np.ones(E, np.int32), R, rank_node=rn,
                                     n_nodes=2, src_rank=src)
    assert f == 0 and np.array_equal(slot, er[ids])
    a = oracle.plan(ids, E, er, R, rank_node=rn, n_nodes=2, src_rank=src)
    b = oracle.plan(ids, E, None, R, rank_node=rn, n_nodes=2, src_rank=src, slot_rank=slot)
    for key in ("rank_counts", "rank_offsets", "asg_offsets", "rank_mask", "row_token",
                "row_kmask", "send_row", "comb_row", "stats", "src_dst"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("seed", range(12))
def test_slot_plan_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    N, k, R = int(rng.integers(1, 40)), int(rng.integers(1, 5)), int(rng.integers(1, 7))
    slot = rng.integers(0, R, (N, k)).astype(np.int32)
    rn = np.sort(rng.integers(0, 3, R)).astype(np.int32)
    src = rng.integers(0, R, N).astype(np.int32)
    # one pseudo-expert per slot whose rank is the slot's: the brute-force planner over it
    pseudo = np.arange(N * k, dtype=np.int32).reshape(N, k)
    want = brute_plan(pseudo, slot.ravel(), R, rn, src)
    got = oracle.plan(pseudo, N * k, None, R, rank_node=rn, n_nodes=int(rn.max()) + 1,
                      src_rank=src, slot_rank=slot)
    assert got["flags"] == 0
    for key in ("rank_counts", "rank_offsets", "asg_offsets", "send_row", "comb_row", "stats",
                "src_dst"):
        assert np.array_equal(got[key], want[key]), key
    D = got["D"]
    assert np.array_equal(got["row_token"][:D], want["row_token"])
    assert np.array_equal(got["row_kmask"][:D], want["row_kmask"])


@pytest.mark.parametrize("seed", range(6))
def test_invariants_on_random_layouts(seed):
    rng = np.random.default_rng(200 + seed)
    N, E, k, R = 500, 24, 4, 6
    ids = rand_ids(rng, N, E, k)
    rep = [sorted(rng.choice(R, int(rng.integers(1, 4)), replace=False).tolist()) for _ in range(E)]
    src = rng.integers(0, R, N).astype(np.int32)
    got, f = assign(ids, rep, src=src)
    assert f == 0
    for t in range(N):
        for j in range(k):
            e, r = ids[t][j], got[t, j]
            assert r in rep[e]                                   # a replica of its expert
            if len(rep[e]) == 1:
                assert r == rep[e][0]                            # forced
            elif src[t] in rep[e]:
                assert r == src[t]                               # served on the home rank


def test_validation_flags():
    rep = np.array([[0, 1], [2, -1]], np.int32)
    ids = np.array([[0, 1], [1, 0], [0, 1]], np.int32)
    bad_n = np.array([2, 0], np.int32)                           # expert 1: no replica
    got, f = oracle.assign_replicas(ids, 2, rep, bad_n, 4, src_rank=[0, 1, 2])
    assert f & 1 and (got == -1).all()
    bad_r = np.array([[0, 7], [2, 3]], np.int32)                 # rank 7 outside [0, 4)
    got, f = oracle.assign_replicas(ids, 2, bad_r, np.array([2, 2], np.int32), 4, src_rank=[0, 1, 2])
    assert f & 1 and (got == -1).all()
    got, f = oracle.assign_replicas(ids, 2, np.array([[0, 1], [2, 3]], np.int32),
                                    np.array([2, 2], np.int32), 4, src_rank=[0, 9, 2])
    assert f & 8 and (got[1] == -1).all() and (got[[0, 2]] >= 0).all()


# ----------------------------------------------------------------------------- replica placement


def sym_pairs(E, w):
    p = np.zeros((E, E), np.int64)
    for (a, b), v in w.items():
        p[a, b] = p[b, a] = v
    return p


def rank_loads(rep, n_rep, loads, R):
    out = np.zeros(R, np.int64)
    for e in range(len(loads)):
        for i in range(n_rep[e]):
            out[rep[e, i]] += loads[e] * 840 // n_rep[e]
    return out


def test_placement_hand_worked_fresh_node():
    # ranks 0,1 on node 0, ranks 2,3 on node 1; rank 0 is the heaviest (experts 0, 1) and
    # expert 0 its heaviest share; the only node without a replica of it is node 1, whose
    # lighter rank is 3
    pair = sym_pairs(4, {(0, 2): 5, (0, 3): 1})
    rep, n_rep, added = oracle.place_replicas(pair, [10, 1, 2, 3], [0, 0, 1, 2], [0, 0, 1, 1], 1)
    assert added == 1
    assert rep.tolist() == [[0, 3], [0, -1], [1, -1], [2, -1]] and n_rep.tolist() == [2, 1, 1, 1]


def test_placement_hand_worked_affinity_picks_the_node():
    # one rank per node; expert 0 (rank 0) is co-activated with expert 2 (node 2) more than
    # with expert 1 (node 1): its replica goes to node 2
    pair = sym_pairs(3, {(0, 1): 1, (0, 2): 4})
    rep, n_rep, _ = oracle.place_replicas(pair, [9, 2, 2], [0, 1, 2], [0, 1, 2], 1)
    assert rep[0].tolist() == [0, 2]
    # without co-activation the lower node wins the tie
    rep, _, _ = oracle.place_replicas(np.zeros((3, 3), np.int64), [9, 2, 2], [0, 1, 2], [0, 1, 2], 1)
    assert rep[0].tolist() == [0, 1]


def test_placement_budget_zero_and_exhaustion():
    er, rn = [0, 1, 2, 3], [0, 0, 1, 1]
    rep, n_rep, added = oracle.place_replicas(np.zeros((4, 4), np.int64), [5, 4, 3, 2], er, rn, 0)
    assert added == 0 and rep[:, 0].tolist() == er and (n_rep == 1).all()
    # max_rep 2 on 4 experts: at most 4 replicas can be added, then the loop stops
    rep, n_rep, added = oracle.place_replicas(np.zeros((4, 4), np.int64), [5, 4, 3, 2], er, rn, 50)
    assert added == 4 and (n_rep == 2).all()
    for e in range(4):
        assert len(set(rep[e].tolist())) == 2                 # distinct ranks per expert


def test_placement_moves_on_when_the_heaviest_rank_is_exhausted():
    """Budget 3, max_rep 2; ranks 0,1 on node 0, ranks 2,3 on node 1; two experts per
    rank, loads 200,200 | 90,10 | 20,20 | 10,10 (units of 1/840 below omitted).
    1. rank 0 (400) gives expert 0 (share 200, lower id of the tie) a replica on node 1's
       lighter rank 3: rank 0 -> 300, rank 3 -> 120;
    2. rank 0 (300) gives expert 1 a replica on rank 2 (40 < 120): rank 0 -> 200,
       rank 2 -> 140;
    3. rank 0 (200) is still the heaviest, but both its experts are at max_rep.  The
       budget is the number of replicas to add, so the next most loaded rank that can
       still be relieved gives one: rank 2 (140), expert 4 (share 20, lower id), on node 0
       (the only node without it), whose lighter rank is 1 (100 < 200).
    Stopping at step 3 instead (added = 2) would leave budget unspent although rank 2
    could still be relieved."""
    er = [0, 0, 1, 1, 2, 2, 3, 3]
    rn = [0, 0, 1, 1]
    loads = [200, 200, 90, 10, 20, 20, 10, 10]
    rep, n_rep, added = oracle.place_replicas(np.zeros((8, 8), np.int64), loads, er, rn, 3, 2)
    assert added == 3
    assert rep.tolist() == [[0, 3], [0, 2], [1, -1], [1, -1], [2, 1], [2, -1], [3, -1], [3, -1]]
    assert n_rep.tolist() == [2, 2, 1, 1, 2, 1, 1, 1]
    assert rank_loads(rep, n_rep, loads, 4).tolist() == [200 * 840, 110 * 840, 130 * 840,
                                                         120 * 840]


def test_placement_skips_experts_already_on_every_rank():
    """Two ranks on two nodes, max_rep 4 > R: replicas sit on distinct ranks, so an
    expert with a replica on each of the R ranks cannot take another.  Loads 100 | 1:
    1. rank 0 (100) gives expert 0 a replica on rank 1: both ranks at 50 + (1 on rank 1);
    2. rank 1 (51) holds expert 0 (on both ranks already: not replicable) and expert 1:
       expert 1 gets its replica on rank 0;
    3. no expert is replicable any more: the loop ends with added = 2.
    Taking expert 0 at step 2 (its share 50 beats 1) would find no rank for it and end
    the loop with added = 1, the budget unspent while expert 1 could still be placed."""
    rep, n_rep, added = oracle.place_replicas(np.zeros((2, 2), np.int64), [100, 1], [0, 1],
                                              [0, 1], 3, 4)
    assert added == 2
    assert rep.tolist() == [[0, 1, -1, -1], [1, 0, -1, -1]] and n_rep.tolist() == [2, 2]


@pytest.mark.parametrize("seed", range(6))
def test_placement_invariants_random(seed):
    rng = np.random.default_rng(700 + seed)
    R = int(rng.choice([4, 8, 16]))
    n_nodes = int(rng.choice([1, 2, 4]))
    E = R * int(rng.integers(1, 5))
    rn = (np.arange(R) * n_nodes // R).astype(np.int32)
    er = rng.permutation(np.arange(E) % R).astype(np.int32)
    loads = rng.zipf(1.5, E).astype(np.int64) * 10
    pair = rng.integers(0, 20, (E, E)).astype(np.int64)
    max_rep = int(rng.integers(2, 5))
    budget = int(rng.integers(1, E))
    rep, n_rep, added = oracle.place_replicas(pair, loads, er, rn, budget, max_rep)
    assert added == int((n_rep - 1).sum()) and added <= budget
    assert (rep[:, 0] == er).all() and (n_rep <= max_rep).all()
    for e in range(E):
        rs = rep[e, :n_rep[e]].tolist()
        assert len(set(rs)) == len(rs) and all(0 <= r < R for r in rs)
        assert (rep[e, n_rep[e]:] == -1).all()
    # replicas only ever take load off the heaviest rank
    before = rank_loads(er[:, None], np.ones(E, np.int32), loads, R)
    after = rank_loads(rep, n_rep, loads, R)
    assert after.sum() <= before.sum() and after.max() <= before.max()


@pytest.mark.parametrize("seed", range(8))
def test_placement_library_matches_oracle_random(seed):
    import co_activation_b200 as coact
    import torch
    rng = np.random.default_rng(800 + seed)
    R = int(rng.choice([2, 8, 32, 64]))
    n_nodes = int(rng.choice([1, 2, 4, 8]))
    E = R * int(rng.integers(1, 5))
    rn = (np.arange(R) * n_nodes // R).astype(np.int32)
    er = rng.permutation(np.arange(E) % R).astype(np.int32)
    loads = rng.integers(0, 6, E).astype(np.int64)                 # many ties
    pair = rng.integers(0, 3, (E, E)).astype(np.int64)
    max_rep = int(rng.integers(1, 9))
    budget = int(rng.integers(0, 2 * E))
    want = oracle.place_replicas(pair, loads, er, rn, budget, max_rep)
    got = coact.coact_place_replicas(torch.from_numpy(pair), torch.from_numpy(loads),
                                     torch.from_numpy(er), torch.from_numpy(rn), budget, max_rep)
    assert np.array_equal(got[0].numpy(), want[0]) and np.array_equal(got[1].numpy(), want[1])
    assert got[2] == want[2]


@pytest.mark.parametrize("cfg", [2, 3])
def test_placement_on_config_counts(cfg):
    """On the configurations' own counts the planned replicas (as many as the load fixture
    places) leave fewer (token, remote node) pairs and a lighter busiest rank than serving
    every slot on replica 0."""
    import co_activation_b200 as coact
    import torch
    import workload
    r = workload.make_routing(cfg)
    c = r.cfg
    pair, loads, _ = oracle.count(r.ids, c.E)
    rep, n_rep, added = oracle.place_replicas(pair, loads, r.expert_rank, r.rank_node, c.E // 8)
    lib = coact.coact_place_replicas(torch.from_numpy(pair), torch.from_numpy(loads),
                                     torch.from_numpy(r.expert_rank.astype(np.int32)),
                                     torch.from_numpy(r.rank_node.astype(np.int32)), c.E // 8)
    assert np.array_equal(lib[0].numpy(), rep) and added == c.E // 8
    slot, _ = oracle.assign_replicas(r.ids, c.E, rep, n_rep, c.R, rank_node=r.rank_node,
                                     n_nodes=c.n_nodes)
    p = oracle.plan(r.ids, c.E, None, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes, slot_rank=slot)
    prim = oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    assert p["stats"][4] < prim["stats"][4]
    asg = lambda pl: np.diff(pl["asg_offsets"])
    assert asg(p).max() < asg(prim).max()


def test_used_rank_beats_home_node_and_rotation_uses_the_slot():
    # expert 0 single on rank 2 (node 1); expert 1 on [1, 2]: home 0 (node 0) -- rank 2 is
    # already used by the token (class b) and comes before the home-node replica 1 (class c)
    got, _ = assign([[0, 1]], [[2], [1, 2], [4, 5]], src=[0])
    assert got.tolist() == [[2, 2]]
    # token 0, slot 1 must open a node: replica (t + j) mod 2 = 1 -> rank 5, not rank 4
    got, _ = assign([[0, 2]], [[0], [1, 2], [4, 5]], src=[0])
    assert got.tolist() == [[0, 5]]
