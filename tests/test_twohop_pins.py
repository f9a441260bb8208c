"""Pins for the oracle's two-hop dispatch (Cobalt English abstract: routing tokens to
fewer remote nodes): a hand-worked case, the composition invariant (hop 1 then hop 2
delivers exactly the rows of the one-hop dispatch), and the cross-check that the
node-level plan's remote rows equal the rank-level plan's node-deduplicated rows."""
import numpy as np
import pytest

import oracle
import workload


def test_hand_worked_two_hop():
    # one token on experts {0, 2, 3}, each expert alone on its rank; ranks {0,1} on node
    # 0 and {2,3} on node 1; home rank 0.  Hop 1: one row per node (node 0, node 1);
    # hop 2: rank rows 0 (rank 0), 1 (rank 2), 2 (rank 3), fed by node rows 0, 1, 1.
    ids = np.array([[0, 2, 3]], np.int32)
    node, rank, fwd = oracle.plan_two_hop(ids, 4, np.arange(4), 4, [0, 0, 1, 1], 2, src_rank=[0])
    assert node["D"] == 2 and rank["D"] == 3
    assert node["row_token"][:2].tolist() == [0, 0]
    assert node["row_kmask"][:2].tolist() == [0b001, 0b110]
    assert fwd.tolist() == [0, 1, 1]
    assert node["stats"][2] == 1 and rank["stats"][3] == 2     # 1 remote node row, 2 remote rank rows


@pytest.mark.parametrize("cfg", [2, 3])
def test_composition_equals_one_hop(cfg):
    r = workload.make_routing(cfg, N=3000)
    c = r.cfg
    node, rank, fwd = oracle.plan_two_hop(r.ids, c.E, r.expert_rank, c.R, r.rank_node, c.n_nodes)
    x = oracle._bits(workload.fill_bf16(r.N, 64, 0, 1))
    hop1 = oracle.gather(x, node["row_token"], node["D"])
    hop2 = oracle.forward_gather(hop1, fwd)
    direct = oracle.gather(x, rank["row_token"], rank["D"])
    assert np.array_equal(hop2[:rank["D"]], direct)
    assert (fwd[rank["D"]:] == -1).all()
    assert node["D"] <= rank["D"]


@pytest.mark.parametrize("cfg", [2, 3])
def test_node_plan_counts_remote_nodes(cfg):
    r = workload.make_routing(cfg)
    c = r.cfg
    node, rank, fwd = oracle.plan_two_hop(r.ids, c.E, r.expert_rank, c.R, r.rank_node, c.n_nodes)
    # rows that leave the home node in hop 1 == (token, remote node) pairs of the rank plan
    assert node["stats"][2] == rank["stats"][4]
    # every rank row is fed by a node row of the same token on its rank's node
    D = rank["D"]
    rn = np.asarray(r.rank_node)
    rank_of_row = np.repeat(np.arange(c.R), np.diff(rank["rank_offsets"]))
    node_of_nrow = np.repeat(np.arange(c.n_nodes), np.diff(node["rank_offsets"]))
    assert (fwd[:D] >= 0).all() and (fwd[:D] < node["D"]).all()
    assert np.array_equal(node["row_token"][fwd[:D]], rank["row_token"][:D])
    assert np.array_equal(node_of_nrow[fwd[:D]], rn[rank_of_row])
