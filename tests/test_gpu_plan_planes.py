"""The planner's per-warp rank tables at their edges, against the oracle's plan.

The planner builds, per warp of 32 tokens, each token's per-rank slot counts as bit planes
(one plane per count bit: four for k = 8, where a count reaches 8 only when all of a
token's experts sit on one rank) over one 32-bit word per 32 ranks (one word for R <= 32,
two above), and transposes them across the warp.  These cases reach every plane and both
words: all slots of many tokens on one rank (count 8, on low and high ranks), R = 1, 2,
32, 33, 48 and 64, placements skewed onto one rank, several home ranks inside one warp
(the split-matrix groups), invalid tokens between valid ones (lanes without planes), and
batch sizes on both planner paths (the scan folded into the scatter kernel, and the
three-launch path) with ragged last tiles.  Every output is compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, assert_plan_equal, plan_to_host, run_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def _routing(ids, E, er, R, nodes, src, k):
    N = ids.shape[0]
    cfg = workload.CONFIGS[0].with_(N=N, E=E, k=k, R=R, n_nodes=nodes)
    rn = (np.arange(R) * nodes // R).astype(np.int32)
    return workload.Routing(cfg=cfg, ids=ids, gates=np.full((N, k), 1.0 / k, np.float32),
                            expert_rank=er, rank_node=rn, src_rank=src,
                            groups=np.zeros((0, 2), np.int32), planted=np.zeros(N, bool),
                            seed=0)


def _ids_same_rank(rng, N, E, k, er, R, share):
    """Top-k-like ids (distinct per token); a `share` of the tokens takes all k experts
    from one rank (a random rank holding at least k experts)."""
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    members = [np.flatnonzero(er == r) for r in range(R)]
    full = [r for r in range(R) if len(members[r]) >= k]
    if full and share > 0:
        pick = np.flatnonzero(rng.random(N) < share)
        for t in pick:
            r = full[rng.integers(len(full))]
            ids[t] = rng.choice(members[r], size=k, replace=False)
    return ids


CASES = [
    # N, E, k, R, nodes, placement, share of tokens with all k slots on one rank, src
    (3001, 16, 8, 1, 1, "contiguous", 0.0, "blocks"),       # one rank: every count is k
    (5000, 16, 8, 2, 1, "skew", 0.5, "blocks"),             # 15 experts on rank 0
    (9000, 256, 8, 32, 4, "contiguous", 0.4, "blocks"),     # one word, counts of 8
    (9000, 264, 8, 33, 4, "contiguous", 0.4, "random"),     # two words, rank 32 alone above
    (20000, 512, 8, 64, 8, "contiguous", 0.4, "blocks"),    # scan path, counts of 8 up high
    (12345, 512, 8, 64, 8, "contiguous", 0.3, "random"),    # many home ranks per warp
    (7777, 64, 7, 64, 8, "permuted", 0.0, "random"),        # one expert per rank
    (6000, 200, 5, 48, 6, "skew", 0.2, "random"),
    (4099, 1024, 1, 64, 8, "permuted", 0.0, "blocks"),      # k = 1: one plane
    (16385, 96, 3, 40, 5, "permuted", 0.3, "random"),       # three slots: two planes
]


@pytest.mark.parametrize("N,E,k,R,nodes,placement,share,src_kind", CASES)
def test_plan_bit_planes(coact, N, E, k, R, nodes, placement, share, src_kind):
    rng = np.random.default_rng(N + 31 * R + k)
    if placement == "contiguous":
        er = (np.arange(E) * R // E).astype(np.int32)
    elif placement == "permuted":
        er = (rng.permutation(E) % R).astype(np.int32)
    else:                      # all but one expert per other rank on rank 0
        er = np.zeros(E, np.int32)
        er[:R - 1] = np.arange(1, R, dtype=np.int32) if R > 1 else 0
        er = rng.permutation(er).astype(np.int32)
    ids = _ids_same_rank(rng, N, E, k, er, R, share)
    src = (rng.integers(0, R, N) if src_kind == "random"
           else (np.arange(N) * R // N)).astype(np.int32)
    r = _routing(ids, E, er, R, nodes, src, k)
    o = oracle.plan(ids, E, er, R, rank_node=r.rank_node, n_nodes=nodes, src_rank=src)
    assert o["flags"] == 0
    if share > 0 and R > 1:    # the case reaches counts of k on one rank
        assert any((er[ids[t]] == er[ids[t, 0]]).all() for t in range(min(N, 500)))
    plan, err = run_plan(coact, r, src_rank=src)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(plan), o)


@pytest.mark.parametrize("R", [32, 64])
def test_plan_bit_planes_invalid_lanes(coact, R):
    """Invalid tokens (an id out of range, a repeated id, a home rank out of range) between
    valid ones with all slots on one rank: the invalid lanes add nothing to any table."""
    rng = np.random.default_rng(R)
    N, E, k, nodes = 4133, 8 * R, 8, 8
    er = (np.arange(E) * R // E).astype(np.int32)
    ids = _ids_same_rank(rng, N, E, k, er, R, 0.5)
    src = rng.integers(0, R, N).astype(np.int32)
    bad = rng.choice(N, 300, replace=False)
    ids[bad[:100], 3] = E + 5                       # out of range
    ids[bad[100:200], 5] = ids[bad[100:200], 2]     # repeated within the token
    src[bad[200:]] = R + 1                          # home rank out of range
    r = _routing(ids, E, er, R, nodes, src, k)
    o = oracle.plan(ids, E, er, R, rank_node=r.rank_node, n_nodes=nodes, src_rank=src)
    plan, err = run_plan(coact, r, src_rank=src)
    assert err.item() == o["flags"] == (oracle.FLAG_ID_RANGE | oracle.FLAG_DUP_ID
                                        | oracle.FLAG_SRC_RANK)
    assert_plan_equal(plan_to_host(plan), o)
