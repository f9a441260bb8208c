"""plan_dispatch_noalloc -- the planner for callers that cannot allocate device memory
(a runtime that owns all device memory through its own pool or fixed memory plan, or a
caller that cannot afford cudaMalloc's device-wide synchronisation).  It uses the
library's own file-scope device scratch instead of a workspace; its results must be
those of plan_dispatch, and both must be the oracle's.  Calls in a row check that the
scratch, which keeps the previous call's contents, leaks nothing into the next call --
also when the calls are enqueued back to back with no synchronisation between them,
where one call's first kernel may start while the previous call's last kernel still
reads the scratch.

This file is collected last on purpose (pytest orders files by name)."""
import numpy as np
import pytest
import torch

import oracle
import workload

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
FIELDS = ("rank_counts", "rank_offsets", "asg_offsets", "rank_mask", "send_row", "comb_row",
          "stats", "src_dst")


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU test"
    import co_activation_b200 as c
    return c


def _to(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _enqueue(coact, fn, r, ids=None, src=None, cap=None):
    """Enqueues one plan (no synchronisation); returns (plan, err_flag)."""
    cfg = r.cfg
    ids = r.ids if ids is None else ids
    plan = coact.alloc_plan(len(ids), r.k, cfg.E, cfg.R, DEV, row_capacity=cap)
    plan.row_token.fill_(-7)
    plan.row_kmask.fill_(0xEE)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    fn(_to(ids), cfg.E, _to(r.expert_rank), cfg.R, plan, rank_node=_to(r.rank_node),
       n_nodes=cfg.n_nodes, src_rank=None if src is None else _to(src), err_flag=err)
    return plan, err


def _assert_equal_plans(got, want, tag):
    for f in FIELDS:
        assert torch.equal(getattr(got, f), getattr(want, f)), (tag, f)
    assert torch.equal(got.row_token, want.row_token), tag     # incl. untouched rows past D
    assert torch.equal(got.row_kmask, want.row_kmask), tag


def _assert_oracle(plan, r, ids=None, src=None, cap=None):
    cfg = r.cfg
    ids = r.ids if ids is None else ids
    o = oracle.plan(ids, cfg.E, r.expert_rank, cfg.R, rank_node=r.rank_node, n_nodes=cfg.n_nodes,
                    src_rank=src, row_capacity=cap)
    for f in ("rank_counts", "rank_offsets", "asg_offsets", "send_row", "comb_row", "stats",
              "src_dst"):
        assert np.array_equal(getattr(plan, f).cpu().numpy(), o[f]), f
    assert np.array_equal(plan.rank_mask.cpu().numpy().view(np.uint64), o["rank_mask"])
    n = min(o["D"], o["row_capacity"])
    rt, km = plan.row_token.cpu().numpy(), plan.row_kmask.cpu().numpy()
    assert np.array_equal(rt[:n], o["row_token"][:n]) and np.array_equal(km[:n], o["row_kmask"][:n])
    assert (rt[n:] == -7).all() and (km[n:] == 0xEE).all()     # nothing written past D
    return o["flags"]


def test_noalloc_matches_plan_dispatch_on_two_calls_in_a_row(coact):
    # a large batch first (fills most of the scratch), then a small one
    for cfg in (2, 0):
        r = workload.make_routing(cfg)
        want, e1 = _enqueue(coact, coact.plan_dispatch, r)
        got, e2 = _enqueue(coact, coact.plan_dispatch_noalloc, r)
        torch.cuda.synchronize()
        assert e1.item() == e2.item() == 0
        _assert_equal_plans(got, want, cfg)
        assert _assert_oracle(got, r) == 0


@pytest.mark.parametrize("order", [(2, 0), (0, 2), (3, 1, 2)])
def test_noalloc_back_to_back_without_sync(coact, order):
    """Different batches planned back to back on one stream with no synchronisation:
    config 2 and 3 take the three-launch planner (scan kernel), configs 0 and 1 the
    two-launch one; each result equals plan_dispatch's and the oracle's."""
    routings = [workload.make_routing(c) for c in order]
    got = [_enqueue(coact, coact.plan_dispatch_noalloc, r) for r in routings]
    torch.cuda.synchronize()
    for r, (plan, err) in zip(routings, got):
        assert err.item() == 0
        want, _ = _enqueue(coact, coact.plan_dispatch, r)
        torch.cuda.synchronize()
        _assert_equal_plans(plan, want, r.cfg.index)
        assert _assert_oracle(plan, r) == 0


def test_noalloc_batch_that_fills_the_scratch(coact):
    """N = NOALLOC_MAX_TOKENS tokens over R = 64 ranks: the scratch is used to its end."""
    r = workload.make_routing(3, N=coact.NOALLOC_MAX_TOKENS)
    assert r.cfg.R == coact.MAX_R
    plan, err = _enqueue(coact, coact.plan_dispatch_noalloc, r)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert _assert_oracle(plan, r) == 0
    want, _ = _enqueue(coact, coact.plan_dispatch, r)
    torch.cuda.synchronize()
    _assert_equal_plans(plan, want, "full")


def test_noalloc_flags_invalid_tokens_home_ranks_and_capacity(coact):
    """Invalid ids, repeated ids and home ranks out of range (with a src_rank array), then a
    row capacity too small for the batch: the same flags and outputs as the oracle."""
    r = workload.make_routing(1, N=3001)
    ids = r.ids.copy()
    ids[5, 1] = 99
    ids[6, 1] = ids[6, 0]
    src = np.random.default_rng(4).integers(0, r.cfg.R, r.N).astype(np.int32)
    src[7] = r.cfg.R
    src[8] = -1
    plan, err = _enqueue(coact, coact.plan_dispatch_noalloc, r, ids=ids, src=src)
    torch.cuda.synchronize()
    f = _assert_oracle(plan, r, ids=ids, src=src)
    assert f == err.item() == (oracle.FLAG_ID_RANGE | oracle.FLAG_DUP_ID | oracle.FLAG_SRC_RANK)
    cap = 1000
    plan, err = _enqueue(coact, coact.plan_dispatch_noalloc, r, src=src[::-1].copy() % r.cfg.R,
                         cap=cap)
    torch.cuda.synchronize()
    f = _assert_oracle(plan, r, src=src[::-1].copy() % r.cfg.R, cap=cap)
    assert f == err.item() == oracle.FLAG_CAPACITY


def test_noalloc_rejects_batches_beyond_its_scratch(coact):
    N = coact.NOALLOC_MAX_TOKENS + 1
    ids = torch.zeros((N, 2), dtype=torch.int32, device=DEV)
    plan = coact.alloc_plan(N, 2, 8, 4, DEV, row_capacity=16)
    with pytest.raises(ValueError, match="at most"):
        coact.plan_dispatch_noalloc(ids, 8, torch.zeros(8, dtype=torch.int32, device=DEV), 4, plan)
    # and the C ABI refuses it on the host, before enqueuing anything
    status = coact._lib.plan_dispatch_noalloc(
        coact._ptr(ids), N, 2, 8, coact._ptr(torch.zeros(8, dtype=torch.int32, device=DEV)), 4,
        None, 1, None, coact._ptr(plan.rank_counts), coact._ptr(plan.rank_offsets),
        coact._ptr(plan.asg_offsets), None, coact._ptr(plan.row_token), coact._ptr(plan.row_kmask),
        16, coact._ptr(plan.send_row), coact._ptr(plan.comb_row), coact._ptr(plan.stats), None,
        None, coact._stream(None))
    assert status == coact.ERR_UNSUPPORTED
