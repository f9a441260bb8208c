"""plan_dispatch_noalloc -- the planner for callers that cannot allocate device memory
(a runtime that owns all device memory through its own pool or fixed memory plan, or a
caller that cannot afford cudaMalloc's device-wide synchronisation).  It uses the
library's own file-scope device scratch instead of a workspace; its results must be
those of plan_dispatch.  Two different calls in a row check that the scratch, which
keeps the previous call's contents, leaks nothing into the next call.

This file is collected last on purpose (pytest orders files by name)."""
import numpy as np
import pytest
import torch

import workload

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
FIELDS = ("rank_counts", "rank_offsets", "asg_offsets", "rank_mask", "send_row", "comb_row",
          "stats", "src_dst")


def _inputs(r):
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)
    return to(r.ids), to(r.expert_rank), to(r.rank_node)


def _plan(coact, fn, r, ids, er, rn):
    cfg = r.cfg
    plan = coact.alloc_plan(r.N, r.k, cfg.E, cfg.R, DEV)
    plan.row_token.fill_(-7)
    plan.row_kmask.fill_(0xEE)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    fn(ids, cfg.E, er, cfg.R, plan, rank_node=rn, n_nodes=cfg.n_nodes, err_flag=err)
    torch.cuda.synchronize()
    return plan, err.item()


def test_noalloc_matches_plan_dispatch_on_two_calls_in_a_row():
    assert torch.cuda.is_available(), "GPU test"
    import co_activation_b200 as coact
    # a large batch first (fills most of the scratch), then a small one
    for cfg in (2, 0):
        r = workload.make_routing(cfg)
        ids, er, rn = _inputs(r)
        want, e1 = _plan(coact, coact.plan_dispatch, r, ids, er, rn)
        got, e2 = _plan(coact, coact.plan_dispatch_noalloc, r, ids, er, rn)
        assert e1 == e2 == 0
        for f in FIELDS:
            assert torch.equal(getattr(got, f), getattr(want, f)), (cfg, f)
        assert torch.equal(got.row_token, want.row_token)      # incl. untouched rows past D
        assert torch.equal(got.row_kmask, want.row_kmask)


def test_noalloc_rejects_batches_beyond_its_scratch():
    import co_activation_b200 as coact
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
