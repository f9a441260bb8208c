"""GPU parity of the EP row metadata (plan_row_meta, gather_row_slots) against the oracle,
bit for bit: on the configurations' full-size plans, on random small plans with invalid
tokens and empty rank segments, with and without a per-rank slot base, and the way
back of per-slot values to token order."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, cuda, run_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def _check(coact, r, plan, o, slot_base=None):
    D, k = o["D"], r.k
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ex, gt, sl = coact.plan_row_meta(plan, cuda(r.ids), cuda(r.gates),
                                     None if slot_base is None else cuda(slot_base, np.int32),
                                     err_flag=err)
    wex, wgt, wsl, f = oracle.row_meta(o, r.ids, r.gates, slot_base=slot_base)
    torch.cuda.synchronize()
    assert err.item() == f == 0
    assert np.array_equal(ex[:D].cpu().numpy(), wex)
    assert np.array_equal(gt[:D].cpu().numpy().view(np.uint32), wgt.view(np.uint32))
    assert np.array_equal(sl[:D].cpu().numpy(), wsl)
    # the way back: random per-slot values in send-row order to token order
    vals = np.random.default_rng(k).standard_normal((D, k)).astype(np.float32)
    out = coact.gather_row_slots(cuda(vals), plan.send_row, plan.row_kmask, err_flag=err)
    want, f = oracle.gather_row_slots(vals, o["send_row"], o["row_kmask"])
    torch.cuda.synchronize()
    assert err.item() == f == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_row_meta_full_size(coact, cfg):
    r = workload.make_routing(cfg)
    c = r.cfg
    plan, _ = run_plan(coact, r)
    o = oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    _check(coact, r, plan, o)
    # the receive-order base an EP rank uses: here 1000 * r - asg_offsets[r]
    base = (1000 * np.arange(c.R) - o["asg_offsets"][:c.R]).astype(np.int32)
    _check(coact, r, plan, o, slot_base=base)


@pytest.mark.parametrize("seed", range(8))
def test_row_meta_random(coact, seed):
    import types
    from test_gpu_random_chains import rand_ids
    rng = np.random.default_rng(seed)
    k = int(rng.integers(1, 9))
    E = int(rng.integers(k + 1, 300))
    R = int(rng.integers(1, 65))
    N = int(rng.integers(1, 5000))
    ids = rand_ids(rng, N, E, k)
    ids[0, 0] = E + 3                                  # an invalid token: no rows
    er = rng.integers(0, R, E).astype(np.int32)        # some ranks may hold nothing
    gates = rng.random((N, k)).astype(np.float32)
    plan = coact.alloc_plan(N, k, E, R, DEV)
    coact.plan_dispatch(cuda(ids), E, cuda(er), R, plan)
    o = oracle.plan(ids, E, er, R)
    base = rng.integers(-50, 50, R).astype(np.int32)
    r = types.SimpleNamespace(ids=ids, gates=gates, k=k)
    _check(coact, r, plan, o, slot_base=base)


def test_row_meta_flags_and_untouched_rows(coact):
    r = workload.make_routing(0, N=64)
    c = r.cfg
    plan, _ = run_plan(coact, r)
    o = oracle.plan(r.ids, c.E, r.expert_rank, c.R)
    D = o["D"]
    plan.row_token[3] = 10 ** 6                           # a token outside [0, N)
    bad = dict(o)
    bad["row_token"] = o["row_token"].copy()
    bad["row_token"][3] = 10 ** 6
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ex = torch.full((plan.row_capacity, r.k), 77, dtype=torch.int32, device=DEV)
    status = coact._lib.plan_row_meta(
        coact._ptr(plan.row_token), coact._ptr(plan.row_kmask), plan.row_capacity,
        coact._ptr(plan.rank_offsets), c.R, coact._ptr(cuda(r.ids)), None,
        coact._ptr(plan.comb_row), r.N, r.k, None, coact._ptr(ex), None, None, coact._ptr(err),
        coact._stream(None))
    assert status == 0
    wex, _, _, f = oracle.row_meta(bad, r.ids, r.gates)
    torch.cuda.synchronize()
    assert err.item() == f == coact.EFLAG_ROW_RANGE
    got = ex.cpu().numpy()
    assert np.array_equal(got[:D], wex) and (got[D:] == 77).all()    # rows past D untouched
    sr = plan.send_row.clone()
    sr[2, 0] = D + 5                                                 # beyond n_rows
    err.zero_()
    coact.gather_row_slots(torch.ones((D, r.k), dtype=torch.float32, device=DEV), sr,
                           plan.row_kmask, err_flag=err)
    assert err.item() == coact.EFLAG_ROW_RANGE
