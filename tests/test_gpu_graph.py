"""The path inside a CUDA graph, captured as the very first library calls of a fresh
process (per-device caches cold): the library enqueues everything on the given stream
with no allocation and no host synchronisation, so capture must succeed and every
replay must equal the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys
sys.path.insert(0, ROOT)
import numpy as np, torch
import oracle, workload
import co_activation_b200 as coact
dev = torch.device("cuda", 0)
r = workload.make_routing(1, N=3000)
c = r.cfg
H = 256
to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
ids, er, rn, gates = to(r.ids), to(r.expert_rank.astype(np.int32)), to(r.rank_node.astype(np.int32)), to(r.gates)
x = workload.fill_bf16(r.N, H, 0, 1, device=dev)
y = workload.fill_bf16(r.N * r.k, H, 0, 2, device=dev)
plan = coact.alloc_plan(r.N, r.k, c.E, c.R, dev)
send = torch.zeros((plan.row_capacity, H), dtype=torch.bfloat16, device=dev)
out = torch.zeros((r.N, H), dtype=torch.float32, device=dev)
pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=dev)
loads = torch.zeros(c.E, dtype=torch.int64, device=dev)
err = torch.zeros(1, dtype=torch.int32, device=dev)
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):          # first library calls of this process
    pair.zero_(); loads.zero_()
    coact.coact_count(ids, c.E, pair, loads, err_flag=err)
    coact.plan_dispatch(ids, c.E, er, c.R, plan, rank_node=rn, n_nodes=c.n_nodes, err_flag=err)
    coact.dispatch_gather(x, plan.send_row, send, err_flag=err)
    coact.combine_scatter(y, gates, plan.comb_row, out, err_flag=err)
o = oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
op, ol, _ = oracle.count(r.ids, c.E)
xb = oracle._bits(x); yb = oracle._bits(y)
want_send = oracle.gather(xb, o["row_token"], o["D"])
want_out = oracle.combine_f32chain(yb, r.gates, o["comb_row"])
for rep in range(2):
    out.zero_(); send.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(pair.cpu().numpy(), op) and np.array_equal(loads.cpu().numpy(), ol)
    assert np.array_equal(plan.send_row.cpu().numpy(), o["send_row"])
    assert np.array_equal(oracle._bits(send)[:o["D"]], want_send)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want_out.view(np.uint32))
print("graph ok")
'''


def test_first_calls_captured_in_a_graph():
    code = SCRIPT.replace("ROOT", repr(ROOT), 1)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    assert "graph ok" in p.stdout


SCRIPT_STAGE2 = r'''
import sys
sys.path.insert(0, ROOT)
import numpy as np, torch
import oracle, workload
import co_activation_b200 as coact
dev = torch.device("cuda", 0)
r = workload.make_routing(2, N=5000)
c = r.cfg
H = 128
to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
op, ol, _ = oracle.count(r.ids, c.E)
en = oracle.place_correlated(op, c.n_nodes)            # stage 1: periodic, outside the step
ids, rn, en_d, gates = to(r.ids), to(r.rank_node.astype(np.int32)), to(en), to(r.gates)
x = workload.fill_bf16(r.N, H, 0, 1, device=dev)
y = workload.fill_bf16(r.N * r.k, H, 0, 2, device=dev)
plan = coact.alloc_plan(r.N, r.k, c.E, c.R, dev)
send = torch.zeros((plan.row_capacity, H), dtype=torch.bfloat16, device=dev)
out = torch.zeros((r.N, H), dtype=torch.float32, device=dev)
pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=dev)
loads = torch.zeros(c.E, dtype=torch.int64, device=dev)
er = torch.zeros(c.E, dtype=torch.int32, device=dev)
back = torch.zeros((r.N, r.k), dtype=torch.float32, device=dev)
err = torch.zeros(1, dtype=torch.int32, device=dev)
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):          # stage 2 every step, the first library calls of this process
    pair.zero_(); loads.zero_()
    coact.coact_count(ids, c.E, pair, loads, err_flag=err)
    coact.rebalance_ranks(loads, en_d, rn, c.n_nodes, out=er, err_flag=err)
    coact.plan_dispatch(ids, c.E, er, c.R, plan, rank_node=rn, n_nodes=c.n_nodes, err_flag=err)
    coact.dispatch_gather(x, plan.send_row, send, err_flag=err)
    coact.combine_scatter(y, gates, plan.comb_row, out, err_flag=err)
    ex, gt, sl = coact.plan_row_meta(plan, ids, gates, err_flag=err)
    coact.gather_row_slots(gt, plan.send_row, plan.row_kmask, out=back, err_flag=err)
want_er = oracle.rebalance_ranks(ol, en, r.rank_node)
o = oracle.plan(r.ids, c.E, want_er, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
xb = oracle._bits(x); yb = oracle._bits(y)
want_send = oracle.gather(xb, o["row_token"], o["D"])
want_out = oracle.combine_f32chain(yb, r.gates, o["comb_row"])
wex, wgt, _, _ = oracle.row_meta(o, r.ids, r.gates)
for rep in range(2):
    out.zero_(); send.zero_(); er.zero_(); back.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(er.cpu().numpy(), want_er)
    assert np.array_equal(plan.send_row.cpu().numpy(), o["send_row"])
    assert np.array_equal(oracle._bits(send)[:o["D"]], want_send)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want_out.view(np.uint32))
    assert np.array_equal(ex[:o["D"]].cpu().numpy(), wex)
    assert np.array_equal(back.cpu().numpy(), r.gates)   # every token valid: the gates return
print("graph ok")
'''


def test_per_step_stage2_and_row_metadata_captured_in_a_graph():
    """Cobalt's per-step stage 2 (fresh counts -> device rebalance -> plan over that
    placement) with gather, combine and the EP row metadata, captured as one CUDA graph
    as the first library calls of a fresh process: nothing in the step needs the host."""
    code = SCRIPT_STAGE2.replace("ROOT", repr(ROOT), 1)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    assert "graph ok" in p.stdout
