"""The EP layer's GPU code on a real NCCL process group of one rank (one GPU): both
transports -- NCCL all-to-all and symmetric-memory peer access -- for dispatch, combine,
the pre-reduced combine, the backward and the token shuffle, against the single-GPU
library calls.  With one rank every exchange is local, so this exercises the layer's own
code (buffer rendezvous, barriers, the peer kernels' arguments) where a GPU group is not
available; the multi-rank exchange logic is covered by the gloo tests."""
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import datetime, os, sys
sys.path.insert(0, ROOT)
import numpy as np, torch
import torch.distributed as dist
import workload
import co_activation_b200 as coact
import co_activation_b200.ep as ep
dev = torch.device("cuda", 0)
torch.cuda.set_device(dev)
dist.init_process_group("nccl", rank=0, world_size=1, init_method="tcp://127.0.0.1:PORT",
                        timeout=datetime.timedelta(seconds=60), device_id=dev)
r = workload.make_routing(0)
c = r.cfg
H = 256
ids, gates = torch.from_numpy(r.ids).to(dev), torch.from_numpy(r.gates).to(dev)
er = torch.zeros(c.E, dtype=torch.int32, device=dev)          # one rank holds every expert
x = workload.fill_bf16(r.N, H, 0, 1, device=dev)
g_out = workload.fill_bf16(r.N, H, 0, 6, device=dev)
# the single-GPU library path with the same plan
p = coact.alloc_plan(r.N, r.k, c.E, 1, dev)
coact.plan_dispatch(ids, c.E, er, 1, p)
D = int(p.rank_offsets[-1].item())
send = torch.empty((p.row_capacity, H), dtype=torch.bfloat16, device=dev)
coact.dispatch_gather(x, p.send_row, send)
results = {}
for transport in ("nccl", "peer"):
    layer = ep.EPLayer(dist.group.WORLD, c.E, er, transport=transport)
    d = layer.dispatch(ids, x, gates=gates)
    assert torch.equal(d.rows.view(torch.int16), send[:D].view(torch.int16)), transport
    y = ep.expand_identity(d)
    out = layer.combine(y, gates, torch.empty((r.N, H), dtype=torch.float32, device=dev))
    want = torch.empty_like(out)
    coact.combine_scatter(y, gates, p.comb_row, want)
    assert torch.equal(out.view(torch.int32), want.view(torch.int32)), transport
    pre = layer.combine(y, gates, torch.empty((r.N, H), dtype=torch.float32, device=dev), reduce="rows")
    pr = torch.empty((D, H), dtype=torch.bfloat16, device=dev)
    coact.combine_rows(y, gates, p.comb_row, p.row_token, p.row_kmask, pr)
    want_pre = torch.empty_like(out)
    coact.dispatch_gather_backward(pr, p.send_row, want_pre)
    assert torch.equal(pre.view(torch.int32), want_pre.view(torch.int32)), transport
    gy, gg = layer.backward_combine(g_out, y)
    wgy, wgg = torch.empty_like(y), torch.empty_like(gates)
    coact.combine_scatter_backward(y, gates, p.comb_row, g_out, wgy, wgg)
    assert torch.equal(gy.view(torch.int16), wgy.view(torch.int16)), transport
    assert torch.equal(gg.view(torch.int32), wgg.view(torch.int32)), transport
    gx = layer.backward_dispatch(d.rows, torch.empty((r.N, H), dtype=torch.float32, device=dev))
    wgx = torch.empty_like(gx)
    coact.dispatch_gather_backward(send, p.send_row, wgx)
    assert torch.equal(gx.view(torch.int32), wgx.view(torch.int32)), transport
    home = torch.zeros(r.N, dtype=torch.int32, device=dev)
    rows, tok = layer.shuffle_reduce_scatter(x, home)
    assert torch.equal(tok, torch.arange(r.N, dtype=torch.int32, device=dev)), transport
    assert torch.equal(rows.view(torch.int16), x.view(torch.int16)), transport
    pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=dev)
    loads = torch.zeros(c.E, dtype=torch.int64, device=dev)
    layer.count(ids, pair, loads)
    assert int(loads.sum()) == r.N * r.k, transport
    torch.cuda.synchronize()
    del layer
dist.destroy_process_group()
print("ep single ok")
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_ep_layer_on_one_rank_both_transports():
    code = SCRIPT.replace("ROOT", repr(ROOT), 1).replace("PORT", str(_free_port()), 1)
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       cwd=ROOT, env=env)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    assert "ep single ok" in p.stdout
