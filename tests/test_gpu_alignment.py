"""Buffers that are 16-byte but not 32-byte aligned through every kernel with a 32-byte
path (the gather, the combine, combine_rows, the transposed dispatch, the combine backward,
the two-hop forward).  The library takes 256-bit accesses only when every row pointer it
would use is 32-byte aligned, which it checks on the host; any other buffer the ABI accepts
(16-byte aligned) must take the 16-byte path and give the same bits.  Each call runs twice,
on aligned buffers and on views shifted by 16 bytes, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import DEV, cuda, host_bits, run_plan

pytestmark = pytest.mark.gpu

H = 256                     # H % 16 == 0: only the pointers decide the path


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def shifted(rows, dtype=torch.bfloat16, shift_bytes=16, fill=None):
    """A [rows, H] tensor whose data starts 16 bytes past a 32-byte boundary (or on one,
    shift_bytes=0), as a view into a larger buffer."""
    esize = torch.tensor([], dtype=dtype).element_size()
    off = shift_bytes // esize
    buf = torch.zeros(rows * H + off + 64, dtype=dtype, device=DEV)
    t = buf[off:off + rows * H].view(rows, H)
    assert t.data_ptr() % 32 == shift_bytes % 32
    if fill is not None:
        t.copy_(fill)
    return t


@pytest.fixture(scope="module")
def case(coact):
    r = workload.make_routing(2, N=3001)
    c = r.cfg
    plan, _ = run_plan(coact, r, sentinel=False)
    o = oracle.plan(r.ids, c.E, r.expert_rank, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    x = workload.fill_bf16(r.N, H, 0, 1, device=DEV)
    y = workload.fill_bf16(r.N * r.k, H, 0, 2, device=DEV)
    return r, plan, o, x, y


@pytest.mark.parametrize("shift", [0, 16])
def test_gather_and_combine(coact, case, shift):
    r, plan, o, x0, y0 = case
    D = o["D"]
    x = shifted(r.N, shift_bytes=shift, fill=x0)
    send = shifted(plan.row_capacity, shift_bytes=shift)
    coact.dispatch_gather(x, plan.send_row, send)
    y = shifted(r.N * r.k, shift_bytes=shift, fill=y0)
    for dt in (torch.bfloat16, torch.float32):
        out = shifted(r.N, dtype=dt, shift_bytes=shift)
        coact.combine_scatter(y, cuda(r.gates), plan.comb_row, out)
        torch.cuda.synchronize()
        chain = oracle.combine_f32chain(host_bits(y0), r.gates, o["comb_row"])
        if dt == torch.float32:
            assert np.array_equal(out.cpu().numpy().view(np.uint32), chain.view(np.uint32))
        else:
            assert np.array_equal(host_bits(out), oracle.bf16_rne(chain))
    assert np.array_equal(host_bits(send)[:D], oracle.gather(host_bits(x0), o["row_token"], D))


@pytest.mark.parametrize("shift", [0, 16])
def test_units_transpose_and_backward(coact, case, shift):
    r, plan, o, x0, y0 = case
    D = o["D"]
    y = shifted(r.N * r.k, shift_bytes=shift, fill=y0)
    pre = shifted(D, dtype=torch.float32, shift_bytes=shift)
    coact.combine_rows(y, cuda(r.gates), plan.comb_row, plan.row_token, plan.row_kmask, pre)
    g0 = workload.fill_bf16(D, H, 0, 5, device=DEV)
    g = shifted(D, shift_bytes=shift, fill=g0)
    gx = shifted(r.N, dtype=torch.float32, shift_bytes=shift)
    coact.dispatch_gather_backward(g, plan.send_row, gx)
    go0 = workload.fill_bf16(r.N, H, 0, 6, device=DEV)
    go = shifted(r.N, shift_bytes=shift, fill=go0)
    gy = shifted(r.N * r.k, shift_bytes=shift)
    gg = torch.empty((r.N, r.k), dtype=torch.float32, device=DEV)
    coact.combine_scatter_backward(y, cuda(r.gates), plan.comb_row, go, gy, gg)
    torch.cuda.synchronize()
    want_pre = oracle.combine_units_f32chain(host_bits(y0), r.gates, o["comb_row"],
                                             o["row_token"], o["row_kmask"], D)
    assert np.array_equal(pre.cpu().numpy().view(np.uint32), want_pre.view(np.uint32))
    want_gx = oracle.gather_backward_f32chain(host_bits(g0), o["send_row"])
    assert np.array_equal(gx.cpu().numpy().view(np.uint32), want_gx.view(np.uint32))
    gy_o, gg_o, ga_o = oracle.combine_backward(host_bits(y0), r.gates, o["comb_row"],
                                               host_bits(go0))
    assert np.array_equal(host_bits(gy), gy_o)
    m = 16                      # terms per lane at H = 256 on either path
    assert (np.abs(gg.cpu().numpy().astype(np.float64) - gg_o)
            <= 1.01 * (m + 5) * 2.0 ** -24 * ga_o + 1e-30).all()


@pytest.mark.parametrize("shift", [0, 16])
def test_two_hop_forward(coact, shift):
    r = workload.make_routing(2, N=2000)
    c = r.cfg
    th = coact.alloc_two_hop(r.N, r.k, c.E, c.R, c.n_nodes, DEV)
    coact.plan_two_hop(cuda(r.ids), c.E, cuda(r.expert_rank, np.int32), c.R,
                       cuda(r.rank_node, np.int32), c.n_nodes, th)
    node_o, rank_o, fwd_o = oracle.plan_two_hop(r.ids, c.E, r.expert_rank, c.R, r.rank_node,
                                                c.n_nodes)
    h0 = workload.fill_bf16(th.node.row_capacity, H, 0, 3, device=DEV)
    hop1 = shifted(th.node.row_capacity, shift_bytes=shift, fill=h0)
    hop2 = shifted(th.rank.row_capacity, shift_bytes=shift)
    coact.forward_gather_tokens(hop1, th.rank.send_row, th.fwd_src, hop2)
    torch.cuda.synchronize()
    D = rank_o["D"]
    want = oracle.forward_gather(host_bits(h0), fwd_o)
    assert np.array_equal(host_bits(hop2)[:D], want[:D])
