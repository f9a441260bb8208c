"""The benchmark's own steps at full size against the oracle, every output in full.

bench.py times these step objects (count on a side stream, plan, gather, combine; config
4 as two consecutive layers with token shuffling).  Here each step runs once on the
GPU, then the oracle runs the same chain from the same generated inputs and every
output is compared: counts, placements, predicted homes and plans bit-exact, every
gathered row bit-exact, every combined row bit-identical to the fixed-order fp32 chain
(and within the stated tolerance of the float64 reference).

Config 3 uses the co-activation-grouped placement (Zyphra, English abstract: experts
often selected together placed on the same GPU) that the library builds from the
batch's own pair counts; the oracle builds its own from its own counts.  Config 4 is
the token-shuffling chain (Zyphra, English abstract: tokens moved to the GPU predicted
to hold their next-layer experts): layer 1's combined rows are layer 2's input rows,
and layer 2's tokens are homed on the rank predicted from cross-layer counts of a
calibration batch."""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import (DEV, assert_plan_equal, check_combine_complete, check_gather_complete,
                       host_bits, plan_to_host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


@pytest.fixture(scope="module")
def bench():
    import bench as b
    return b


@pytest.mark.parametrize("cfg", [1, 3])
def test_bench_one_layer_step(coact, bench, cfg):
    S, _ = bench.make_step(coact, cfg, 0, DEV)
    L, c = S.L, S.cfg
    L.send.view(torch.int16).fill_(-1)
    S.step()
    torch.cuda.synchronize()
    assert L.err.item() == 0
    r = L.r
    op, ol, f = oracle.count(r.ids, c.E)
    assert f == 0
    assert np.array_equal(L.pair.cpu().numpy(), op)
    assert np.array_equal(L.loads.cpu().numpy(), ol)
    if cfg == 3:   # the oracle's own placement from its own counts
        er = oracle.place_correlated(op, c.R)
        assert np.array_equal(er, r.expert_rank), "correlated placement"
    else:
        er = r.expert_rank
    o = oracle.plan(r.ids, c.E, er, c.R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    assert o["flags"] == 0
    assert_plan_equal(plan_to_host(L.plan), o, sentinel=False)
    D = o["D"]
    check_gather_complete(L.send, host_bits(L.x), o["row_token"], D)
    if D < L.send.shape[0]:
        assert (L.send[D:].view(torch.int16) == -1).all().item(), "row past D written"
    check_combine_complete(L.out, L.y, r.gates, o["comb_row"])


def test_bench_two_layer_step_config4(coact, bench):
    S, _ = bench.make_step(coact, 4, 0, DEV)
    c, tl = S.cfg, S.tl
    E, R = c.E, c.R
    S.L1.send.view(torch.int16).fill_(-1)
    S.L2.send.view(torch.int16).fill_(-1)
    S.step()
    torch.cuda.synchronize()
    assert S.L1.err.item() == 0 and S.L2.err.item() == 0
    l1, l2 = tl.layer1, tl.layer2

    # statistics: both layers' pair counts and the live cross-layer counts
    for L, lr in ((S.L1, l1), (S.L2, l2)):
        op, ol, _ = oracle.count(lr.ids, E)
        assert np.array_equal(L.pair.cpu().numpy(), op)
        assert np.array_equal(L.loads.cpu().numpy(), ol)
    live, _, _ = oracle.count_cross(l1.ids, E, l2.ids, E)
    assert np.array_equal(S.C12_live.cpu().numpy(), live)

    # the prediction: calibration counts -> predicted layer-2 home rank
    oc, _, _ = oracle.count_cross(tl.calib1, E, tl.calib2, E)
    assert np.array_equal(S.C12.cpu().numpy(), oc)
    home, f = oracle.predict_home(l1.ids, E, oc, l2.expert_rank, R)
    assert f == 0
    assert np.array_equal(S.home.cpu().numpy(), home)

    # layer 1 (contiguous home ranks)
    p1 = oracle.plan(l1.ids, E, l1.expert_rank, R, rank_node=l1.rank_node, n_nodes=c.n_nodes)
    assert_plan_equal(plan_to_host(S.L1.plan), p1, sentinel=False)
    check_gather_complete(S.L1.send, host_bits(S.L1.x), p1["row_token"], p1["D"])
    check_combine_complete(S.L1.out, S.L1.y, l1.gates, p1["comb_row"])
    # the oracle's layer-1 output, rounded to bf16 as the rows layer 2 reads
    x2 = oracle.bf16_rne(oracle.combine_f32chain(host_bits(S.L1.y), l1.gates, p1["comb_row"]))
    assert np.array_equal(host_bits(S.L1.out), x2)

    # layer 2, tokens homed on the predicted rank; its input rows are the oracle's x2
    p2 = oracle.plan(l2.ids, E, l2.expert_rank, R, rank_node=l2.rank_node, n_nodes=c.n_nodes,
                     src_rank=home)
    assert p2["flags"] == 0
    assert_plan_equal(plan_to_host(S.L2.plan), p2, sentinel=False)
    check_gather_complete(S.L2.send, x2, p2["row_token"], p2["D"])
    if p2["D"] < S.L2.send.shape[0]:
        assert (S.L2.send[p2["D"]:].view(torch.int16) == -1).all().item()
    check_combine_complete(S.L2.out, S.L2.y, l2.gates, p2["comb_row"])
    # the point of the prediction: more layer-2 assignments served on the token's rank
    base = oracle.plan(l2.ids, E, l2.expert_rank, R, rank_node=l2.rank_node, n_nodes=c.n_nodes)
    assert p2["stats"][5] > 2 * base["stats"][5]


def test_bench_hbm_mix_line():
    """`bench.py --hbm-mix` (the per-mix HBM figures behind the roofline's context) runs
    through the library's gather and combine and prints one JSON line with every mix."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--hbm-mix",
                        "--mix-gb", "0.5", "--steps", "5", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=root)
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    mix = line["hbm_mix"]
    want = {"torch_copy", "torch_sum"} | {f"gather_fanout{f}" for f in (1, 2, 4, 8)} | \
        {f"combine_k{k}{s}" for k in (1, 2, 4, 8) for s in ("", "_random_rows")}
    assert set(mix) == want
    for name, v in mix.items():
        assert 0 <= v["write_share"] <= 0.5 or name.startswith("gather")
        assert v["GBps"] > 500, (name, v)     # half a GB per launch still streams at TB/s
    f8 = mix["gather_fanout8"]["write_share"]
    assert abs(f8 - 8 / 9) < 0.01 and abs(mix["combine_k8"]["write_share"] - 1 / 9) < 0.01
