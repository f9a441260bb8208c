"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on the same
seeded inputs.  Integers, masks, offsets, positions and gathered rows must be
bit-exact; the combine must match the float64 reference within the stated tolerance
and the fixed-order fp32 chain bit for bit.  Full-size workloads are checked in full:
counts and plans directly, gathered and combined rows streamed in chunks against
the oracle, with the same launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import workload
from _gpu_util import (DEV, X_STREAM, Y_STREAM, assert_plan_equal, check_combine,
                       check_combine_complete, check_gather_complete, cuda, host_bits,
                       plan_to_host, run_plan)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def coact():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import co_activation_b200 as c
    return c


def zero_flag():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def oracle_plan_for(r, **kw):
    cfg = r.cfg
    args = dict(E=cfg.E, expert_rank=r.expert_rank, R=cfg.R, rank_node=r.rank_node,
                n_nodes=cfg.n_nodes, src_rank=None)
    args.update(kw)
    return oracle.plan(r.ids, args["E"], args["expert_rank"], args["R"],
                       rank_node=args["rank_node"], n_nodes=args["n_nodes"],
                       src_rank=args["src_rank"], row_capacity=args.get("row_capacity"))


# ----------------------------------------------------------------------------- counting


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_count_full_size(coact, cfg):
    r = workload.make_routing(cfg)
    E = r.cfg.E
    pair = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    loads = torch.zeros(E, dtype=torch.int64, device=DEV)
    err = zero_flag()
    ids = cuda(r.ids)
    coact.coact_count(ids, E, pair, loads, err_flag=err)
    op, ol, f = oracle.count(r.ids, E)
    assert f == 0 and err.item() == 0
    assert np.array_equal(pair.cpu().numpy(), op)
    assert np.array_equal(loads.cpu().numpy(), ol)
    coact.coact_count(ids, E, pair, loads)                 # accumulates
    assert np.array_equal(pair.cpu().numpy(), 2 * op)
    assert np.array_equal(loads.cpu().numpy(), 2 * ol)


@pytest.mark.parametrize("N,E,k", [(1, 8, 2), (37, 8, 3), (5000, 1024, 4), (3000, 300, 8),
                                   (70000, 32, 5), (2049, 256, 1)])
def test_count_shapes(coact, N, E, k):
    rng = np.random.default_rng(N + E + k)
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    pair = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    loads = torch.zeros(E, dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(ids), E, pair, loads)
    op, ol, _ = oracle.count(ids, E)
    assert np.array_equal(pair.cpu().numpy(), op) and np.array_equal(loads.cpu().numpy(), ol)


def test_count_flags_and_skips(coact):
    r = workload.make_routing(0)
    ids = r.ids.copy()
    ids[10, 0] = 8           # out of range
    ids[20, 1] = ids[20, 0]  # repeated
    ids[30, 0] = -1
    pair = torch.zeros((8, 8), dtype=torch.int64, device=DEV)
    loads = torch.zeros(8, dtype=torch.int64, device=DEV)
    err = zero_flag()
    coact.coact_count(cuda(ids), 8, pair, loads, err_flag=err)
    op, ol, f = oracle.count(ids, 8)
    assert err.item() == f == (coact.EFLAG_ID_RANGE | coact.EFLAG_DUP_ID)
    assert np.array_equal(pair.cpu().numpy(), op) and np.array_equal(loads.cpu().numpy(), ol)


def test_count_cross_full_size(coact):
    tl = workload.make_two_layer(4)
    E = tl.layer1.cfg.E
    C = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    l1 = torch.zeros(E, dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(tl.calib1), E, C, l1, ids2=cuda(tl.calib2), E2=E)
    oc, ol, f = oracle.count_cross(tl.calib1, E, tl.calib2, E)
    assert f == 0
    assert np.array_equal(C.cpu().numpy(), oc) and np.array_equal(l1.cpu().numpy(), ol)


def test_count_deterministic(coact):
    r = workload.make_routing(3)
    outs = []
    for _ in range(3):
        pair = torch.zeros((256, 256), dtype=torch.int64, device=DEV)
        coact.coact_count(cuda(r.ids), 256, pair)
        outs.append(pair.cpu().numpy())
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


# ----------------------------------------------------------------------------- plans


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_plan_full_size(coact, cfg):
    r = workload.make_routing(cfg)
    plan, err = run_plan(coact, r)
    o = oracle_plan_for(r)
    assert err.item() == 0 and o["flags"] == 0
    assert_plan_equal(plan_to_host(plan), o)


@pytest.mark.parametrize("variant", ["identity", "one_rank", "planted3", "random_src2",
                                     "two_nodes1", "ragged", "beyond_one_wave"])
def test_plan_variants(coact, variant):
    if variant == "identity":            # every expert alone on its rank: D == N*k
        r = workload.make_routing(0)
        kw = dict(E=8, expert_rank=np.arange(8, dtype=np.int32), R=8,
                  rank_node=np.zeros(8, np.int32), n_nodes=1)
    elif variant == "one_rank":          # one rank: nothing remote, D == N
        r = workload.make_routing(1)
        kw = dict(expert_rank=np.zeros(64, np.int32), R=1, rank_node=np.zeros(1, np.int32))
    elif variant == "planted3":
        r = workload.make_routing(3, placement_kind="planted")
        kw = {}
    elif variant == "random_src2":
        r = workload.make_routing(2)
        kw = dict(src_rank=np.random.default_rng(5).integers(0, 32, r.N).astype(np.int32))
    elif variant == "two_nodes1":
        r = workload.make_routing(1)
        kw = dict(rank_node=(np.arange(8) // 4).astype(np.int32), n_nodes=2)
    elif variant == "ragged":            # token counts that leave partial warps and tiles
        r = workload.make_routing(2, N=65536 - 4093)
        kw = {}
    else:                                # more tiles than fit on the GPU at once: the
        r = workload.make_routing(3, N=200003)   # planner's multi-launch path
        kw = {}
    o = oracle_plan_for(r, **kw)
    plan, err = run_plan(coact, r, E=kw.get("E"), expert_rank=kw.get("expert_rank"),
                         R=kw.get("R"), rank_node=kw.get("rank_node"),
                         n_nodes=kw.get("n_nodes"), src_rank=kw.get("src_rank"))
    assert err.item() == 0
    g = plan_to_host(plan)
    assert_plan_equal(g, o)
    if variant == "identity":
        assert g["rank_offsets"][-1] == r.N * r.k
    if variant == "one_rank":
        assert g["rank_offsets"][-1] == r.N and g["stats"][2] == 0


@pytest.mark.parametrize("N,E,k,R,nodes", [(1, 8, 2, 4, 1), (31, 16, 3, 4, 2), (257, 64, 8, 64, 8),
                                           (1000, 128, 6, 16, 4), (4096, 1024, 8, 64, 8),
                                           (513, 12, 1, 3, 1),
                                           # the one-cluster planner's edges: odd cluster
                                           # sizes, the largest batch it takes, the first
                                           # one it leaves to the multi-launch planner
                                           (8193, 64, 2, 8, 1), (12289, 256, 8, 64, 8),
                                           (32768, 64, 4, 32, 4), (32769, 64, 4, 32, 4)])
def test_plan_shapes(coact, N, E, k, R, nodes):
    rng = np.random.default_rng(N * 7 + k)
    cfg = workload.CONFIGS[0].with_(N=N, E=E, k=k, R=R, n_nodes=nodes)
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    er = (rng.permutation(E) % R).astype(np.int32)
    rn = (np.arange(R) * nodes // R).astype(np.int32)
    src = rng.integers(0, R, N).astype(np.int32)
    r = workload.Routing(cfg=cfg, ids=ids, gates=np.full((N, k), 1.0 / k, np.float32),
                         expert_rank=er, rank_node=rn, src_rank=src,
                         groups=np.zeros((0, 2), np.int32), planted=np.zeros(N, bool), seed=0)
    o = oracle.plan(ids, E, er, R, rank_node=rn, n_nodes=nodes, src_rank=src)
    plan, err = run_plan(coact, r, src_rank=src)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(plan), o)


def test_plan_empty(coact):
    cfg = workload.CONFIGS[0].with_(N=0)
    r = workload.Routing(cfg=cfg, ids=np.zeros((0, 2), np.int32), gates=np.zeros((0, 2), np.float32),
                         expert_rank=np.arange(8, dtype=np.int32) // 2,
                         rank_node=np.zeros(4, np.int32), src_rank=np.zeros(0, np.int32),
                         groups=np.zeros((0, 2), np.int32), planted=np.zeros(0, bool), seed=0)
    plan, err = run_plan(coact, r, sentinel=False)
    assert err.item() == 0
    assert plan.rank_offsets.cpu().tolist() == [0] * 5
    assert plan.stats.cpu().tolist() == [0] * 8


def test_plan_capacity_overflow(coact):
    r = workload.make_routing(1)
    full = oracle_plan_for(r)
    cap = full["D"] - 1000
    o = oracle_plan_for(r, row_capacity=cap)
    plan, err = run_plan(coact, r, row_capacity=cap)
    assert err.item() == coact.EFLAG_CAPACITY and o["flags"] == oracle.FLAG_CAPACITY
    assert_plan_equal(plan_to_host(plan), o, sentinel=False)


def test_plan_invalid_tokens(coact):
    r = workload.make_routing(0)
    ids = r.ids.copy()
    ids[5, 1] = 99
    ids[6, 1] = ids[6, 0]
    src = r.src_rank.copy()
    src[7] = 4
    r2 = workload.Routing(**{**r.__dict__, "ids": ids})
    o = oracle_plan_for(r2, src_rank=src)
    plan, err = run_plan(coact, r2, src_rank=src)
    assert err.item() == o["flags"] == (oracle.FLAG_ID_RANGE | oracle.FLAG_DUP_ID | oracle.FLAG_SRC_RANK)
    assert_plan_equal(plan_to_host(plan), o)


def test_plan_deterministic(coact):
    r = workload.make_routing(3)
    a = plan_to_host(run_plan(coact, r)[0])
    b = plan_to_host(run_plan(coact, r)[0])
    for key in a:
        assert np.array_equal(a[key], b[key]), key


# ----------------------------------------------------------------------------- gather


def _gather(coact, r, H, plan, sentinel_rows=True, tma=False):
    x = workload.fill_bf16(r.N, H, r.seed, X_STREAM, device=DEV)
    send = torch.empty((plan.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    if sentinel_rows:
        send.view(torch.int16).fill_(-1)
    err = zero_flag()
    coact.dispatch_gather(x, plan.send_row, send, err_flag=err, tma=tma)
    torch.cuda.synchronize()
    return x, send, err


@pytest.mark.parametrize("cfg,tma", [(0, False), (1, False), (1, True)])
def test_gather_full(coact, cfg, tma):
    r = workload.make_routing(cfg)
    H = r.cfg.H
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    x, send, err = _gather(coact, r, H, plan, tma=tma)
    assert err.item() == 0
    xh = host_bits(workload.fill_bf16(r.N, H, r.seed, X_STREAM))
    want = oracle.gather(xh, o["row_token"], o["D"])
    got = host_bits(send)
    assert np.array_equal(got[:o["D"]], want)
    assert (got[o["D"]:] == 0xFFFF).all()                   # rows past D untouched


@pytest.mark.parametrize("cfg,tma", [(2, False), (3, False), (3, True)])
def test_gather_full_size_complete(coact, cfg, tma):
    """Configs 2 and 3 at full size: every gathered row against the oracle (streamed in
    chunks), and every row past D untouched."""
    r = workload.make_routing(cfg)
    H = r.cfg.H
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    x, send, err = _gather(coact, r, H, plan, tma=tma)
    assert err.item() == 0
    D, cap = o["D"], plan.row_capacity
    check_gather_complete(send, host_bits(x), o["row_token"], D)
    if D < cap:
        assert (send[D:].view(torch.int16) == -1).all().item(), "row past D written"


@pytest.mark.parametrize("H,tma", [(8, False), (256, False), (520, False), (2048, False),
                                   (7168, False), (16400, False), (8, True), (256, True),
                                   (2048, True), (7168, True), (16384, True)])
def test_gather_row_sizes(coact, H, tma):
    # the vector path (short, odd-length and very long rows) and the TMA bulk path
    r = workload.make_routing(2, N=3001)
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    x, send, err = _gather(coact, r, H, plan, tma=tma)
    assert err.item() == 0
    want = oracle.gather(host_bits(x), o["row_token"], o["D"])
    got = host_bits(send)
    assert np.array_equal(got[:o["D"]], want)
    assert (got[o["D"]:] == 0xFFFF).all()


@pytest.mark.parametrize("tma", [False, True])
def test_gather_row_range_flag(coact, tma):
    N, H, k = 100, 64, 2
    x = workload.fill_bf16(N, H, 0, 1, device=DEV)
    send_row = torch.full((N, k), -1, dtype=torch.int32, device=DEV)
    send_row[:, 0] = torch.arange(N, dtype=torch.int32, device=DEV)
    send_row[3, 1] = 100                                     # == capacity: out of range
    send = torch.zeros((N, H), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.dispatch_gather(x, send_row, send, err_flag=err, tma=tma)
    assert err.item() == coact.EFLAG_ROW_RANGE
    assert torch.equal(send, x)


# ----------------------------------------------------------------------------- combine


@pytest.mark.parametrize("cfg", [0, 1])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_combine_full(coact, cfg, out_dtype):
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    out = torch.empty((r.N, H), dtype=out_dtype, device=DEV)
    err = zero_flag()
    coact.combine_scatter(y, cuda(r.gates), plan.comb_row, out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    yh = host_bits(workload.fill_bf16(nk, H, r.seed, Y_STREAM))
    check_combine(out, yh, r.gates, o["comb_row"])


@pytest.mark.parametrize("cfg", [2, 3])
def test_combine_full_size_complete(coact, cfg):
    """Configs 2 and 3 at full size: every combined row against the oracle (fixed-order
    fp32 chain bit for bit, float64 reference within tolerance), in chunks of tokens."""
    r = workload.make_routing(cfg)
    H, nk = r.cfg.H, r.N * r.k
    plan, _ = run_plan(coact, r)
    o = oracle_plan_for(r)
    y = workload.fill_bf16(nk, H, r.seed, Y_STREAM, device=DEV)
    out = torch.empty((r.N, H), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.combine_scatter(y, cuda(r.gates), plan.comb_row, out, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    check_combine_complete(out, y, r.gates, o["comb_row"])
    del y, out


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("H", [8, 1000])
def test_combine_k_and_h(coact, k, H):
    rng = np.random.default_rng(k * 100 + H)
    N = 777
    gates = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    y = workload.fill_bf16(N * k, H, k, 3, device=DEV)
    for dt in (torch.bfloat16, torch.float32):
        out = torch.empty((N, H), dtype=dt, device=DEV)
        coact.combine_scatter(y, cuda(gates), cuda(comb), out)
        check_combine(out, host_bits(y), gates, comb)


def test_combine_invalid_rows(coact):
    N, k, H = 64, 3, 16
    rng = np.random.default_rng(1)
    gates = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    comb[4, 1] = -1                       # an invalid token's slot: skipped silently
    comb[9, 2] = N * k + 5                # out of range: skipped and flagged
    y = workload.fill_bf16(N * k, H, 0, 4, device=DEV)
    out = torch.empty((N, H), dtype=torch.float32, device=DEV)
    err = zero_flag()
    coact.combine_scatter(y, cuda(gates), cuda(comb), out, err_flag=err)
    assert err.item() == coact.EFLAG_ROW_RANGE
    check_combine(out, host_bits(y), gates, comb)


# ----------------------------------------------------------------------------- the whole path


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_identity_experts_end_to_end(coact, cfg):
    """plan -> gather -> identity experts -> combine reproduces the naive (one row per
    token-expert pair) combine bit for bit: deduplication leaves the result unchanged."""
    r = workload.make_routing(cfg, N=min(workload.CONFIGS[cfg].N, 16384))
    H = min(r.cfg.H, 1024)
    plan, _ = run_plan(coact, r)
    x, send, _ = _gather(coact, r, H, plan, sentinel_rows=False)
    D = int(plan.rank_offsets[-1].item())
    reps = torch.bitwise_count(plan.row_kmask[:D].to(torch.int32)) if hasattr(torch, "bitwise_count") \
        else torch.tensor([bin(int(v)).count("1") for v in plan.row_kmask[:D].cpu()], device=DEV)
    y = send[:D].repeat_interleave(reps.to(torch.int64), dim=0)     # identity experts
    assert y.shape[0] == r.N * r.k
    out = torch.empty((r.N, H), dtype=torch.float32, device=DEV)
    coact.combine_scatter(y, cuda(r.gates), plan.comb_row, out)
    want = oracle.naive_combine_identity_f32(host_bits(x), r.gates)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("cfg,seed", [(1, 1), (1, 7), (2, 3), (3, 5)])
def test_whole_path_other_seeds(coact, cfg, seed):
    """The whole path on other seeded batches of the configurations (full N, rows of at
    most 2048 elements): counts and plan bit-exact, every gathered row bit-exact, every
    combined row equal to the oracle's fixed-order chain."""
    r = workload.make_routing(cfg, seed=seed)
    c = r.cfg
    H = min(c.H, 2048)
    pair = torch.zeros((c.E, c.E), dtype=torch.int64, device=DEV)
    loads = torch.zeros(c.E, dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(r.ids), c.E, pair, loads)
    op, ol, _ = oracle.count(r.ids, c.E)
    assert np.array_equal(pair.cpu().numpy(), op) and np.array_equal(loads.cpu().numpy(), ol)
    plan, err = run_plan(coact, r)
    o = oracle_plan_for(r)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(plan), o)
    x = workload.fill_bf16(r.N, H, seed, X_STREAM, device=DEV)
    send = torch.empty((plan.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather(x, plan.send_row, send)
    y = workload.fill_bf16(r.N * r.k, H, seed, Y_STREAM, device=DEV)
    out = torch.empty((r.N, H), dtype=torch.bfloat16, device=DEV)
    coact.combine_scatter(y, cuda(r.gates), plan.comb_row, out)
    torch.cuda.synchronize()
    check_gather_complete(send, host_bits(x), o["row_token"], o["D"])
    check_combine_complete(out, y, r.gates, o["comb_row"])


def test_token_shuffle_two_layers(coact):
    """Config 4: cross-layer counts on a calibration batch -> predicted home rank ->
    layer-2 plan with the tokens pre-sharded to it; every step against the oracle."""
    tl = workload.make_two_layer(4)
    cfg = tl.layer1.cfg
    E, R = cfg.E, cfg.R
    C = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(tl.calib1), E, C, ids2=cuda(tl.calib2), E2=E)
    oc, _, _ = oracle.count_cross(tl.calib1, E, tl.calib2, E)
    assert np.array_equal(C.cpu().numpy(), oc)
    er2 = tl.layer2.expert_rank
    home = torch.empty(tl.layer1.N, dtype=torch.int32, device=DEV)
    err = zero_flag()
    coact.predict_home(cuda(tl.layer1.ids), E, C, cuda(er2), R, home, err_flag=err)
    oh, f = oracle.predict_home(tl.layer1.ids, E, oc, er2, R)
    assert err.item() == 0 and f == 0
    assert np.array_equal(home.cpu().numpy(), oh)
    plan, err = run_plan(coact, tl.layer2, src_rank=oh)
    o = oracle_plan_for(tl.layer2, src_rank=oh)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(plan), o)
    base = oracle_plan_for(tl.layer2)
    nk = tl.layer2.N * tl.layer2.k
    shuffled, baseline = o["stats"][5] / nk, base["stats"][5] / nk
    assert abs(baseline - 1.0 / R) < 0.01       # contiguous shards: 1/R served locally
    assert shuffled > 2 * baseline              # prediction keeps far more assignments local


def test_correlated_placement_chain_config3(coact):
    """Config 3's co-activation-grouped placement: GPU pair counts -> the library's
    correlated placement -> GPU plan, against oracle counts -> oracle placement ->
    oracle plan; compared with round-robin placement."""
    r = workload.make_routing(3, placement_kind="roundrobin")
    E, R = r.cfg.E, r.cfg.R
    pair = torch.zeros((E, E), dtype=torch.int64, device=DEV)
    coact.coact_count(cuda(r.ids), E, pair)
    placed = coact.coact_place_correlated(pair, R).numpy()
    op, _, _ = oracle.count(r.ids, E)
    oplaced = oracle.place_correlated(op, R)
    assert np.array_equal(placed, oplaced)
    plan, err = run_plan(coact, r, expert_rank=placed)
    o = oracle_plan_for(r, expert_rank=oplaced)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(plan), o)
    rr = oracle_plan_for(r)
    assert o["D"] < rr["D"] and o["stats"][4] < rr["stats"][4]   # fewer rows, fewer remote nodes


# ----------------------------------------------------------------------------- two-hop dispatch


@pytest.mark.parametrize("cfg,N", [(2, None), (3, None), (2, 5000)])
def test_two_hop_dispatch(coact, cfg, N):
    """Hop 1 to nodes, hop 2 inside the node (Cobalt: fewer remote nodes): both plans and
    the forward map against the oracle, and the two-hop rows against the one-hop rows."""
    r = workload.make_routing(cfg, N=N)
    c = r.cfg
    src = None if N is None else np.random.default_rng(3).integers(0, c.R, r.N).astype(np.int32)
    th = coact.alloc_two_hop(r.N, r.k, c.E, c.R, c.n_nodes, DEV)
    err = zero_flag()
    coact.plan_two_hop(cuda(r.ids), c.E, cuda(r.expert_rank, np.int32), c.R,
                       cuda(r.rank_node, np.int32), c.n_nodes, th,
                       src_rank=None if src is None else cuda(src), err_flag=err)
    torch.cuda.synchronize()
    node_o, rank_o, fwd_o = oracle.plan_two_hop(r.ids, c.E, r.expert_rank, c.R, r.rank_node,
                                                c.n_nodes, src_rank=src)
    assert err.item() == 0
    assert_plan_equal(plan_to_host(th.node), node_o, sentinel=False)
    assert_plan_equal(plan_to_host(th.rank), rank_o, sentinel=False)
    assert np.array_equal(th.fwd_src.cpu().numpy(), fwd_o)
    assert node_o["stats"][2] == rank_o["stats"][4]
    # rows: x -> hop 1 (node segments) -> hop 2 (rank segments) == x -> rank segments
    H = c.H if N is None else 520
    x = workload.fill_bf16(r.N, H, r.seed, X_STREAM, device=DEV)
    hop1 = torch.empty((th.node.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    coact.dispatch_gather(x, th.node.send_row, hop1, err_flag=err)
    hop2 = torch.empty((th.rank.row_capacity, H), dtype=torch.bfloat16, device=DEV)
    hop2.view(torch.int16).fill_(-1)
    coact.forward_gather(hop1, th.fwd_src, hop2, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    D, cap = rank_o["D"], th.rank.row_capacity
    check_gather_complete(hop2, host_bits(x), rank_o["row_token"], D)
    if D < cap:
        assert (hop2[D:].view(torch.int16) == -1).all().item(), "row past D written"
    # the token-major forward writes the same rows, bit for bit, and nothing past D
    hop2t = torch.empty_like(hop2)
    hop2t.view(torch.int16).fill_(-1)
    coact.forward_gather_tokens(hop1, th.rank.send_row, th.fwd_src, hop2t, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(hop2t.view(torch.int16), hop2.view(torch.int16))


def test_forward_gather_tokens_flags(coact):
    N, k, H = 40, 3, 64
    src = workload.fill_bf16(10, H, 0, 5, device=DEV)
    send_row = np.full((N, k), -1, np.int32)
    send_row[:, 0] = np.arange(N)
    send_row[:20, 1] = np.arange(N, N + 20)
    send_row[3, 2] = 2 * N + 5                 # beyond n_rows: skipped, flagged
    fwd = np.full(2 * N, -1, np.int32)
    fwd[:N] = np.arange(N) % 10
    fwd[N:N + 20] = (np.arange(20) * 3) % 10
    fwd[7] = 12                                # beyond the hop-1 rows: skipped, flagged
    dst = torch.full((2 * N, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    err = zero_flag()
    coact.forward_gather_tokens(src, cuda(send_row), cuda(fwd), dst, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == coact.EFLAG_ROW_RANGE
    sb, db = host_bits(src), host_bits(dst)
    for d in range(2 * N):
        s_ = fwd[d]
        reached = d < N or (N <= d < N + 20)
        if reached and 0 <= s_ < 10:
            assert np.array_equal(db[d], sb[s_]), d
        else:
            assert (db[d] == 0xFFFF).all(), d


def test_forward_gather_flags_and_compose_map(coact):
    src = workload.fill_bf16(10, 16, 0, 5, device=DEV)
    fwd = torch.tensor([3, -1, 9, 10, 0], dtype=torch.int32, device=DEV)   # 10 is out of range
    dst = torch.zeros((5, 16), dtype=torch.bfloat16, device=DEV)
    err = zero_flag()
    coact.forward_gather(src, fwd, dst, err_flag=err)
    assert err.item() == coact.EFLAG_ROW_RANGE
    assert torch.equal(dst[0], src[3]) and torch.equal(dst[2], src[9]) and torch.equal(dst[4], src[0])
    assert (dst[1] == 0).all() and (dst[3] == 0).all()
    a = torch.tensor([2, 0, 5, 1], dtype=torch.int32, device=DEV)
    b = torch.tensor([10, 11, 12], dtype=torch.int32, device=DEV)
    err.zero_()
    out = coact.coact_compose_map(a, b, err_flag=err)
    assert out.cpu().tolist() == [12, 10, -1, 11] and err.item() == coact.EFLAG_ID_RANGE


# ----------------------------------------------------------------------------- across GPUs (emulated)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_peer_dispatch_combine_emulated(coact, cfg):
    """Expert parallelism with the exchange fused into the data movement, on one GPU: each
    of S = R source ranks plans its own contiguous block of tokens and writes its rows
    straight into R per-rank buffers (dispatch_gather_peer), then combines reading the
    expert outputs from the R per-rank buffers (combine_scatter_peer).  The sources run
    one after another -- nothing waits on anything.  Every destination buffer must equal
    the rank-r segment of the single-GPU plan of all tokens, and every source's combined
    rows the single-GPU combine of its tokens, bit for bit."""
    import co_activation_b200.ep as ep
    r = workload.make_routing(cfg)
    c = r.cfg
    N, k, E, R, H = r.N, r.k, c.E, c.R, min(c.H, 1024)
    S = R
    blocks = [(s * N // S, (s + 1) * N // S) for s in range(S)]
    x = workload.fill_bf16(N, H, r.seed, X_STREAM, device=DEV)
    er = cuda(r.expert_rank, np.int32)
    plans = []
    for s, (lo, hi) in enumerate(blocks):
        p = coact.alloc_plan(hi - lo, k, E, R, DEV)
        coact.plan_dispatch(cuda(r.ids[lo:hi]), E, er, R, p,
                            src_rank=torch.full((hi - lo,), s, dtype=torch.int32, device=DEV))
        plans.append(p)
    C = torch.stack([p.rank_counts.to(torch.int64) for p in plans]).cpu()
    A = torch.stack([(p.asg_offsets[1:] - p.asg_offsets[:-1]).to(torch.int64) for p in plans]).cpu()
    recv = [torch.full((int(C[:, q].sum()), H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
            for q in range(R)]
    bases = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device=DEV)
    caps = torch.tensor([t.shape[0] for t in recv], dtype=torch.int32, device=DEV)
    offC, offA = ep.exclusive_offsets(C), ep.exclusive_offsets(A)
    err = zero_flag()
    for s, (lo, hi) in enumerate(blocks):
        coact.dispatch_gather_peer(x[lo:hi], plans[s].send_row, plans[s].rank_offsets, bases,
                                   offC[s].to(torch.int32).to(DEV), caps, err_flag=err)
    torch.cuda.synchronize()
    src = np.concatenate([np.full(hi - lo, s, np.int32) for s, (lo, hi) in enumerate(blocks)])
    full = oracle.plan(r.ids, E, r.expert_rank, R, src_rank=src)
    xb = host_bits(x)
    for q in range(R):
        seg = full["row_token"][full["rank_offsets"][q]:full["rank_offsets"][q + 1]]
        assert np.array_equal(host_bits(recv[q]), xb[seg]), f"rank {q}"
    # expert outputs in the single-GPU expanded order, split into per-rank buffers
    y = workload.fill_bf16(N * k, H, r.seed, Y_STREAM, device=DEV)
    ybuf = [y[full["asg_offsets"][q]:full["asg_offsets"][q + 1]].clone() for q in range(R)]
    ybases = torch.tensor([t.data_ptr() for t in ybuf], dtype=torch.int64, device=DEV)
    ycaps = torch.tensor([t.shape[0] for t in ybuf], dtype=torch.int32, device=DEV)
    want = oracle.combine_f32chain(host_bits(y), r.gates, full["comb_row"])
    for s, (lo, hi) in enumerate(blocks):
        out = torch.empty((hi - lo, H), dtype=torch.float32, device=DEV)
        coact.combine_scatter_peer(ybases, offA[s].to(torch.int32).to(DEV), ycaps,
                                   plans[s].asg_offsets, cuda(r.gates[lo:hi]), plans[s].comb_row,
                                   out, H, err_flag=err)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy().view(np.uint32), want[lo:hi].view(np.uint32)), s
    assert err.item() == 0


@pytest.mark.parametrize("cfg", [1, 2])
def test_peer_sum_back_emulated(coact, cfg):
    """The way back of the pre-reduced combine and of the dispatch's gradient over peers,
    on one GPU: rows held per received row in R per-rank buffers (the rank-r segments of the
    single-GPU send layout) are read in place by combine_scatter_peer with unit weights over
    each source's send_row / rank_offsets.  Every source's result must equal the
    transposed dispatch of the single-GPU layout for its tokens, bit for bit; and with the
    partial rows of combine_rows as the held rows, the pre-reduced combine."""
    import co_activation_b200.ep as ep
    r = workload.make_routing(cfg)
    c = r.cfg
    N, k, E, R, H = r.N, r.k, c.E, c.R, min(c.H, 1024)
    S = R
    blocks = [(s * N // S, (s + 1) * N // S) for s in range(S)]
    er = cuda(r.expert_rank, np.int32)
    plans = []
    for s, (lo, hi) in enumerate(blocks):
        p = coact.alloc_plan(hi - lo, k, E, R, DEV)
        coact.plan_dispatch(cuda(r.ids[lo:hi]), E, er, R, p,
                            src_rank=torch.full((hi - lo,), s, dtype=torch.int32, device=DEV))
        plans.append(p)
    C = torch.stack([p.rank_counts.to(torch.int64) for p in plans]).cpu()
    offC = ep.exclusive_offsets(C)
    src = np.concatenate([np.full(hi - lo, s, np.int32) for s, (lo, hi) in enumerate(blocks)])
    full = oracle.plan(r.ids, E, r.expert_rank, R, src_rank=src)
    ro = full["rank_offsets"]
    # held rows: single-GPU send-layout rows, split into per-rank buffers
    G = workload.fill_bf16(int(ro[-1]), H, r.seed, 7, device=DEV)
    y = workload.fill_bf16(N * k, H, r.seed, Y_STREAM, device=DEV)
    fp = coact.alloc_plan(N, k, E, R, DEV)
    coact.plan_dispatch(cuda(r.ids), E, er, R, fp, src_rank=cuda(src))
    pre = torch.empty((int(ro[-1]), H), dtype=torch.bfloat16, device=DEV)
    coact.combine_rows(y, cuda(r.gates), fp.comb_row, fp.row_token, fp.row_kmask, pre)
    torch.cuda.synchronize()
    want_g = oracle.gather_backward_f32chain(host_bits(G), full["send_row"])
    _, want_pre = oracle.combine_prereduced(host_bits(y), r.gates, full)
    err = zero_flag()
    for held, want in ((G, want_g), (pre, want_pre)):
        bufs = [held[ro[q]:ro[q + 1]].clone() for q in range(R)]
        bases = torch.tensor([t.data_ptr() for t in bufs], dtype=torch.int64, device=DEV)
        caps = torch.tensor([t.shape[0] for t in bufs], dtype=torch.int32, device=DEV)
        for s, (lo, hi) in enumerate(blocks):
            out = torch.empty((hi - lo, H), dtype=torch.float32, device=DEV)
            coact.combine_scatter_peer(bases, offC[s].to(torch.int32).to(DEV), caps,
                                       plans[s].rank_offsets, None, plans[s].send_row, out, H,
                                       err_flag=err)
            torch.cuda.synchronize()
            assert np.array_equal(out.cpu().numpy().view(np.uint32), want[lo:hi].view(np.uint32)), s
    assert err.item() == 0


def test_peer_row_range_flag(coact):
    r = workload.make_routing(0)
    c = r.cfg
    p = coact.alloc_plan(r.N, r.k, c.E, c.R, DEV)
    coact.plan_dispatch(cuda(r.ids), c.E, cuda(r.expert_rank, np.int32), c.R, p)
    x = workload.fill_bf16(r.N, 64, 0, 1, device=DEV)
    counts = p.rank_counts.cpu()
    bufs = [torch.zeros((max(int(n) - 5, 1), 64), dtype=torch.bfloat16, device=DEV) for n in counts]
    bases = torch.tensor([t.data_ptr() for t in bufs], dtype=torch.int64, device=DEV)
    caps = torch.tensor([t.shape[0] for t in bufs], dtype=torch.int32, device=DEV)
    err = zero_flag()
    coact.dispatch_gather_peer(x, p.send_row, p.rank_offsets, bases,
                               torch.zeros(c.R, dtype=torch.int32, device=DEV), caps, err_flag=err)
    assert err.item() == coact.EFLAG_ROW_RANGE        # the last 5 rows of every rank do not fit
