"""Pins for the CPU oracle: each test checks the oracle against something other than
itself -- a hand-worked case, a closed form, an invariant the pages fix, a library
routine that computes the same quantity another way, or brute force on tiny inputs.

Sources: Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English
abstracts (pair co-activation, once-per-GPU dispatch, node-level routing, combine,
routing decisions left unchanged).
"""
from fractions import Fraction
import itertools
import math
import struct

import numpy as np
import pytest

import oracle
import workload


# ----------------------------------------------------------------------------- helpers


def rand_ids(rng, N, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(N)]).astype(np.int32)


def indicator(ids, E):
    A = np.zeros((ids.shape[0], E), np.int64)
    for j in range(ids.shape[1]):
        A[np.arange(ids.shape[0]), ids[:, j]] = 1
    return A


def brute_plan(ids, er, R, rank_node, src):
    """Positions by sorting: every (r, t) with r among t's ranks, in (r, t) order, is
    one send row; every (r, t, j) with slot j on r, in (r, t, j) order, is one
    assignment row."""
    N, k = ids.shape
    rows = sorted({(int(er[ids[t, j]]), t) for t in range(N) for j in range(k)})
    asg = sorted((int(er[ids[t, j]]), t, j) for t in range(N) for j in range(k))
    row_of = {rt: i for i, rt in enumerate(rows)}
    comb = np.full((N, k), -1, np.int32)
    for i, (r, t, j) in enumerate(asg):
        comb[t, j] = i
    send = np.full((N, k), -1, np.int32)
    for t in range(N):
        seen = set()
        for j in range(k):
            r = int(er[ids[t, j]])
            if r not in seen:
                send[t, j] = row_of[(r, t)]
                seen.add(r)
    row_token = np.array([t for (_, t) in rows], np.int32)
    row_kmask = np.array([sum(1 << j for j in range(k) if er[ids[t, j]] == r) for (r, t) in rows],
                         np.uint8)
    counts = np.bincount([r for (r, _) in rows], minlength=R)
    acounts = np.bincount([r for (r, _, _) in asg], minlength=R)
    node = lambda r: int(rank_node[r])
    st = np.zeros(8, np.int64)
    st[0] = N * k
    st[1] = len(rows)
    for t in range(N):
        ranks = {int(er[e]) for e in ids[t]}
        nodes = {node(r) for r in ranks}
        s, ns = int(src[t]), node(int(src[t]))
        st[2] += len(ranks - {s})
        st[3] += sum(1 for r in ranks if node(r) != ns)
        st[4] += len(nodes - {ns})
        st[5] += sum(1 for e in ids[t] if er[e] == s)
        st[7] += sum(1 for e in ids[t] if node(int(er[e])) != ns)
    st[6] = N * k - st[5]
    src_dst = np.zeros((R, R), np.int32)
    for (r, t) in rows:
        src_dst[src[t], r] += 1
    return dict(rank_counts=counts, rank_offsets=np.concatenate([[0], np.cumsum(counts)]),
                asg_offsets=np.concatenate([[0], np.cumsum(acounts)]), row_token=row_token,
                row_kmask=row_kmask, send_row=send, comb_row=comb, stats=st, src_dst=src_dst)


def f32_round_exact(q: Fraction) -> float:
    """Round an exact rational to the nearest float32, ties to even (normal range)."""
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    scaled = a / Fraction(2) ** (e - 23)          # in [2^23, 2^24)
    m = scaled.numerator // scaled.denominator
    rem = scaled - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    return sign * float(m) * 2.0 ** (e - 23)


def bf16(v):
    return workload.bf16_bits_to_float(np.asarray(v, np.uint16))


# ----------------------------------------------------------------------------- hand-worked cases

# Four tokens, four experts, top-2, two ranks (experts 0,1 -> rank 0; 2,3 -> rank 1),
# rank r on node r, contiguous source shards src = [0, 0, 1, 1].  Worked by hand:
#   rank sets  t0 {0}, t1 {0,1}, t2 {0,1}, t3 {1};  D = 6 < N*k = 8
#   rank 0 rows: t0 (slots 0,1 -> kmask 3), t1 (slot 0 -> 1), t2 (slot 1 -> 2)
#   rank 1 rows: t1 (slot 1 -> 2), t2 (slot 0 -> 1), t3 (slots 0,1 -> 3)
#   assignment rows: rank 0 = (t0,0) (t0,1) (t1,0) (t2,1); rank 1 = (t1,1) (t2,0) (t3,0) (t3,1)
HAND_IDS = np.array([[0, 1], [1, 2], [3, 0], [2, 3]], np.int32)
HAND_ER = np.array([0, 0, 1, 1], np.int32)


def test_hand_worked_plan():
    p = oracle.plan(HAND_IDS, 4, HAND_ER, 2, rank_node=[0, 1], n_nodes=2)
    assert p["flags"] == 0
    assert p["rank_counts"].tolist() == [3, 3]
    assert p["rank_offsets"].tolist() == [0, 3, 6]
    assert p["asg_offsets"].tolist() == [0, 4, 8]
    assert p["row_token"][:6].tolist() == [0, 1, 2, 1, 2, 3]
    assert p["row_kmask"][:6].tolist() == [3, 1, 2, 2, 1, 3]
    assert p["send_row"].tolist() == [[0, -1], [1, 3], [4, 2], [5, -1]]
    assert p["comb_row"].tolist() == [[0, 1], [2, 4], [5, 3], [6, 7]]
    # naive 8, dedup 6, remote rows 2 (t1->r1, t2->r0), cross-node rows 2, node-dedup 2,
    # local-served assignments 6, remote assignments 2, cross-node assignments 2
    assert p["stats"].tolist() == [8, 6, 2, 2, 2, 6, 2, 2]
    assert p["src_dst"].tolist() == [[2, 1], [1, 2]]
    assert p["rank_mask"].tolist() == [1, 3, 3, 2]


def test_hand_worked_count():
    pair, loads, f = oracle.count(HAND_IDS, 4)
    assert f == 0
    want = np.zeros((4, 4), np.int64)
    for a, b in [(0, 1), (1, 2), (0, 3), (2, 3)]:
        want[a, b] = want[b, a] = 1
    assert (pair == want).all()
    assert loads.tolist() == [2, 2, 2, 2]


def test_hand_worked_node_dedup():
    # one token on experts {0, 2, 3}, each expert alone on its rank, ranks {0,1} on
    # node 0 and {2,3} on node 1, home rank 0: two remote rows (ranks 2 and 3), both
    # cross-node, but one remote *node* -- the "fewer remote nodes" count (Cobalt).
    p = oracle.plan(np.array([[0, 2, 3]], np.int32), 4, np.arange(4), 4,
                    rank_node=[0, 0, 1, 1], n_nodes=2, src_rank=[0])
    assert p["stats"].tolist() == [3, 3, 2, 2, 1, 1, 2, 2]


# ----------------------------------------------------------------------------- counting pins


@pytest.mark.parametrize("seed", range(20))
def test_count_brute_force(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(2, 17))
    k = int(rng.integers(1, min(4, E) + 1))
    N = int(rng.integers(0, 65))
    ids = rand_ids(rng, N, E, k) if N else np.zeros((0, k), np.int32)
    pair, loads, f = oracle.count(ids, E)
    assert f == 0
    for a, b in itertools.product(range(E), range(E)):
        want = 0 if a == b else sum(1 for t in range(N) if a in ids[t] and b in ids[t])
        assert pair[a, b] == want
    assert (loads == np.bincount(ids.ravel(), minlength=E)).all()


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_count_invariants_and_matmul(cfg):
    r = workload.make_routing(cfg)
    N, k, E = r.N, r.k, r.cfg.E
    pair, loads, f = oracle.count(r.ids, E)
    assert f == 0
    assert (pair == pair.T).all() and (np.diag(pair) == 0).all()
    assert np.triu(pair, 1).sum() == N * k * (k - 1) // 2
    assert loads.sum() == N * k
    # co-occurrence by a library matmul: A^T A minus its diagonal
    A = indicator(r.ids, E).astype(np.float64)
    co = (A.T @ A).round().astype(np.int64)
    assert (np.diag(co) == loads).all()
    np.fill_diagonal(co, 0)
    assert (co == pair).all()


def test_count_closed_form_and_accumulate():
    N, E = 100, 10
    ids = np.tile(np.array([[7, 2, 4]], np.int32), (N, 1))
    pair, loads, _ = oracle.count(ids, E)
    want = np.zeros((E, E), np.int64)
    for a, b in itertools.permutations([7, 2, 4], 2):
        want[a, b] = N
    assert (pair == want).all()
    oracle.count(ids, E, pair, loads)                     # accumulates
    assert (pair == 2 * want).all() and loads[7] == 2 * N


def test_count_errors_skip_token():
    ids = np.array([[0, 1], [1, 9], [2, 2], [3, 0]], np.int32)
    pair, loads, f = oracle.count(ids, 4)
    assert f == oracle.FLAG_ID_RANGE | oracle.FLAG_DUP_ID
    assert pair.sum() == 4 and loads.sum() == 4           # only tokens 0 and 3 counted


@pytest.mark.parametrize("seed", range(5))
def test_count_cross_matmul(seed):
    rng = np.random.default_rng(100 + seed)
    N, E1, E2, k1, k2 = 500, 12, 9, 3, 2
    ids1, ids2 = rand_ids(rng, N, E1, k1), rand_ids(rng, N, E2, k2)
    C, l1, f = oracle.count_cross(ids1, E1, ids2, E2)
    assert f == 0
    want = indicator(ids1, E1).T @ indicator(ids2, E2)
    assert (C == want).all() and C.sum() == N * k1 * k2
    assert (l1 == np.bincount(ids1.ravel(), minlength=E1)).all()


# ----------------------------------------------------------------------------- plan pins


@pytest.mark.parametrize("seed", range(30))
def test_plan_brute_force(seed):
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.choice([1, 2, 3, 4, 8]))
    epr = int(rng.integers(1, 4))
    E = R * epr
    k = int(rng.integers(1, min(4, E) + 1))
    N = int(rng.integers(1, 65))
    ids = rand_ids(rng, N, E, k)
    er = rng.permutation(np.arange(E) // epr).astype(np.int32)
    n_nodes = int(rng.choice([n for n in (1, 2, 4) if R % n == 0]))
    rank_node = (np.arange(R) // (R // n_nodes)).astype(np.int32)
    src = rng.integers(0, R, N).astype(np.int32) if seed % 2 else workload.contiguous_src_rank(N, R)
    p = oracle.plan(ids, E, er, R, rank_node=rank_node, n_nodes=n_nodes,
                    src_rank=None if seed % 2 == 0 else src)
    b = brute_plan(ids, er, R, rank_node, src)
    assert p["flags"] == 0
    D = p["D"]
    for key in ("rank_counts", "rank_offsets", "asg_offsets", "send_row", "comb_row", "stats",
                "src_dst"):
        assert np.array_equal(np.asarray(p[key]), np.asarray(b[key])), key
    assert np.array_equal(p["row_token"][:D], b["row_token"])
    assert np.array_equal(p["row_kmask"][:D], b["row_kmask"])


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_plan_invariants(cfg):
    r = workload.make_routing(cfg)
    N, k, E, R, epr = r.N, r.k, r.cfg.E, r.cfg.R, r.cfg.epr
    p = oracle.plan(r.ids, E, r.expert_rank, R, r.rank_node, r.cfg.n_nodes)
    D = p["D"]
    assert p["flags"] == 0
    # each token goes to each rank once: N*ceil(k/epr) <= D <= N*min(k,R)
    assert N * math.ceil(k / epr) <= D <= N * min(k, R)
    assert p["stats"][1] == D and p["stats"][0] == N * k
    # bijections: every (t, r) pair is one row, every (t, j) one assignment row
    rm = p["rank_mask"]
    assert sum(bin(int(m)).count("1") for m in rm) == D
    pairs = {(int(p["row_token"][d]), r_) for r_ in range(R)
             for d in range(p["rank_offsets"][r_], p["rank_offsets"][r_ + 1])}
    assert len(pairs) == D
    assert sorted(p["comb_row"].ravel().tolist()) == list(range(N * k))
    # the first slot of each rank carries a send row; the send rows are a bijection of [0, D)
    sr = p["send_row"].ravel()
    assert sorted(sr[sr >= 0].tolist()) == list(range(D))
    # rows ascend by token inside each rank segment
    for r_ in range(R):
        seg = p["row_token"][p["rank_offsets"][r_]:p["rank_offsets"][r_ + 1]]
        assert (np.diff(seg) > 0).all()
    st = p["stats"]
    assert st[5] + st[6] == N * k
    assert st[4] <= st[3] <= st[2] <= D
    assert p["src_dst"].sum() == D and (p["src_dst"].sum(0) == p["rank_counts"]).all()
    if r.cfg.n_nodes == 1:
        assert st[3] == st[4] == st[7] == 0


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_plan_identity_placement_and_single_rank(cfg):
    r = workload.make_routing(cfg)
    N, k, E = r.N, r.k, r.cfg.E
    # every expert alone on its rank (E == R): nothing to deduplicate, D == N*k
    p = oracle.plan(r.ids, E, np.arange(E), E)
    assert p["D"] == N * k
    # a single rank: every token is local; no remote, no cross-node rows, D == N
    p1 = oracle.plan(r.ids, E, np.zeros(E, np.int32), 1)
    assert p1["D"] == N
    assert p1["stats"][2] == p1["stats"][3] == p1["stats"][6] == 0
    assert p1["stats"][5] == N * k


def test_plan_top2_removes_at_most_half(pages_figures):
    # at top-k the dedup dispatcher removes at most (k-1)/k of the rows, so the pages'
    # "up to 58%" needs top-k with k >= 3; at top-2 at most 50% can go
    for cfg in (0, 1):
        r = workload.make_routing(cfg)
        p = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)
        removed = 1 - p["D"] / (r.N * r.k)
        assert 0 <= removed <= 0.5
    assert pages_figures["max_rows_removed"]["fraction"] > 0.5


def test_plan_baseline_local_share(pages_figures):
    # uniform routing, one node of 8 ranks, contiguous shards: a token's experts do not
    # depend on its home rank, so 1/8 = 12.5% of assignments are served locally
    fig = pages_figures["local_served_baseline_one_node"]
    cfg = workload.CONFIGS[1].with_(n_groups=0, plant_prob=0.0, placement="contiguous")
    assert cfg.R == fig["gpus"]
    r = workload.make_routing(cfg)
    p = oracle.plan(r.ids, cfg.E, r.expert_rank, cfg.R)
    share = p["stats"][5] / (r.N * r.k)
    assert abs(share - fig["share"]) < 0.01


def test_plan_capacity_and_errors():
    r = workload.make_routing(0)
    full = oracle.plan(r.ids, 8, r.expert_rank, 4)
    cap = full["D"] - 100
    p = oracle.plan(r.ids, 8, r.expert_rank, 4, row_capacity=cap)
    assert p["flags"] & oracle.FLAG_CAPACITY
    assert np.array_equal(p["row_token"][:cap], full["row_token"][:cap])
    assert (p["send_row"] < cap).all()
    bad = r.ids.copy()
    bad[3, 1] = 8
    bad[5, 1] = bad[5, 0]
    q = oracle.plan(bad, 8, r.expert_rank, 4, src_rank=np.r_[[9], np.zeros(r.N - 1, np.int32)])
    assert q["flags"] == oracle.FLAG_ID_RANGE | oracle.FLAG_DUP_ID | oracle.FLAG_SRC_RANK
    assert (q["send_row"][[0, 3, 5]] == -1).all() and q["D"] < full["D"]


# ----------------------------------------------------------------------------- rows and combine


def test_gather_is_fancy_index():
    r = workload.make_routing(0)
    p = oracle.plan(r.ids, 8, r.expert_rank, 4)
    x = workload.fill_bf16(r.N, 256, 0, 1)
    xb = oracle._bits(x)
    send = oracle.gather(xb, p["row_token"], p["D"])
    assert np.array_equal(send, xb[p["row_token"][:p["D"]]])


@pytest.mark.parametrize("cfg", [0, 1])
def test_combine_identity_closed_form_and_naive(cfg):
    r = workload.make_routing(cfg)
    H = 64
    x = oracle._bits(workload.fill_bf16(r.N, H, 0, 3))
    p = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)
    y = oracle.expand_identity(x, p["row_token"], p["row_kmask"], p["D"])
    assert y.shape[0] == r.N * r.k
    # layout: the expert output for (t, j) sits at comb_row[t, j] and is x[t]
    assert np.array_equal(y[p["comb_row"]], np.repeat(x[:, None, :], r.k, axis=1))
    # identity experts: combine = x[t] * sum_j gate[t,j]
    out = oracle.combine_f64(y, r.gates, p["comb_row"])
    want = bf16(x).astype(np.float64) * r.gates.astype(np.float64).sum(1, keepdims=True)
    assert np.allclose(out, want, rtol=1e-12, atol=1e-12)
    # routing unchanged by deduplication: dedup combine == naive combine, bit for bit
    c32 = oracle.combine_f32chain(y, r.gates, p["comb_row"])
    n32 = oracle.naive_combine_identity_f32(x, r.gates)
    assert np.array_equal(c32.view(np.uint32), n32.view(np.uint32))


def test_combine_f64_matches_numpy_and_chain_bound():
    rng = np.random.default_rng(7)
    N, k, H, rows = 300, 5, 40, 300 * 5
    y = oracle._bits(workload.fill_bf16(rows, H, 1, 9))
    g = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(rows).reshape(N, k).astype(np.int32)
    out = oracle.combine_f64(y, g, comb)
    yf = bf16(y).astype(np.float64)
    want = sum(g[:, j, None].astype(np.float64) * yf[comb[:, j]] for j in range(k))
    assert np.allclose(out, want, rtol=1e-13, atol=1e-13)
    c32 = oracle.combine_f32chain(y, g, comb).astype(np.float64)
    mag = sum(np.abs(g[:, j, None].astype(np.float64) * yf[comb[:, j]]) for j in range(k))
    # k fused multiply-adds, each one rounding of at most 2^-24 relative
    assert (np.abs(c32 - out) <= k * 2.0 ** -24 * mag + 1e-30).all()


@pytest.mark.parametrize("seed", range(4))
def test_combine_chain_exact_rational(seed):
    # the fp32 chain against exact rational arithmetic, rounded once per step
    rng = np.random.default_rng(50 + seed)
    N, k, H = 6, 4, 8
    y = oracle._bits(workload.fill_bf16(N * k, H, seed, 11))
    g = rng.random((N, k)).astype(np.float32)
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    c32 = oracle.combine_f32chain(y, g, comb)
    yf = bf16(y)
    for t in range(N):
        for h in range(H):
            acc = 0.0
            for j in range(k):
                exact = Fraction(float(g[t, j])) * Fraction(float(yf[comb[t, j], h])) + Fraction(acc)
                acc = f32_round_exact(exact)
            assert float(c32[t, h]) == acc


def test_combine_special_cases():
    y = oracle._bits(workload.fill_bf16(8, 16, 2, 2))
    # k = 1 with gate 1: the row itself
    out = oracle.combine_f32chain(y, np.ones((8, 1), np.float32), np.arange(8).reshape(8, 1))
    assert np.array_equal(out, bf16(y))
    # two equal rows with gates 1/2, 1/2: the row itself, exactly
    comb = np.stack([np.arange(8), np.arange(8)], 1).astype(np.int32)
    out = oracle.combine_f32chain(y, np.full((8, 2), 0.5, np.float32), comb)
    assert np.array_equal(out, bf16(y))


def test_bf16_rne_against_torch():
    import torch
    rng = np.random.default_rng(3)
    u = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]                      # finite values
    ties = (u & 0xFFFF0000) | 0x8000                       # exact halfway cases, odd and even
    vals = np.concatenate([u, ties]).view(np.float32)
    got = oracle.bf16_rne(vals)
    want = torch.from_numpy(vals.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    special = np.array([np.inf, -np.inf, 0.0, -0.0, 3.4028235e38, 1e-45], np.float32)
    assert oracle.bf16_rne(special).tolist() == [0x7F80, 0xFF80, 0x0000, 0x8000, 0x7F80, 0x0000]
    nan = oracle.bf16_rne(np.array([np.nan], np.float32))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0


def _nan_as_nan_equal(a: np.ndarray, b: np.ndarray) -> bool:
    """Bitwise equality of float32 arrays where a NaN meets a NaN of any payload."""
    na, nb = np.isnan(a), np.isnan(b)
    return bool(np.array_equal(na, nb) and np.array_equal(a.view(np.uint32)[~na],
                                                         b.view(np.uint32)[~nb]))


@pytest.mark.parametrize("k", [1, 2])
def test_combine_chain_special_values_ieee(k):
    """The fixed-order chain on every class of bf16 value (+-0, subnormals, +-inf, NaNs,
    the largest values) and special gates, against IEEE float32 arithmetic in numpy.
    The gates are bf16-representable with |g| in {0} u [2^-8, 1] or infinite, so every
    product g*y is exact in fp32 (at most 16 significant bits, no overflow, no loss in
    the subnormal range): then fma(g1, y1, +0) is the product plus +0 (which turns -0
    into +0) and fma(g2, y2, acc) is one rounded float32 addition.  NaN meets NaN."""
    rng = np.random.default_rng(40 + k)
    N, H = 3000, 64
    y = rng.integers(0, 1 << 16, (N * k, H), dtype=np.uint32).astype(np.uint16)
    y[:, :13] = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F81, 0x0001,
                          0x8001, 0x007F, 0x7F7F, 0xFF7F, 0x3F80], np.uint16)
    pool = np.array([0.0, -0.0, 1.0, -1.0, 0.5, 0.75, -0.375, 2.0 ** -8, 0.9921875,
                     np.inf, -np.inf, np.nan], np.float32)
    g = pool[rng.integers(0, len(pool), (N, k))]
    comb = rng.permutation(N * k).reshape(N, k).astype(np.int32)
    got = oracle.combine_f32chain(y, g, comb)
    yf = workload.bf16_bits_to_float(y)
    with np.errstate(invalid="ignore", over="ignore"):
        want = g[:, 0, None] * yf[comb[:, 0]] + np.float32(0.0)
        for j in range(1, k):
            want = want + g[:, j, None] * yf[comb[:, j]]
    assert want.dtype == np.float32
    assert _nan_as_nan_equal(got, want)
    assert np.isnan(got).any() and np.isinf(got).any() and (got == 0).any()
    # and its rounding to bf16 matches torch's conversion (NaN as NaN)
    import torch
    b = oracle.bf16_rne(got)
    t = torch.from_numpy(got.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert _nan_as_nan_equal(workload.bf16_bits_to_float(b), workload.bf16_bits_to_float(t))


# ----------------------------------------------------------------------------- prediction pins


@pytest.mark.parametrize("seed", range(5))
def test_predict_home_matmul(seed):
    rng = np.random.default_rng(200 + seed)
    N, E1, E2, R, k1 = 400, 16, 12, 4, 2
    ids1 = rand_ids(rng, N, E1, k1)
    C = rng.integers(0, 5, (E1, E2)).astype(np.int64)
    er2 = (rng.permutation(E2) % R).astype(np.int32)
    home, f = oracle.predict_home(ids1, E1, C, er2, R)
    assert f == 0
    onehot = np.zeros((E2, R), np.int64)
    onehot[np.arange(E2), er2] = 1
    S = C @ onehot                                         # [E1, R] counts per rank
    score = S[ids1[:, 0]] + S[ids1[:, 1]]
    assert np.array_equal(home, score.argmax(1))           # argmax: first (lowest) rank on ties


def test_predict_home_ties_lowest_rank():
    C = np.zeros((4, 4), np.int64)                         # all scores zero -> rank 0
    home, _ = oracle.predict_home(np.array([[0, 1], [2, 3]], np.int32), 4, C, [0, 1, 2, 3], 4)
    assert home.tolist() == [0, 0]
    C[0, 3] = C[1, 2] = 5                                  # ranks 2 and 3 tie at 5 -> 2
    home, _ = oracle.predict_home(np.array([[0, 1]], np.int32), 4, C, [0, 1, 2, 3], 4)
    assert home.tolist() == [2]
