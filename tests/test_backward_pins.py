"""Pins for the oracle's backward pass and pre-reduced reverse path.

Both forward maps are linear in the rows they move, so their gradients are the transposed
maps; each pin ties the new oracle functions to something outside them: a hand-worked
case, a dense matrix and its transpose, the adjoint identity <A x, g> = <x, A^T g> with the
(already pinned) forward oracle, one-hot probes through the forward combine, exact
rational arithmetic for the accumulation order, and torch's own rounding.

Sources: Cobalt (arxivdaily 2609.36959) and Zyphra (arxivdaily 2610.09372), English
abstracts (each token to each GPU once, dispatch then combine).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workload
from test_oracle_pins import HAND_ER, HAND_IDS, f32_round_exact, rand_ids


def bf16(bits):
    return workload.bf16_bits_to_float(np.asarray(bits, np.uint16))


def bf16_bits_torch(values) -> np.ndarray:
    """float values -> bf16 bits through torch's own round-to-nearest-even."""
    t = torch.as_tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def small_int_bits(rng, shape, lo=-8, hi=8) -> np.ndarray:
    return bf16_bits_torch(rng.integers(lo, hi + 1, shape).astype(np.float32))


def random_plan(seed, N=40, E=8, k=3, R=4):
    rng = np.random.default_rng(seed)
    ids = rand_ids(rng, N, E, k)
    er = rng.permutation(np.repeat(np.arange(R), E // R)).astype(np.int32)
    return rng, ids, er, oracle.plan(ids, E, er, R)


# ----------------------------------------------------------------------------- hand-worked

# The hand-worked plan of test_oracle_pins: send rows (row_token) [0, 1, 2, 1, 2, 3],
# send_row [[0,-1],[1,3],[4,2],[5,-1]], comb_row [[0,1],[2,4],[5,3],[6,7]].


def test_hand_worked_gather_backward():
    p = oracle.plan(HAND_IDS, 4, HAND_ER, 2, rank_node=[0, 1], n_nodes=2)
    g_send = bf16_bits_torch(np.arange(1, 7, dtype=np.float32)[:, None])   # rows 0..5 = 1..6
    gx = oracle.gather_backward_f32chain(g_send, p["send_row"])
    # t0: row 0; t1: rows 1 + 3; t2: rows 4 + 2; t3: row 5
    assert gx[:, 0].tolist() == [1.0, 2.0 + 4.0, 5.0 + 3.0, 6.0]


def test_hand_worked_prereduced_and_backward():
    p = oracle.plan(HAND_IDS, 4, HAND_ER, 2, rank_node=[0, 1], n_nodes=2)
    y = bf16_bits_torch(np.arange(1, 9, dtype=np.float32)[:, None])        # rows 0..7 = 1..8
    gates = np.array([[1, 2], [3, 4], [5, 6], [7, 8]], np.float32)
    pre, out = oracle.combine_prereduced(y, gates, p)
    # row 0 (t0, slots 0,1) = 1*1 + 2*2; row 1 (t1, slot 0) = 3*3; row 2 (t2, slot 1) = 6*4
    # row 3 (t1, slot 1) = 4*5; row 4 (t2, slot 0) = 5*6; row 5 (t3, slots 0,1) = 7*7 + 8*8
    assert bf16(pre)[:, 0].tolist() == [5.0, 9.0, 24.0, 20.0, 30.0, 113.0]
    assert out[:, 0].tolist() == [5.0, 29.0, 54.0, 113.0]
    g_out = bf16_bits_torch(np.array([[1], [2], [3], [4]], np.float32))
    gy, gg, _ = oracle.combine_backward(y, gates, p["comb_row"], g_out)
    # g_y[comb_row[t,j]] = gates[t,j] * g_out[t]
    assert bf16(gy)[:, 0].tolist() == [1.0, 2.0, 6.0, 18.0, 8.0, 15.0, 28.0, 32.0]
    # g_gates[t,j] = g_out[t] * y[comb_row[t,j]]
    assert gg.tolist() == [[1.0, 2.0], [6.0, 10.0], [18.0, 12.0], [28.0, 32.0]]


# ----------------------------------------------------------------------------- dispatch transpose


@pytest.mark.parametrize("seed", range(4))
def test_gather_backward_is_the_dense_transpose(seed):
    rng, ids, er, p = random_plan(seed)
    N, D, cap = ids.shape[0], p["D"], p["row_capacity"]
    A = np.zeros((cap, N), np.int64)                 # forward: send = A x (send[d] = x[row_token[d]])
    A[np.arange(D), p["row_token"][:D]] = 1
    G = small_int_bits(rng, (cap, 5))
    want = A.T @ bf16(G).astype(np.int64)            # integers: exact in fp32 for k <= 8
    got = oracle.gather_backward_f32chain(G, p["send_row"])
    assert np.array_equal(got, want.astype(np.float32))


@pytest.mark.parametrize("cfg", [0, 1])
def test_gather_backward_adjoint_identity(cfg):
    r = workload.make_routing(cfg)
    H = 32
    p = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)
    x = oracle._bits(workload.fill_bf16(r.N, H, 1, 3))
    G = oracle._bits(workload.fill_bf16(p["row_capacity"], H, 2, 4))
    send = oracle.gather(x, p["row_token"], p["D"])                # pinned forward
    lhs = (bf16(send).astype(np.float64) * bf16(G[:p["D"]]).astype(np.float64)).sum()
    gx = oracle.gather_backward_f32chain(G, p["send_row"]).astype(np.float64)
    rhs = (bf16(x).astype(np.float64) * gx).sum()
    mag = (np.abs(bf16(x).astype(np.float64)) *
           oracle.gather_backward_f32chain(bf16_bits_torch(np.abs(bf16(G))), p["send_row"])).sum()
    # each grad_x element is a chain of at most k fp32 adds
    assert abs(lhs - rhs) <= r.k * 2.0 ** -24 * mag + 1e-9


@pytest.mark.parametrize("seed", range(3))
def test_gather_backward_chain_exact_rational(seed):
    rng, ids, er, p = random_plan(10 + seed, N=8, k=4)
    G = oracle._bits(workload.fill_bf16(p["row_capacity"], 6, seed, 12))
    got = oracle.gather_backward_f32chain(G, p["send_row"])
    Gf = bf16(G)
    for t in range(ids.shape[0]):
        for h in range(6):
            acc = 0.0
            for j in range(ids.shape[1]):
                d = p["send_row"][t, j]
                if d >= 0:
                    acc = f32_round_exact(Fraction(acc) + Fraction(float(Gf[d, h])))
            assert float(got[t, h]) == acc


# ----------------------------------------------------------------------------- combine backward


@pytest.mark.parametrize("seed", range(4))
def test_combine_backward_grad_y_is_the_dense_transpose(seed):
    rng, ids, er, p = random_plan(20 + seed)
    N, k = ids.shape
    H, rows = 7, N * k
    gates = rng.random((N, k)).astype(np.float32)
    B = np.zeros((N, rows), np.float64)              # forward: out = B y
    for t in range(N):
        for j in range(k):
            B[t, p["comb_row"][t, j]] = gates[t, j]
    y = oracle._bits(workload.fill_bf16(rows, H, seed, 5))
    g_out = oracle._bits(workload.fill_bf16(N, H, seed, 6))
    # the forward oracle is this matrix
    assert np.allclose(oracle.combine_f64(y, gates, p["comb_row"]), B @ bf16(y).astype(np.float64),
                       rtol=1e-13, atol=1e-13)
    # B^T g is exact in float64 (one nonzero per column; fp32 x bf16 products fit 53 bits);
    # then one rounding to fp32 and one to bf16, through torch
    exact = B.T @ bf16(g_out).astype(np.float64)
    want = bf16_bits_torch(exact.astype(np.float32))
    gy, _, _ = oracle.combine_backward(y, gates, p["comb_row"], g_out)
    assert np.array_equal(gy, want)


def test_combine_backward_grad_gates_one_hot_probes():
    rng, ids, er, p = random_plan(30, N=12, k=3)
    N, k = ids.shape
    H, rows = 16, N * k
    y = oracle._bits(workload.fill_bf16(rows, H, 3, 7))
    g_out = oracle._bits(workload.fill_bf16(N, H, 3, 8))
    gates = rng.random((N, k)).astype(np.float32)
    _, gg, ga = oracle.combine_backward(y, gates, p["comb_row"], g_out)
    gof = bf16(g_out).astype(np.float64)
    for t in range(N):
        for j in range(k):
            e = np.zeros((N, k), np.float32)
            e[t, j] = 1.0
            # d<g_out, combine(y, gates)>/d gates[t,j] = <g_out, combine(y, e_tj)>
            probe = (gof * oracle.combine_f64(y, e, p["comb_row"])).sum()
            assert abs(gg[t, j] - probe) <= 1e-12 * ga[t, j] + 1e-30
            assert ga[t, j] >= abs(gg[t, j])


@pytest.mark.parametrize("seed", range(3))
def test_combine_backward_adjoint_identities_exact(seed):
    # small integers and power-of-two gates: every sum and product below is exact
    rng, ids, er, p = random_plan(40 + seed)
    N, k = ids.shape
    H, rows = 9, N * k
    y = small_int_bits(rng, (rows, H))
    g_out = small_int_bits(rng, (N, H))
    gates = (2.0 ** -rng.integers(0, 4, (N, k))).astype(np.float32)
    out = oracle.combine_f64(y, gates, p["comb_row"])
    gy, gg, _ = oracle.combine_backward(y, gates, p["comb_row"], g_out)
    gof, yf = bf16(g_out).astype(np.float64), bf16(y).astype(np.float64)
    inner = (gof * out).sum()
    assert (bf16(gy).astype(np.float64) * yf).sum() == inner     # <B^T g, y> = <g, B y>
    assert (gates.astype(np.float64) * gg).sum() == inner        # out is linear in the gates


def test_combine_backward_invalid_slot_and_untouched_rows():
    y = oracle._bits(workload.fill_bf16(6, 8, 4, 1))
    gates = np.array([[0.5, 2.0], [1.0, 3.0]], np.float32)
    comb = np.array([[0, 3], [-1, 5]], np.int32)
    g_out = oracle._bits(workload.fill_bf16(2, 8, 4, 2))
    sentinel = np.full((6, 8), 0x7fc1, np.uint16)
    gy, gg, ga = oracle.combine_backward(y, gates, comb, g_out, g_y=sentinel)
    assert gg[1, 0] == 0.0 and ga[1, 0] == 0.0
    for r in (1, 2, 4):                                          # rows no slot names
        assert (gy[r] == 0x7fc1).all()
    assert not (gy[[0, 3, 5]] == 0x7fc1).any()


@pytest.mark.parametrize("seed", range(3))
def test_combine_backward_over_plan_rows_equals_tokens(seed):
    # units = the plan's send rows (each with the dispatched g_out row of its token): the
    # slot masks partition every token's slots, so the result is the token-mode result
    rng, ids, er, p = random_plan(50 + seed)
    N, k = ids.shape
    H, rows = 12, N * k
    y = oracle._bits(workload.fill_bf16(rows, H, seed, 13))
    g_out = oracle._bits(workload.fill_bf16(N, H, seed, 14))
    gates = rng.random((N, k)).astype(np.float32)
    D = p["D"]
    gy_t, gg_t, _ = oracle.combine_backward(y, gates, p["comb_row"], g_out)
    g_rows = oracle.gather(g_out, p["row_token"], D)[:D]
    gy_r, gg_r, _ = oracle.combine_backward(y, gates, p["comb_row"], g_rows, p["row_token"],
                                            p["row_kmask"], D)
    assert np.array_equal(gy_t, gy_r)
    assert np.array_equal(gg_t, gg_r)


# ----------------------------------------------------------------------------- pre-reduced combine


@pytest.mark.parametrize("cfg", [0, 1])
def test_combine_units_over_tokens_is_the_forward_chain(cfg):
    r = workload.make_routing(cfg)
    p = oracle.plan(r.ids, r.cfg.E, r.expert_rank, r.cfg.R)
    y = oracle._bits(workload.fill_bf16(r.N * r.k, 24, 0, 15))
    a = oracle.combine_units_f32chain(y, r.gates, p["comb_row"])
    b = oracle.combine_f32chain(y, r.gates, p["comb_row"])           # pinned forward
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("seed", range(4))
def test_prereduced_equals_combine_when_nothing_rounds(seed):
    rng, ids, er, p = random_plan(60 + seed, k=4)
    N, k = ids.shape
    y = small_int_bits(rng, (N * k, 10), -4, 4)
    gates = (2.0 ** -rng.integers(0, 3, (N, k))).astype(np.float32)
    pre, out = oracle.combine_prereduced(y, gates, p)
    assert pre.shape[0] == p["D"]
    want = oracle.combine_f32chain(y, gates, p["comb_row"])
    assert np.array_equal(out, want)
    assert np.array_equal(out.astype(np.float64), oracle.combine_f64(y, gates, p["comb_row"]))


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_prereduced_within_bound_of_exact(cfg):
    r = workload.make_routing(cfg)
    c = r.cfg
    H = 16
    p = oracle.plan(r.ids, c.E, r.expert_rank, c.R)
    y = oracle._bits(workload.fill_bf16(c.N * c.k, H, 0, 16))
    pre, out = oracle.combine_prereduced(y, r.gates, p)
    exact = oracle.combine_f64(y, r.gates, p["comb_row"])
    yf = bf16(y).astype(np.float64)
    mag = sum(np.abs(r.gates[:, j, None].astype(np.float64) * yf[p["comb_row"][:, j]])
              for j in range(c.k))
    # partial rows: k fp32 fmas, then one bf16 rounding (8 significant bits: unit
    # roundoff 2^-8); then at most k fp32 adds
    bound = (2.0 ** -8 + 3 * c.k * 2.0 ** -24) * mag
    assert (np.abs(out.astype(np.float64) - exact) <= bound + 1e-30).all()
    # and it does round: the pre-reduced result is not the direct chain everywhere
    if c.k > c.E // c.R:
        assert not np.array_equal(out, oracle.combine_f32chain(y, r.gates, p["comb_row"]))


def test_gather_backward_slot_order_matters():
    # one token whose three slots go to three ranks: rows 1, 2^24, -2^24 summed in slot
    # order give 0 (1 + 2^24 rounds to 2^24), in reverse order 1
    send_row = np.array([[0, 1, 2]], np.int32)
    g = bf16_bits_torch(np.array([[1.0], [2.0 ** 24], [-2.0 ** 24]], np.float32))
    assert oracle.gather_backward_f32chain(g, send_row)[0, 0] == 0.0
    g2 = bf16_bits_torch(np.array([[-2.0 ** 24], [2.0 ** 24], [1.0]], np.float32))
    assert oracle.gather_backward_f32chain(g2, send_row)[0, 0] == 1.0
