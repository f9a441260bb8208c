"""Pins of the oracle's EP row metadata (CPU): what a rank receiving a deduplicated row
needs besides the row -- each served slot's expert id, gate and output position -- and
the way back of one value per (send row, slot) to token order (e.g. gate gradients).
Cobalt and Zyphra, English abstracts: under expert parallelism each token travels to the
ranks of its experts, which send their results back to be combined."""
import numpy as np
import pytest

import oracle
from test_oracle_pins import rand_ids


def test_hand_worked():
    # experts 0, 1 on rank 0 and 2, 3 on rank 1
    ids = np.array([[0, 2], [1, 0], [3, 2]], np.int32)
    gates = np.array([[0.625, 0.375], [0.75, 0.25], [0.5, 0.5]], np.float32)
    p = oracle.plan(ids, 4, [0, 0, 1, 1], 2)
    # rank 0: token 0 (slot 0), token 1 (slots 0, 1); rank 1: token 0 (slot 1), token 2
    assert p["row_token"][:4].tolist() == [0, 1, 0, 2]
    assert p["row_kmask"][:4].tolist() == [0b01, 0b11, 0b10, 0b11]
    assert p["comb_row"].tolist() == [[0, 3], [1, 2], [4, 5]]
    ex, g, sl, f = oracle.row_meta(p, ids, gates)
    assert f == 0
    assert ex.tolist() == [[0, -1], [1, 0], [-1, 2], [3, 2]]
    assert g.tolist() == [[0.625, 0.0], [0.75, 0.25], [0.0, 0.375], [0.5, 0.5]]
    assert sl.tolist() == [[0, -1], [1, 2], [-1, 3], [4, 5]]
    # slot_base[r] = 10 - asg_offsets[0], 20 - asg_offsets[1]: outputs at 10.. and 20..
    _, _, sl, _ = oracle.row_meta(p, ids, gates, slot_base=[10 - 0, 20 - 3])
    assert sl.tolist() == [[10, -1], [11, 12], [-1, 20], [21, 22]]
    back, f = oracle.gather_row_slots(g, p["send_row"], p["row_kmask"])
    assert f == 0 and back.tolist() == gates.tolist()


def _plan_with_invalid(seed):
    rng = np.random.default_rng(seed)
    N, E, k, R = 300, 16, int(rng.integers(1, 6)), int(rng.integers(1, 9))
    ids = rand_ids(rng, N, E, k)
    ids[3, 0] = E + 4                              # invalid tokens: no rows at all
    if k > 1:
        ids[9, 1] = ids[9, 0]
    er = rng.integers(0, R, E).astype(np.int32)
    gates = rng.random((N, k)).astype(np.float32)
    return ids, gates, er, R, oracle.plan(ids, E, er, R)


@pytest.mark.parametrize("seed", range(12))
def test_expert_ids_and_gates_are_the_slots_rows_serve(seed):
    ids, gates, er, R, p = _plan_with_invalid(seed)
    D, k = p["D"], ids.shape[1]
    ex, g, _, f = oracle.row_meta(p, ids, gates)
    assert f == 0
    tok = p["row_token"][:D]
    bits = ((p["row_kmask"][:D, None].astype(np.int64) >> np.arange(k)) & 1).astype(bool)
    assert np.array_equal(ex, np.where(bits, ids[tok], -1))
    assert np.array_equal(g, np.where(bits, gates[tok], 0.0).astype(np.float32))
    # every slot of every valid token is served by exactly one send row, on its rank
    valid = np.ones(len(ids), bool)
    valid[[3, 9] if k > 1 else [3]] = False
    hits = np.zeros(ids.shape, np.int64)
    np.add.at(hits, (np.repeat(tok, k)[bits.ravel()], np.tile(np.arange(k), D)[bits.ravel()]), 1)
    assert (hits[valid] == 1).all() and (hits[~valid] == 0).all()


@pytest.mark.parametrize("seed", range(12))
def test_slots_are_the_expanded_receive_order(seed):
    """With slot_base[r] = -asg_offsets[r], the served slots of rank r's rows, listed row by
    row and slot by slot in ascending order, are 0, 1, 2, ... (the expanded receive
    order), computed here from the masks alone by a running count of set bits."""
    ids, gates, er, R, p = _plan_with_invalid(100 + seed)
    k = ids.shape[1]
    ao, ro = p["asg_offsets"], p["rank_offsets"]
    _, _, sl, _ = oracle.row_meta(p, ids, gates, slot_base=-ao[:R])
    for r in range(R):
        km = p["row_kmask"][ro[r]:ro[r + 1]].astype(np.int64)
        bits = ((km[:, None] >> np.arange(k)) & 1).astype(bool)
        run = np.cumsum(bits.ravel()).reshape(bits.shape) - 1
        want = np.where(bits, run, -1)
        assert np.array_equal(sl[ro[r]:ro[r + 1]], want), r
        assert bits.sum() == ao[r + 1] - ao[r]


@pytest.mark.parametrize("seed", range(12))
def test_gather_row_slots_brute_force(seed):
    ids, gates, er, R, p = _plan_with_invalid(200 + seed)
    N, k = ids.shape
    D = p["D"]
    vals = np.random.default_rng(seed).standard_normal((D, k)).astype(np.float32)
    got, f = oracle.gather_row_slots(vals, p["send_row"], p["row_kmask"])
    assert f == 0
    want = np.zeros((N, k), np.float32)
    for d in range(D):                       # every row, every slot it holds
        for j in range(k):
            if (p["row_kmask"][d] >> j) & 1:
                want[p["row_token"][d], j] = vals[d, j]
    assert np.array_equal(got, want)
    # the round trip of the gates through the rows gives the gates of the valid tokens
    _, g, _, _ = oracle.row_meta(p, ids, gates)
    back, _ = oracle.gather_row_slots(g, p["send_row"], p["row_kmask"])
    valid = (p["send_row"] >= 0).any(axis=1)
    assert np.array_equal(back[valid], gates[valid]) and (back[~valid] == 0).all()


def test_flags():
    ids = np.array([[0, 1], [1, 2]], np.int32)
    p = oracle.plan(ids, 4, [0, 1, 1, 0], 2)
    bad = dict(p)
    bad["row_token"] = p["row_token"].copy()
    bad["row_token"][0] = 7                    # a token outside [0, N)
    ex, g, sl, f = oracle.row_meta(bad, ids, np.ones((2, 2), np.float32))
    assert f == 16 and (ex[0] == -1).all() and (g[0] == 0).all() and (sl[0] == -1).all()
    sr = p["send_row"].copy()
    sr[1, 0] = 99                              # a send row beyond n_rows: skipped
    out, f = oracle.gather_row_slots(np.ones((p["D"], 2), np.float32), sr, p["row_kmask"])
    assert f == 16
