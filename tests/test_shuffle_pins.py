"""Pins for the oracle's token shuffling (Zyphra, arxivdaily 2610.09372, English abstract:
under sequence parallelism each token moves, during the reduce-scatter after attention,
to the GPU predicted to hold its next-layer experts): the permutation (tokens grouped by
predicted home rank, ascending token order) and the reduce-scatter along it (the P
partial rows of a token added in rank order in fp32).  Pinned by a hand-worked case,
numpy's stable argsort, fancy indexing, exact integer sums and exact rational arithmetic."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workload
from test_oracle_pins import f32_round_exact


def bf16_bits(values) -> np.ndarray:
    t = torch.as_tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def test_hand_worked():
    home = [1, 0, 1, 2, 0]
    o = oracle.shuffle_order(home, 3)
    # rank 0: tokens 1, 4; rank 1: tokens 0, 2; rank 2: token 3
    assert o["row_token"][:5].tolist() == [1, 4, 0, 2, 3]
    assert o["rank_offsets"].tolist() == [0, 2, 4, 5]
    parts = bf16_bits([[[1], [2], [3], [4], [5]], [[10], [20], [30], [40], [50]]])
    out = oracle.shuffle_reduce_f32chain(parts, o["row_token"][:5])
    assert out[:, 0].tolist() == [22.0, 55.0, 11.0, 33.0, 44.0]


@pytest.mark.parametrize("seed", range(5))
def test_order_is_the_stable_sort_by_home(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(2, 65))
    N = int(rng.integers(1, 3000))
    home = rng.integers(0, R, N).astype(np.int32)
    o = oracle.shuffle_order(home, R)
    assert np.array_equal(o["row_token"][:N], np.argsort(home, kind="stable"))
    assert np.array_equal(o["rank_offsets"], np.concatenate([[0], np.cumsum(np.bincount(home, minlength=R))]))
    assert o["D"] == N and (o["send_row"][:, 0] >= 0).all()


def test_single_partial_is_the_permutation_gather():
    rng = np.random.default_rng(3)
    N, H = 500, 24
    x = oracle._bits(workload.fill_bf16(N, H, 1, 2))
    perm = rng.permutation(N).astype(np.int32)
    out = oracle.shuffle_reduce_f32chain(x[None], perm)
    assert np.array_equal(out, workload.bf16_bits_to_float(x[perm]))


@pytest.mark.parametrize("P", [2, 5, 16])
def test_integer_partials_sum_exactly(P):
    rng = np.random.default_rng(P)
    N, H = 300, 16
    vals = rng.integers(-64, 65, (P, N, H))
    parts = bf16_bits(vals.astype(np.float32))
    rt = rng.permutation(N).astype(np.int32)[:200]
    out = oracle.shuffle_reduce_f32chain(parts, rt)
    assert np.array_equal(out, vals.sum(0)[rt].astype(np.float32))


@pytest.mark.parametrize("seed", range(3))
def test_rank_order_chain_exact_rational(seed):
    rng = np.random.default_rng(20 + seed)
    P, N, H = 6, 5, 4
    parts = oracle._bits(workload.fill_bf16(P * N, H, seed, 9)).reshape(P, N, H)
    rt = rng.permutation(N).astype(np.int32)
    out = oracle.shuffle_reduce_f32chain(parts, rt)
    pf = workload.bf16_bits_to_float(parts)
    for i, t in enumerate(rt):
        for h in range(H):
            acc = 0.0
            for q in range(P):
                acc = f32_round_exact(Fraction(acc) + Fraction(float(pf[q, t, h])))
            assert float(out[i, h]) == acc


def test_invalid_token_gives_a_zero_row():
    parts = oracle._bits(workload.fill_bf16(2 * 4, 8, 0, 3)).reshape(2, 4, 8)
    out = oracle.shuffle_reduce_f32chain(parts, np.array([1, -1, 4, 2], np.int32))
    assert (out[1] == 0).all() and (out[2] == 0).all()
    assert (out[0] != 0).any()


def test_one_rank_is_the_identity():
    o = oracle.shuffle_order([0, 0, 0, 0], 1)
    assert o["row_token"][:4].tolist() == [0, 1, 2, 3]
    assert o["rank_offsets"].tolist() == [0, 4]
    with pytest.raises(ValueError):
        oracle.shuffle_order([0], 0)


def test_rank_order_matters():
    # 1 + 2^24 rounds back to 2^24 in fp32, so the rank order decides the result:
    # ((0 + 1) + 2^24) - 2^24 = 0, while the reverse order gives 1
    parts = bf16_bits(np.array([[[1.0]], [[2.0 ** 24]], [[-2.0 ** 24]]], np.float32))
    out = oracle.shuffle_reduce_f32chain(parts, np.array([0], np.int32))
    assert out[0, 0] == 0.0
