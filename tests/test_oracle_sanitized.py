"""The oracle's C code under gcc's undefined-behaviour sanitizer (CPU only).

Every parity claim rests on the oracle, so a signed overflow, an out-of-range shift or
an out-of-bounds index inside it must not pass silently.  This test compiles a second
copy of coact_oracle.c with -fsanitize=undefined (bounds checks included), points the
oracle's numpy front end at it, drives every entry point -- valid inputs, flagged
inputs and capacity overflow -- and fails on any sanitizer report.  (The same tests
also pass against an -fsanitize=address,undefined build with libasan preloaded; that
form needs the preload and is not run here.)
"""
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import workload


@pytest.fixture
def ubsan_oracle(tmp_path, monkeypatch):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    lib = str(tmp_path / "liboracle_ubsan.so")
    subprocess.check_call([gcc, "-O1", "-g", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fsanitize=undefined,bounds", "-fno-omit-frame-pointer", "-shared",
                           "-fPIC", "-o", lib, oracle._SRC, "-lm"])
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "build", lambda force=False: lib)
    yield lib


def _drive_all():
    r = workload.make_routing(0)
    cfg = r.cfg
    E, R, k, H = cfg.E, cfg.R, cfg.k, cfg.H
    ids, gates, er = r.ids[:600], r.gates[:600], r.expert_rank
    N = ids.shape[0]
    rn = np.array([0, 0, 1, 1], np.int32)
    rng = np.random.default_rng(5)
    src = rng.integers(0, R, N).astype(np.int32)

    pair, loads, _ = oracle.count(ids, E)
    C12, _, _ = oracle.count_cross(ids, E, ids[::-1].copy(), E)
    p = oracle.plan(ids, E, er, R, rank_node=rn, n_nodes=2, src_rank=src)
    oracle.plan(ids, E, er, R, row_capacity=p["D"] // 2)               # capacity flag
    bad = ids.copy()
    bad[0, 0], bad[1, 1], bad[2] = E + 3, bad[1, 0], -1                  # range, repeat
    oracle.count(bad, E)
    oracle.plan(bad, E, er, R, src_rank=np.where(np.arange(N) == 3, R + 1, src).astype(np.int32))

    x = oracle._bits(workload.fill_bf16(N, H, 0, 1))
    y = oracle._bits(workload.fill_bf16(N * k, H, 0, 2))
    oracle.gather(x, p["row_token"], p["D"])
    oracle.combine_f64(y, gates, p["comb_row"])
    oracle.combine_f32chain(y, gates, p["comb_row"])
    oracle.bf16_rne(rng.standard_normal(64).astype(np.float32))
    oracle.expand_identity(x, p["row_token"], p["row_kmask"], p["D"])
    oracle.naive_combine_identity_f32(x, gates)

    oracle.predict_home(ids, E, C12, er, R)
    oracle.place_correlated(pair, R)
    node, rank, fwd = oracle.plan_two_hop(ids, E, er, R, rn, 2, src_rank=src)
    hop1 = oracle.gather(x, node["row_token"], node["D"])
    oracle.forward_gather(hop1, fwd)
    en = rn[er]
    oracle.rebalance_ranks(loads, en, rn)
    oracle.place_two_stage(pair, loads, rn, 2)

    g_send = oracle._bits(workload.fill_bf16(max(p["D"], 1), H, 0, 4))
    oracle.gather_backward_f32chain(g_send, p["send_row"])
    D = p["D"]
    oracle.combine_units_f32chain(y, gates, p["comb_row"], p["row_token"][:D], p["row_kmask"][:D], D)
    g_out = oracle._bits(workload.fill_bf16(N, H, 0, 5))
    oracle.combine_backward(y, gates, p["comb_row"], g_out)
    oracle.combine_prereduced(y, gates, p)

    home = rng.integers(0, R, N).astype(np.int32)
    order = oracle.shuffle_order(home, R)
    parts = np.stack([oracle._bits(workload.fill_bf16(N, H, 0, 10 + q)) for q in range(3)])
    oracle.shuffle_reduce_f32chain(parts, order["row_token"][:N])

    rep, nrep, _ = oracle.place_replicas(pair, loads, er, rn, budget=3, max_rep=2)
    slot, _ = oracle.assign_replicas(ids, E, rep, nrep, R, rank_node=rn, n_nodes=2, src_rank=src)
    oracle.plan(ids, E, None, R, rank_node=rn, n_nodes=2, slot_rank=slot)
    hot_rep, hot_n = workload.replicate_hot(loads, er, rn, 2)
    oracle.assign_replicas(bad, E, hot_rep, hot_n, R, rank_node=rn, n_nodes=2)


def test_oracle_has_no_undefined_behaviour(ubsan_oracle, capfd):
    _drive_all()
    err = capfd.readouterr().err
    assert oracle._lib._name == ubsan_oracle      # the sanitized copy did the work
    assert "runtime error" not in err, err[:2000]
