"""Pins for the shared input generator: calibration against the pages' routing
statistic, and the bulk bf16 hash against an independent uint64 formulation."""
import numpy as np
import pytest

import workload


def test_config1_coselect_share_matches_pages(pages_figures):
    fig = pages_figures["coselect_share_top2"]
    cfg = workload.CONFIGS[1]
    pairs = cfg.E * (cfg.E - 1) // 2
    assert abs(cfg.n_groups / pairs - fig["pairs_fraction"]) < 0.0005   # 16 of 2016 pairs
    r = workload.make_routing(cfg)
    share = workload.pages_stats(r)["group_coselect_share"]
    assert abs(share - fig["token_share"]) < 0.015


def test_routing_shapes_and_gates():
    for c in (0, 1, 2):
        r = workload.make_routing(c)
        cfg = r.cfg
        assert r.ids.shape == (cfg.N, cfg.k) and r.ids.dtype == np.int32
        assert ((r.ids >= 0) & (r.ids < cfg.E)).all()
        assert all(len(set(row)) == cfg.k for row in r.ids[:2000].tolist())
        assert np.allclose(r.gates.sum(1), 1.0, atol=1e-5)
        assert (np.diff(r.gates, axis=1) <= 0).all()         # slot order = descending logit
        assert np.bincount(r.expert_rank, minlength=cfg.R).tolist() == [cfg.epr] * cfg.R
        assert r.rank_node.max() == cfg.n_nodes - 1


def test_routing_deterministic():
    a, b = workload.make_routing(2), workload.make_routing(2)
    assert np.array_equal(a.ids, b.ids) and np.array_equal(a.gates, b.gates)
    c = workload.make_routing(2, seed=1)
    assert not np.array_equal(a.ids, c.ids)


def test_planted_and_roundrobin_placement():
    cfg = workload.CONFIGS[3]
    r = workload.make_routing(cfg.with_(N=256), placement_kind="planted")
    er = r.expert_rank
    for g in r.groups:                                      # every planted pair co-located
        assert er[g[0]] == er[g[1]]
    rr = workload.placement(cfg, "roundrobin")
    assert rr.tolist() == [e % cfg.R for e in range(cfg.E)]


def test_two_layer_structure():
    tl = workload.make_two_layer(4, N=4096)
    ids2 = tl.layer2.ids
    assert (ids2[:, 0] != ids2[:, 1]).all()
    # the 4 heavy successors take ~70% of layer-2 picks (redraws shift it a little)
    heavy = np.mean([ids2[t, j] in tl.succ[tl.layer1.ids[t, j]]
                     for t in range(2000) for j in range(2)])
    assert 0.62 < heavy < 0.76
    assert tl.calib1.shape == tl.layer1.ids.shape


def _ref_value(key, i, h, H):
    M = (1 << 64) - 1
    z = (i * H + h + (key % (1 << 64))) & M
    z = (z + 0x9E3779B97F4A7C15) & M
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    z ^= z >> 31
    s = (z & 0xFFFF) + ((z >> 16) & 0xFFFF) + ((z >> 32) & 0xFFFF)
    f = np.float32((2 * s - 196605) * 2.0 ** -16)
    u = int(f.view(np.uint32))
    kept, dropped = u >> 16, u & 0xFFFF
    if dropped > 0x8000 or (dropped == 0x8000 and kept & 1):
        kept += 1
    return kept & 0xFFFF


def test_fill_bf16_matches_uint64_reference():
    import torch
    H = 96
    x = workload.fill_bf16(50, H, 5, 7)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    key = workload._stream_key(5, 7)
    rng = np.random.default_rng(0)
    for _ in range(300):
        i, h = int(rng.integers(50)), int(rng.integers(H))
        assert bits[i, h] == _ref_value(key, i, h, H)
    # row_ids / row0 regenerate the same rows
    sub = workload.fill_bf16(3, H, 5, 7, row_ids=[49, 0, 7])
    assert torch.equal(sub, x[[49, 0, 7]])
    assert torch.equal(workload.fill_bf16(10, H, 5, 7, row0=40), x[40:50])
    f = x.float()
    assert abs(f.mean().item()) < 0.02 and abs(f.std().item() - 1.0) < 0.02
