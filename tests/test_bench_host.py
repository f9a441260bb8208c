"""Host-side helpers of bench.py that its JSON line depends on (CPU only): the launch
count behind `gpu_launches`, the source-tied DRAM traffic behind `roofline.traffic`, and
the receive-side balance."""
import os
import re
import shutil

import numpy as np
import pytest
import torch

import bench

CSRC = os.path.join(bench.ROOT, "co_activation_b200", "csrc")


def _plan_constants():
    src = open(os.path.join(CSRC, "plan.cu")).read()
    tile = int(re.search(r"constexpr int kTile = (\d+);", src).group(1))
    small = int(re.search(r"#define COACT_PLAN_SMALL_MAX (\d+)", src).group(1))
    return tile, small


@pytest.mark.parametrize("R,N", [(1, 0), (8, 0), (8, 1), (8, 16384), (64, 16384), (64, 16385),
                                 (16, 65536), (17, 65536), (32, 65536), (64, 131072)])
def test_plan_launches_matches_the_library(R, N):
    """plan_dispatch folds the scan into the scatter kernel when R x tiles is small (two
    launches: tiles + scatter); otherwise tiles + scan + scatter; N = 0 runs scan + scatter."""
    tile, small = _plan_constants()
    n_tiles = -(-N // tile)
    expect = 2 if n_tiles == 0 or R * n_tiles <= small else 3
    assert bench.plan_launches(R, N) == expect


def _fake_root(tmp_path):
    root = tmp_path / "root"
    shutil.copytree(CSRC, root / "co_activation_b200" / "csrc")
    (root / "profiles").mkdir()
    return root


def test_read_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_hash("k_combine_v16")
    (root / "profiles" / "dram_traffic.txt").write_text(
        "# kernel workload bytes sha\n"
        f"k_combine_v16 config1 123456789 {sha}\n"
        "k_gather_v16 config1 987654321 0000000000000000\n")
    assert bench.read_traffic("k_combine_v16", "config1") == 123456789
    assert bench.read_traffic("k_combine_v16", "config2") is None       # other workload
    assert bench.read_traffic("k_gather_v16", "config1") is None        # stale hash
    assert bench.read_traffic("k_not_a_kernel", "config1") is None
    # any change to a source the kernel is built from retires the figure
    for fn in bench.KERNEL_SOURCES["k_combine_v16"]:
        p = root / "co_activation_b200" / "csrc" / fn
        p.write_text(p.read_text() + "\n// edited\n")
        assert bench.read_traffic("k_combine_v16", "config1") is None
        p.write_text(p.read_text()[: -len("\n// edited\n")])
        assert bench.read_traffic("k_combine_v16", "config1") == 123456789


def test_committed_traffic_lines_are_well_formed():
    """Every committed traffic line names a known kernel, a workload and a 16-hex hash."""
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.txt")
    lines = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert lines
    for kern, work, nbytes, sha in lines:
        assert kern in bench.KERNEL_SOURCES
        assert re.fullmatch(r"config\d", work)
        assert int(nbytes) > 0
        assert re.fullmatch(r"[0-9a-f]{16}", sha)


class _Plan:
    def __init__(self, counts, asg_offsets):
        self.rank_counts = torch.tensor(counts, dtype=torch.int32)
        self.asg_offsets = torch.tensor(asg_offsets, dtype=torch.int32)


def test_rank_balance():
    b = bench.rank_balance(_Plan([2, 4, 6], [0, 3, 9, 12]))
    assert b["rank_rows_max_over_mean"] == pytest.approx(1.5)
    assert b["rank_asg_max_over_mean"] == pytest.approx(1.5)
    even = bench.rank_balance(_Plan([5, 5], [0, 7, 14]))
    assert even == {"rank_rows_max_over_mean": 1.0, "rank_asg_max_over_mean": 1.0}
    empty = bench.rank_balance(_Plan([0, 0], [0, 0, 0]))
    assert empty == {"rank_rows_max_over_mean": 0.0, "rank_asg_max_over_mean": 0.0}
    assert np.isfinite(list(b.values())).all()
