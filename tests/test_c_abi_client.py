"""The C ABI from plain C programs (cudaMalloc'd buffers, their own CUDA streams, no
Python or torch in the loop): they compile against include/coact.h and libcoact.so (CPU
tests), and on a GPU their results equal the oracle's bit for bit (GPU tests):
tests/c_abi/path.c runs count, plan, gather and combine; tests/c_abi/reset.c runs the
count (shared-memory histogram) and the no-allocation planner before and after a device
reset, which ends the process's context and unloads the library's module."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "path.c")
RESET_SRC = os.path.join(ROOT, "tests", "c_abi", "reset.c")
LIBDIR = os.path.join(ROOT, "co_activation_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def compile_client(out_path, src=SRC):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cmd = [cc, "-std=c11", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), src, "-L", LIBDIR, "-lcoact",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{LIBDIR}", "-o", out_path]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_client_compiles(tmp_path):
    compile_client(str(tmp_path / "path"))
    compile_client(str(tmp_path / "reset"), RESET_SRC)


@pytest.mark.gpu
def test_client_path_matches_oracle(tmp_path):
    exe = str(tmp_path / "path")
    compile_client(exe)
    r = workload.make_routing(1, N=3001)            # ragged: not a multiple of any tile
    c = r.cfg
    N, k, E, R, H = r.N, r.k, c.E, c.R, 64
    x = oracle._bits(workload.fill_bf16(N, H, 0, 1))
    y = oracle._bits(workload.fill_bf16(N * k, H, 0, 2))
    inp, outp = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(np.array([N, k, E, R, H], np.int32).tobytes())
        f.write(np.ascontiguousarray(r.ids, np.int32).tobytes())
        f.write(np.ascontiguousarray(r.gates, np.float32).tobytes())
        f.write(np.ascontiguousarray(r.expert_rank, np.int32).tobytes())
        f.write(x.tobytes())
        f.write(y.tobytes())
    p = subprocess.run([exe, str(inp), str(outp)], capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    o = oracle.plan(r.ids, E, r.expert_rank, R)
    D = o["D"]
    buf = open(outp, "rb").read()
    pos = 0

    def take(dtype, n):
        nonlocal pos
        a = np.frombuffer(buf, dtype=dtype, count=n, offset=pos)
        pos += a.nbytes
        return a

    assert take(np.int32, 1)[0] == 0                                  # device error flags
    pair, loads, _ = oracle.count(r.ids, E)
    assert np.array_equal(take(np.int64, E * E).reshape(E, E), pair)
    assert np.array_equal(take(np.int64, E), loads)
    assert np.array_equal(take(np.int32, R + 1), o["rank_offsets"])
    assert np.array_equal(take(np.int32, N * k).reshape(N, k), o["send_row"])
    assert np.array_equal(take(np.int32, N * k).reshape(N, k), o["comb_row"])
    assert np.array_equal(take(np.uint16, D * H).reshape(D, H), x[o["row_token"][:D]])
    want = oracle.combine_f32chain(y, r.gates, o["comb_row"])
    assert np.array_equal(take(np.float32, N * H).reshape(N, H).view(np.uint32), want.view(np.uint32))
    assert pos == len(buf)


@pytest.mark.gpu
def test_calls_across_a_device_reset_match_oracle(tmp_path):
    """Per-context state (the count kernel's shared-memory opt-in, the device address of
    the no-allocation planner's scratch) is set up again in the new context: both rounds
    equal the oracle."""
    exe = str(tmp_path / "reset")
    compile_client(exe, RESET_SRC)
    r = workload.make_routing(3, N=5000)             # E = 256: the shared-memory histogram
    c = r.cfg
    N, k, E, R = r.N, r.k, c.E, c.R
    inp, outp = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(np.array([N, k, E, R, c.n_nodes], np.int32).tobytes())
        f.write(np.ascontiguousarray(r.ids, np.int32).tobytes())
        f.write(np.ascontiguousarray(r.expert_rank, np.int32).tobytes())
        f.write(np.ascontiguousarray(r.rank_node, np.int32).tobytes())
    p = subprocess.run([exe, str(inp), str(outp)], capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    pair, loads, _ = oracle.count(r.ids, E)
    o = oracle.plan(r.ids, E, r.expert_rank, R, rank_node=r.rank_node, n_nodes=c.n_nodes)
    buf = open(outp, "rb").read()
    pos = 0

    def take(dtype, n):
        nonlocal pos
        a = np.frombuffer(buf, dtype=dtype, count=n, offset=pos)
        pos += a.nbytes
        return a

    for _ in range(2):                                # before and after the reset
        assert take(np.int32, 1)[0] == 0
        assert np.array_equal(take(np.int64, E * E).reshape(E, E), pair)
        assert np.array_equal(take(np.int64, E), loads)
        assert np.array_equal(take(np.int32, R + 1), o["rank_offsets"])
        assert np.array_equal(take(np.int32, N * k).reshape(N, k), o["send_row"])
        assert np.array_equal(take(np.int32, N * k).reshape(N, k), o["comb_row"])
        assert np.array_equal(take(np.int64, 8), o["stats"])
    assert pos == len(buf)
