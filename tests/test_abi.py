"""The C-ABI library without a GPU: it loads, exports every function include/coact.h
declares, and rejects bad arguments on the host (nothing enqueued, no CUDA call)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coact.h")


def _ensure_built():
    from conftest import build_library
    return build_library()


@pytest.fixture(scope="module")
def lib():
    path = _ensure_built()
    return ctypes.CDLL(path)


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_path():
    fns = header_functions()
    for f in ("coact_count", "plan_dispatch", "dispatch_gather", "combine_scatter",
              "predict_home", "plan_dispatch_workspace_bytes", "coact_strerror"):
        assert f in fns


def test_library_exports_every_declared_symbol(lib):
    missing = [f for f in header_functions() if not hasattr(lib, f)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(header_functions()) <= exported


def test_every_entry_point_is_declared():
    """The reverse direction: no extern "C" function of the sources is missing from the
    header (the header is the whole boundary)."""
    csrc = os.path.join(ROOT, "co_activation_b200", "csrc")
    defined = set()
    for fn in os.listdir(csrc):
        if fn.endswith((".cu", ".cuh")):
            src = open(os.path.join(csrc, fn)).read()
            defined |= set(re.findall(r'extern "C"\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(',
                                      src))
    assert defined, "no entry points found"
    assert defined == set(header_functions()), (sorted(defined - set(header_functions())),
                                                 sorted(set(header_functions()) - defined))


def test_binding_names_match_header():
    import co_activation_b200 as coact
    assert set(coact.ABI_SYMBOLS) == set(header_functions())
    for f in ("coact_count", "plan_dispatch", "dispatch_gather", "combine_scatter", "predict_home"):
        assert callable(getattr(coact, f))


def test_last_cuda_error_starts_clear(lib):
    lib.coact_last_cuda_error.restype = ctypes.c_int
    assert lib.coact_last_cuda_error() == 0


def test_strerror_and_version(lib):
    lib.coact_strerror.restype = ctypes.c_char_p
    assert lib.coact_strerror(0) == b"ok"
    assert b"workspace" in lib.coact_strerror(-4)
    import re
    hdr = open(os.path.join(ROOT, "include", "coact.h")).read()
    assert lib.coact_abi_version() == int(re.search(r"#define COACT_ABI_VERSION (\d+)", hdr).group(1))
    assert lib.coact_abi_version() == 3


P = ctypes.c_void_p
FAKE = P(256)   # a non-NULL, 16-byte aligned address the library never dereferences on host


def test_count_rejects_bad_arguments(lib):
    f = lib.coact_count
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                  P, P, P, P]
    assert f(FAKE, -1, 2, 8, None, 0, 0, FAKE, None, None, None) == -1      # N < 0
    assert f(FAKE, 10, 2, 8, None, 0, 0, None, None, None, None) == -1      # pair NULL
    assert f(FAKE, 10, 9, 8, None, 0, 0, FAKE, None, None, None) == -2      # k > 8
    assert f(FAKE, 10, 2, 1, None, 0, 0, FAKE, None, None, None) == -2      # E < 2
    assert f(FAKE, 10, 2, 2000, None, 0, 0, FAKE, None, None, None) == -2   # E > 1024
    assert f(FAKE, 10, 2, 8, FAKE, 0, 8, FAKE, None, None, None) == -2      # bad k2
    assert f(None, 0, 2, 8, None, 0, 0, FAKE, None, None, None) == 0        # N == 0: no-op


def test_plan_rejects_bad_arguments(lib):
    f = lib.plan_dispatch
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                  P, P, P, P, P, P, P, ctypes.c_int64, P, P, P, P, P, ctypes.c_size_t, P, P]
    lib.plan_dispatch_workspace_bytes.restype = ctypes.c_size_t
    lib.plan_dispatch_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    need = lib.plan_dispatch_workspace_bytes(4096, 2, 8, 4)
    assert need > 0

    def call(N=4096, k=2, E=8, R=4, ws=need, wsp=FAKE, cap=8192, n_nodes=1, rank_node=None):
        return f(FAKE, N, k, E, FAKE, R, rank_node, n_nodes, None, FAKE, FAKE, FAKE, None, FAKE,
                 FAKE, cap, FAKE, FAKE, FAKE, None, wsp, ws, None, None)

    assert call(R=65) == -2
    assert call(R=0) == -2
    assert call(k=0) == -2
    assert call(N=-5) == -1
    assert call(cap=-1) == -1
    assert call(ws=need - 1) == -4
    assert call(wsp=None) == -4
    assert call(wsp=P(264)) == -4                                  # misaligned workspace
    assert call(rank_node=FAKE, n_nodes=65) == -2


def test_gather_combine_reject_bad_arguments(lib):
    g = lib.dispatch_gather
    g.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int, P, ctypes.c_int64, P, P]
    assert g(FAKE, 10, 12, FAKE, 2, FAKE, 20, None, None) == -2    # H % 8 != 0
    assert g(P(258), 10, 16, FAKE, 2, FAKE, 20, None, None) == -1  # misaligned x
    assert g(FAKE, 10, 16, FAKE, 9, FAKE, 20, None, None) == -2    # k > 8
    assert g(None, 0, 16, None, 2, None, 0, None, None) == 0       # empty
    t = lib.dispatch_gather_tma
    t.argtypes = g.argtypes
    assert t(FAKE, 10, 12, FAKE, 2, FAKE, 20, None, None) == -2    # H % 8 != 0
    assert t(P(258), 10, 16, FAKE, 2, FAKE, 20, None, None) == -1  # misaligned x
    assert t(FAKE, 10, 16392, FAKE, 2, FAKE, 20, None, None) == -2  # row above 32 KB
    assert t(None, 0, 16, None, 2, None, 0, None, None) == 0       # empty
    c = lib.combine_scatter
    c.argtypes = [P, ctypes.c_int64, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, P,
                  ctypes.c_int, P, P]
    assert c(FAKE, 20, FAKE, FAKE, 10, 2, 16, FAKE, 2, None, None) == -2   # out dtype
    assert c(FAKE, 20, None, FAKE, 10, 2, 16, FAKE, 0, None, None) == -1   # gates NULL
    assert c(FAKE, 20, FAKE, FAKE, 10, 2, 16, P(260), 0, None, None) == -1  # misaligned out
    assert c(None, 0, None, None, 0, 2, 16, None, 0, None, None) == 0      # empty


def test_backward_entry_points_reject_bad_arguments(lib):
    b = lib.dispatch_gather_backward
    b.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, P, ctypes.c_int,
                  P, P]
    assert b(FAKE, 20, FAKE, 10, 2, 12, FAKE, 0, None, None) == -2     # H % 8 != 0
    assert b(FAKE, 20, FAKE, 10, 2, 16, FAKE, 2, None, None) == -2     # out dtype
    assert b(FAKE, 20, None, 10, 2, 16, FAKE, 0, None, None) == -1     # send_row NULL
    assert b(P(258), 20, FAKE, 10, 2, 16, FAKE, 0, None, None) == -1   # misaligned grad_send
    assert b(None, 0, None, 0, 2, 16, None, 0, None, None) == 0        # empty
    c = lib.combine_rows
    c.argtypes = [P, ctypes.c_int64, P, P, ctypes.c_int64, ctypes.c_int, P, P, ctypes.c_int64, P,
                  ctypes.c_int64, P, ctypes.c_int, P, P]
    assert c(FAKE, 20, FAKE, FAKE, 10, 2, None, FAKE, 5, None, 16, FAKE, 0, None, None) == -1
    assert c(FAKE, 20, FAKE, FAKE, 10, 9, FAKE, FAKE, 5, None, 16, FAKE, 0, None, None) == -2
    assert c(FAKE, 20, FAKE, FAKE, 10, 2, FAKE, FAKE, 5, None, 16, P(260), 0, None, None) == -1
    assert c(None, 0, None, None, 0, 2, None, None, 0, None, 16, None, 0, None, None) == 0
    s = lib.combine_scatter_backward
    s.argtypes = [P, ctypes.c_int64, P, P, ctypes.c_int64, ctypes.c_int, P, P, ctypes.c_int64, P, P,
                  ctypes.c_int64, P, P, P, P]
    assert s(FAKE, 20, FAKE, FAKE, 10, 2, None, None, 0, None, FAKE, 12, FAKE, FAKE, None, None) == -2
    assert s(FAKE, 20, FAKE, FAKE, 10, 2, None, None, 0, None, FAKE, 16, FAKE, None, None, None) == -1
    assert s(FAKE, 20, FAKE, FAKE, 10, 2, FAKE, None, 4, None, FAKE, 16, FAKE, FAKE, None, None) == -1
    assert s(FAKE, 20, FAKE, FAKE, 10, 2, None, None, 0, None, P(264), 16, FAKE, FAKE, None,
             None) == -1
    assert s(None, 0, None, None, 0, 2, None, None, 0, None, None, 16, None, None, None, None) == 0


def test_shuffle_rejects_bad_arguments(lib):
    f = lib.shuffle_reduce_scatter
    f.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, P,
                  ctypes.c_int, P, P]
    assert f(FAKE, 4, 100, 12, FAKE, 10, FAKE, 0, None, None) == -2     # H % 8 != 0
    assert f(FAKE, 0, 100, 16, FAKE, 10, FAKE, 0, None, None) == -2     # P < 1
    assert f(FAKE, 65, 100, 16, FAKE, 10, FAKE, 0, None, None) == -2    # P > 64
    assert f(FAKE, 4, 100, 16, FAKE, 10, FAKE, 2, None, None) == -2     # out dtype
    assert f(None, 4, 100, 16, FAKE, 10, FAKE, 0, None, None) == -1     # bases NULL
    assert f(FAKE, 4, 100, 16, FAKE, 10, P(264), 0, None, None) == -1   # misaligned out
    assert f(None, 4, 100, 16, None, 0, None, 0, None, None) == 0       # nothing to write


def test_replica_entry_points_reject_bad_arguments(lib):
    a = lib.assign_replicas
    a.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                  P, ctypes.c_int, P, P, P, P]
    assert a(FAKE, 10, 2, 8, FAKE, 9, FAKE, 4, None, 1, None, FAKE, None, None) == -2   # max_rep 9
    assert a(FAKE, 10, 2, 8, FAKE, 0, FAKE, 4, None, 1, None, FAKE, None, None) == -2   # max_rep 0
    assert a(FAKE, 10, 2, 8, None, 2, FAKE, 4, None, 1, None, FAKE, None, None) == -1   # no table
    assert a(FAKE, 10, 2, 8, FAKE, 2, FAKE, 65, None, 1, None, FAKE, None, None) == -2  # R > 64
    assert a(None, 0, 2, 8, None, 2, None, 4, None, 1, None, None, None, None) == 0     # empty
    p = lib.plan_dispatch_slots
    p.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                  P, P, P, P, P, P, P, ctypes.c_int64, P, P, P, P, P, ctypes.c_size_t, P, P]
    args = [FAKE, 10, 2, 8, None, 4, None, 1, None, FAKE, FAKE, FAKE, None, FAKE, FAKE, 20, FAKE,
            FAKE, FAKE, None, FAKE, 1 << 20, None, None]
    assert p(*args) == -1                                           # slot_rank NULL
    args[4] = FAKE
    args[2] = 9
    assert p(*args) == -2                                           # k > 8


def test_forward_gather_tokens_rejects_bad_arguments(lib):
    f = lib.forward_gather_tokens
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, ctypes.c_int, P,
                  ctypes.c_int64, P, P, P]
    assert f(FAKE, 10, 12, FAKE, 5, 2, FAKE, 20, FAKE, None, None) == -2     # H % 8 != 0
    assert f(FAKE, 10, 16, FAKE, 5, 9, FAKE, 20, FAKE, None, None) == -2     # k > 8
    assert f(FAKE, 10, 16, None, 5, 2, FAKE, 20, FAKE, None, None) == -1     # send_row NULL
    assert f(P(258), 10, 16, FAKE, 5, 2, FAKE, 20, FAKE, None, None) == -1   # misaligned src
    assert f(None, 0, 16, None, 0, 2, None, 0, None, None, None) == 0        # empty


def test_predict_rejects_bad_arguments(lib):
    p = lib.predict_home
    p.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                  P, P, ctypes.c_size_t, P, P]
    assert p(FAKE, 10, 2, 8, FAKE, 8, FAKE, 65, FAKE, FAKE, 4096, None, None) == -2
    assert p(FAKE, 10, 2, 8, FAKE, 8, FAKE, 4, FAKE, FAKE, 8, None, None) == -4


def test_binding_fails_loudly_without_library():
    env = dict(os.environ, COACT_LIB="/nonexistent/libcoact.so")
    r = subprocess.run([sys.executable, "-c", "import co_activation_b200"], cwd=ROOT, env=env,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libcoact.so not found" in r.stderr


def test_two_hop_and_planner_reject_bad_arguments(lib):
    c = lib.coact_compose_map
    c.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, P, P, P]
    assert c(FAKE, -1, FAKE, 4, FAKE, None, None) == -1
    assert c(None, 5, FAKE, 4, FAKE, None, None) == -1
    assert c(None, 0, None, 0, None, None, None) == 0
    f = lib.plan_forward
    f.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int,
                  P, P, P, P, ctypes.c_int64, P, P]
    assert f(FAKE, 10, 9, 8, FAKE, 4, None, 1, FAKE, FAKE, FAKE, FAKE, 20, None, None) == -2  # k
    assert f(FAKE, 10, 2, 8, FAKE, 65, None, 1, FAKE, FAKE, FAKE, FAKE, 20, None, None) == -2  # R
    assert f(FAKE, 10, 2, 8, FAKE, 4, None, 1, None, FAKE, FAKE, FAKE, 20, None, None) == -1   # send_row
    assert f(FAKE, 10, 2, 8, FAKE, 4, None, 1, FAKE, FAKE, FAKE, None, 20, None, None) == -1   # fwd_src
    g = lib.forward_gather
    g.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, P, P, P]
    assert g(FAKE, 10, 12, FAKE, 5, FAKE, None, None) == -2      # H % 8
    assert g(P(264), 10, 16, FAKE, 5, FAKE, None, None) == -1    # misaligned src
    assert g(FAKE, 10, 16, None, 5, FAKE, None, None) == -1      # fwd_src NULL
    r = lib.coact_rebalance_ranks
    r.argtypes = [P, P, ctypes.c_int, P, ctypes.c_int, P]
    loads = (ctypes.c_int64 * 4)(4, 3, 2, 1)
    en = (ctypes.c_int32 * 4)(0, 0, 1, 1)
    rn = (ctypes.c_int32 * 2)(0, 1)
    out = (ctypes.c_int32 * 4)()
    assert r(loads, en, 4, rn, 2, out) == 0 and list(out) == [0, 0, 1, 1]
    bad = (ctypes.c_int32 * 4)(0, 0, 0, 1)                        # node 0 holds 3 of 2 slots
    assert r(loads, bad, 4, rn, 2, out) == -1
    assert r(loads, en, 4, rn, 3, out) == -2                      # 4 % 3 != 0


def test_row_meta_calls_reject_bad_arguments(lib):
    """plan_row_meta / gather_row_slots: host-detectable errors return a status before
    anything is enqueued (no GPU needed to see them)."""
    f, g = lib.plan_row_meta, lib.gather_row_slots
    I64, I32 = ctypes.c_int64, ctypes.c_int
    f.argtypes = [P, P, I64, P, I32, P, P, P, I64, I32, P, P, P, P, P, P]
    g.argtypes = [P, I64, P, P, I64, I32, P, P, P]
    ok = dict(rt=FAKE, km=FAKE, cap=10, ro=FAKE, R=4, ids=FAKE, gates=FAKE, comb=FAKE, N=5, k=2,
              base=None, ex=FAKE, gt=FAKE, sl=FAKE)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["rt"], a["km"], a["cap"], a["ro"], a["R"], a["ids"], a["gates"], a["comb"],
                 a["N"], a["k"], a["base"], a["ex"], a["gt"], a["sl"], None, None)

    assert call(N=-1) == -1 and call(cap=-1) == -1
    assert call(k=0) == -2 and call(k=9) == -2 and call(R=0) == -2 and call(R=65) == -2
    assert call(ro=None) == -1
    assert call(ids=None) == -1 and call(gates=None) == -1 and call(comb=None) == -1
    assert call(rt=None) == -1 and call(km=None) == -1
    assert call(cap=0) == 0                                   # nothing to do
    assert call(ex=None, gt=None, sl=None, rt=None, km=None) == 0
    assert g(FAKE, 4, FAKE, FAKE, -1, 2, FAKE, None, None) == -1
    assert g(FAKE, 4, FAKE, FAKE, 5, 0, FAKE, None, None) == -2
    assert g(FAKE, 4, None, FAKE, 5, 2, FAKE, None, None) == -1
    assert g(None, 4, FAKE, FAKE, 5, 2, FAKE, None, None) == -1
    assert g(FAKE, 4, FAKE, FAKE, 0, 2, FAKE, None, None) == 0


def test_rebalance_ranks_rejects_bad_arguments(lib):
    f = lib.rebalance_ranks
    I32 = ctypes.c_int
    f.argtypes = [P, P, I32, P, I32, I32, P, P, P]
    assert f(None, FAKE, 8, FAKE, 4, 2, FAKE, None, None) == -1
    assert f(FAKE, FAKE, 8, FAKE, 4, 2, None, None, None) == -1
    assert f(FAKE, FAKE, 9, FAKE, 4, 2, FAKE, None, None) == -2       # E % R != 0
    assert f(FAKE, FAKE, 1, FAKE, 1, 1, FAKE, None, None) == -2       # E < 2
    assert f(FAKE, FAKE, 2048, FAKE, 4, 1, FAKE, None, None) == -2    # E > 1024
    assert f(FAKE, FAKE, 8, FAKE, 4, 0, FAKE, None, None) == -2       # no node
    assert f(FAKE, FAKE, 128, FAKE, 128, 2, FAKE, None, None) == -2   # R > 64
