"""The programmatic-dependent-launch contract of the library's kernels, checked on their
source (CPU only).

Every kernel is launched with programmatic stream serialisation, so it may start before
its predecessor on the stream has finished.  Correctness rests on two rules:
  * before its pdl_wait() a kernel touches no global memory through loads, stores or
    atomics -- except k_plan_scatter, the second kernel of plan_dispatch, which reads the
    call's own inputs (its predecessor is the call's own k_plan_tiles / k_plan_scan);
    an L2 prefetch (prefetch_l2_bulk) is allowed anywhere, it reads nothing in;
  * a kernel triggers its dependents only after its own pdl_wait(); k_plan_scatter, the
    last kernel of plan_dispatch, triggers nothing (its successor, usually the dispatch
    gather, launches when it completes, on SMs free of the scatter's blocks).
"""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(__file__), "..", "co_activation_b200", "csrc")
NO_TRIGGER = {"k_plan_scatter"}
PRE_WAIT_READS_OK = {"k_plan_scatter"}
GLOBAL_ACCESS = re.compile(r"__ldg\(|ld_stream\(|st_stream\(|__stcs\(|atomic[A-Z][a-z]+\(|"
                           r"cp\.async\.bulk\.(?!prefetch)|\bld\.global|\bst\.global")


def _kernels():
    """(file, kernel name, body text) of every __global__ function."""
    out = []
    for fn in sorted(os.listdir(CSRC)):
        if not fn.endswith(".cu"):
            continue
        src = open(os.path.join(CSRC, fn)).read()
        for m in re.finditer(r"__global__[^{;]*?\b(k_\w+)\s*\(", src):
            i = src.index("{", m.end())
            depth, j = 0, i
            while True:
                if src[j] == "{":
                    depth += 1
                elif src[j] == "}":
                    depth -= 1
                    if depth == 0:
                        break
                j += 1
            out.append((fn, m.group(1), src[i:j + 1]))
    return out


KERNELS = _kernels()


def test_kernels_found():
    names = {k for _, k, _ in KERNELS}
    for k in ("k_count_smem", "k_plan_tiles", "k_plan_scatter", "k_gather_v16",
              "k_combine_v16", "k_combine_bwd", "k_shuffle_reduce", "k_gather_peer"):
        assert k in names


@pytest.mark.parametrize("fn,name,body", KERNELS, ids=[k for _, k, _ in KERNELS])
def test_wait_then_trigger(fn, name, body):
    waits = [m.start() for m in re.finditer(r"\bpdl_wait\(\);", body)]
    trigs = [m.start() for m in re.finditer(r"\bpdl_trigger\(\);", body)]
    assert len(waits) == 1, f"{fn}:{name} waits {len(waits)} times"
    if name in NO_TRIGGER:
        assert not trigs, f"{fn}:{name} triggers its dependents"
    else:
        assert trigs, f"{fn}:{name} never triggers its dependents"
        assert min(trigs) > waits[0], f"{fn}:{name} triggers before its wait"
    pre = body[:waits[0]]
    if name not in PRE_WAIT_READS_OK:
        hit = GLOBAL_ACCESS.search(pre)
        assert hit is None, f"{fn}:{name} touches global memory before its wait: {hit.group(0)}"


def test_scatter_is_last_kernel_of_plan():
    """k_plan_scatter, which reads its call's inputs before its wait, is the last launch of
    plan_dispatch (and of its variants): every kernel before it in the call triggers only
    after its own wait, so when it starts, everything before the call has completed."""
    src = open(os.path.join(CSRC, "plan.cu")).read()
    body = src[src.index("int launch_plan("):]
    body = body[:body.index("\n}\n")]
    launches = re.findall(r"launch_pdl\((k_\w+)", body)
    assert launches[-1] == "k_plan_scatter"
    returns = re.findall(r"return launch_pdl\((k_\w+)", body)
    assert set(returns) == {"k_plan_scatter"}
