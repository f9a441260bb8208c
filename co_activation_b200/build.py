"""Builds libcoact.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python co_activation_b200/build.py [--force] [-D NAME=VALUE ...] [--out PATH]

(run by path: importing the package itself requires the built library)

Each csrc/*.cu compiles to an object under _build/ (parallel), then links into
co_activation_b200/libcoact.so.  Only B200 code is generated
(-gencode arch=compute_100a,code=sm_100a).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcoact.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libcoact.so")
    return path


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, defines=(), out: str = LIB, verbose: bool = False,
          ptxas_verbose: bool = False) -> str:
    """Compile and link; returns the library path.  Rebuilds only what is stale unless
    `force` or `defines` are given (experiment builds go to a separate `out`)."""
    srcs = _sources()
    deps = srcs + _headers() + [os.path.abspath(__file__)]
    if not force and not defines and not _stale(out, deps):
        return out
    tag = "default" if not defines else "v_" + "_".join(d.replace("=", "") for d in defines)
    objdir = os.path.join(ROOT, "_build", tag)
    os.makedirs(objdir, exist_ok=True)
    flags = NVCC_FLAGS + [f"-D{d}" for d in defines] + ["-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        if force or defines or _stale(obj, [src] + _headers() + [os.path.abspath(__file__)]):
            cmd = [cc, *ARCH, *flags, "-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
            if verbose or ptxas_verbose:
                sys.stdout.write(r.stdout + r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = out + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[])
    ap.add_argument("--out", default=LIB)
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, defines=tuple(a.defines), out=a.out, verbose=True,
                ptxas_verbose=a.ptxas_v))


if __name__ == "__main__":
    main()
