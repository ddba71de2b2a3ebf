"""Build libsala.so (the product kernels + C ABI), libsala_debug.so (the same with the
SALA_DEBUG_BOUNDS index checks) and libsala_selftest.so (tensor-core layout self-test used by the
tests) in-tree, for sm_100a only.

    python -m hybrid_sparse_linear_b200.build [--force] [-j N]

Each ``csrc/*.cu`` is compiled separately with nvcc (``-gencode arch=compute_100a,code=sm_100a
-lineinfo -O3``) into ``_build/`` and linked against the shared CUDA runtime, so the library
shares the runtime (current device, streams) with PyTorch in the same process.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libsala.so")
DEBUG_LIB = os.path.join(HERE, "libsala_debug.so")   # the same kernels with -DSALA_DEBUG_BOUNDS
SELFTEST_LIB = os.path.join(HERE, "libsala_selftest.so")
SELFTEST_SRC = {"selftest_mma.cu"}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills", f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, force: bool, extra=(), tag: str = "") -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + tag + ".o")
    if force or _stale(obj, [src] + _headers()):
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if r.stderr.strip():
            sys.stderr.write(r.stderr)
    return obj


def _link(objs, out: str, force: bool):
    if force or _stale(out, objs):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "shared", *objs, "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed for {out}:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)


def build(force: bool = False, jobs: int | None = None, verbose_ptxas: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    lib_srcs = [s for s in srcs if os.path.basename(s) not in SELFTEST_SRC]
    with cf.ThreadPoolExecutor(max_workers=jobs or os.cpu_count() or 4) as ex:
        futs = {s: ex.submit(_compile, s, force, extra) for s in srcs}
        dfuts = {s: ex.submit(_compile, s, force, [*extra, "-DSALA_DEBUG_BOUNDS"], ".dbg")
                 for s in lib_srcs}
        objs = {os.path.basename(s): f.result() for s, f in futs.items()}
        dobjs = [f.result() for f in dfuts.values()]
    _link([o for n, o in objs.items() if n not in SELFTEST_SRC], LIB, force)
    _link([o for n, o in objs.items() if n in SELFTEST_SRC], SELFTEST_LIB, force)
    _link(dobjs, DEBUG_LIB, force)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(a.force, a.j, a.ptxas_v))
