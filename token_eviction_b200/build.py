"""Build ``libkvp.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python token_eviction_b200/build.py [--force] [-v]

(Run it as a script: importing the package loads the library this builds.)

The library is plain C ABI over CUDA: every ``csrc/*.cu`` is compiled for
``sm_100a`` and linked into one shared object beside this file, with the CUDA runtime
linked statically. The driver API entry points it needs are fetched at run time.
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkvp.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--use_fast_math", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


# Translation units whose kernels must not spill registers. The tcgen05 kernels issue
# asynchronous TMEM loads (tcgen05.ld) and reads their registers only after
# tcgen05.wait::ld; a spill or a reload of such a register in between would read or
# clobber a register the load is still writing, so any spill there fails the build.
NO_SPILL = ("kvp_score.cu", "kvp_leverage.cu")


def _check_no_spills(src: str, ptxas_log: str) -> None:
    spills = re.findall(r"(\d+) bytes spill stores, (\d+) bytes spill loads", ptxas_log)
    if not spills:
        raise RuntimeError(f"{os.path.basename(src)}: no ptxas resource report to check")
    bad = [(a, b) for a, b in spills if int(a) or int(b)]
    if bad:
        raise RuntimeError(f"{os.path.basename(src)}: register spills {bad}; its kernels must not "
                           f"spill (asynchronous TMEM loads write registers in flight)")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False, out: str | None = None,
          defines: tuple = ()) -> str:
    """Compile and link the library (to `out`, default in-tree; `defines` such as
    "KVP_CHECKS" add -D flags, for a debug build with device-side bounds checks)."""
    target = out or LIB
    if not force and out is None and not defines and not _stale():
        return LIB
    objdir = os.path.join(ROOT, "_build", "dbg" if defines else "rel")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-c", src, "-o", obj]
        checked = os.path.basename(src) in NO_SPILL
        if verbose or checked:
            cmd.insert(1, "-Xptxas=-v")
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode:
            sys.stderr.write(res.stdout + res.stderr)
        if res.returncode:
            raise subprocess.CalledProcessError(res.returncode, cmd)
        if checked:
            _check_no_spills(src, res.stdout + res.stderr)
        objs.append(obj)
    tmp = target + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs])
    os.replace(tmp, target)
    return target


# The debug build: device-side bounds checks that record the first failure instead of
# touching memory out of bounds, and the fault-injection hook the tests use to make a
# bounded wait run out (kvp_debug_set_fault).
CHECKS_LIB = os.path.join(PKG, "libkvp_checks.so")


def build_checks(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(CHECKS_LIB):
        t = os.path.getmtime(CHECKS_LIB)
        deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
        if all(os.path.getmtime(f) <= t for f in deps):
            return CHECKS_LIB
    return build(force=True, verbose=verbose, out=CHECKS_LIB, defines=("KVP_CHECKS",))


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
    if "--checks" in sys.argv:
        print(build_checks(force="--force" in sys.argv, verbose="-v" in sys.argv))
