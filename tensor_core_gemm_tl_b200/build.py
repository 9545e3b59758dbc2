"""Build libtlgemm.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc,
and its checked twin libtlgemm_checked.so (-DTL_CHECKED: the GEMM kernel tests
its index invariants at run time and reports a violation in the device error
word; used by the tests, never by the product path).

    python tensor_core_gemm_tl_b200/build.py [--force] [--verbose-ptxas] [--checked]

(Run as a script: importing the package loads the library it builds.)
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtlgemm.so")
CHECKED_LIB = os.path.join(PKG, "libtlgemm_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.inc"))
                              + glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in inputs())


def build(force: bool = False, ptxas_verbose: bool = False, out: str = LIB, extra=()) -> str:
    if not force and not stale(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_checked(force: bool = False) -> str:
    return build(force=force, out=CHECKED_LIB, extra=("-DTL_CHECKED",))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checked", action="store_true", help="also build libtlgemm_checked.so")
    a = ap.parse_args(argv)
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas))
    if a.checked:
        print(build_checked(force=a.force))


if __name__ == "__main__":
    sys.exit(main())
