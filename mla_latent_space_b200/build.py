"""Builds libmla_b200.so in-tree with nvcc for sm_100a.

    python -m mla_latent_space_b200.build [--force]

The library statically links the CUDA runtime, so at run time it needs only
the driver.  Rebuilds when any source under csrc/ or include/ is newer than
the library.

A second library, libmla_b200_test.so, is built beside it for the tests
only: the same objects plus the SIMT decode kernel, with the C-ABI file
compiled under MLA_TEST_ENTRY_POINTS so that it also exports
mla_decode_fwd_simt.  The product library does not contain that kernel.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmla_b200.so")
TEST_LIB = os.path.join(HERE, "libmla_b200_test.so")
TEST_ONLY = ("decode_simt.cu",)        # compiled into the test library alone
TEST_FLAGGED = ("api.cu",)             # compiled a second time with MLA_TEST_ENTRY_POINTS
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(ROOT, "include", "*.h")) + [os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not (os.path.exists(LIB) and os.path.exists(TEST_LIB)):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(TEST_LIB))
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
                    "-I" + os.path.join(ROOT, "include"), *extra]
    jobs = []   # (source, object, extra flags)
    for src in sources():
        base = os.path.basename(src)
        jobs.append((src, os.path.join(objdir, base + ".o"), []))
        if base in TEST_FLAGGED:
            jobs.append((src, os.path.join(objdir, base + ".test.o"), ["-DMLA_TEST_ENTRY_POINTS"]))
    procs = []
    for src, obj, fl in jobs:
        cmd = [NVCC, *flags, *fl, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out = p.communicate()[0].decode()
        if p.returncode != 0:
            failed.append((src, out))
        elif verbose and out.strip():
            print(out)
    if failed:
        msg = "\n".join(f"--- {s}\n{o}" for s, o in failed)
        raise RuntimeError("nvcc failed:\n" + msg)
    product = [o for s_, o, fl in jobs if not fl and os.path.basename(s_) not in TEST_ONLY]
    test = [o for s_, o, fl in jobs if fl or os.path.basename(s_) not in TEST_FLAGGED]
    for lib, objs in ((LIB, product), (TEST_LIB, test)):
        tmp = lib + ".tmp"
        cmd = [NVCC, *ARCH, "-shared", "--cudart", "static", "-o", tmp, *objs, "-lrt", "-ldl", "-lpthread"]
        subprocess.run(cmd, check=True, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
