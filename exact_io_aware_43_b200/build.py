"""Build libfattn.so in-tree for sm_100a (B200) with nvcc.

    python -m exact_io_aware_43_b200.build [--force]

The library is one translation unit (csrc/fattn.cu, which includes the kernels) compiled with
``-gencode arch=compute_100a,code=sm_100a`` and the CUDA runtime linked statically, so the built
file only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB_DIR = os.path.join(HERE, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libfattn.so")
# Test-only variant: the forward's producer leaves one K/V tile unissued, and the d = 256
# backward's one dO tile (FA_TEST_STARVE); the waits are bounded at 1 ms and the pair kernel's
# teardown hand-back wait at 20 ms, so a test can watch a bounded wait run out and the kernel
# report FA_ERR_TIMEOUT without any fault or hang.  The product path never loads it.
STARVE_PATH = os.path.join(LIB_DIR, "libfattn_starve.so")
STARVE_DEFINES = ["-DFA_TEST_STARVE", "-DFA_DEFAULT_WAIT_LIMIT_NS=1000000ull",
                  "-DFA_PAIR_HANDBACK_LIMIT_NS=20000000ull"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(s) <= t for s in sources())


def _compile(out: str, defines, verbose: bool) -> None:
    tmp = out + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *defines, "-o", tmp, os.path.join(CSRC, "fattn.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        print(r.stdout + r.stderr)
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False, starve: bool = True) -> str:
    """Build libfattn.so (and, unless starve=False, the test-only libfattn_starve.so)."""
    os.makedirs(LIB_DIR, exist_ok=True)
    if force or not up_to_date(LIB_PATH):
        _compile(LIB_PATH, [], verbose)
    if starve and (force or not up_to_date(STARVE_PATH)):
        _compile(STARVE_PATH, STARVE_DEFINES, False)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                starve="--no-starve" not in sys.argv))
