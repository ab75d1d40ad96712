"""Build the EFLA CUDA library in-tree: ``delta_rule_linear_03_b200/libefla.so``.

Compiles ``csrc/efla_api.cu`` (which includes every kernel header) for
sm_100a only, with the CUDA runtime linked statically so the library needs
nothing but the driver at run time.  Rebuilds when any source under
``csrc/`` or ``include/`` is newer than the library.

    python delta_rule_linear_03_b200/build.py [--force]

(run it as a file: importing the package needs the library to exist)
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libefla.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) +
                 glob.glob(os.path.join(HERE, "csrc", "*.cuh")) +
                 glob.glob(os.path.join(ROOT, "include", "*.h")))
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-Xptxas", "-v"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(s) > t for s in SOURCES)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return SO
    tmp = SO + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-o", tmp, os.path.join(HERE, "csrc", "efla_api.cu")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libefla.so")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
