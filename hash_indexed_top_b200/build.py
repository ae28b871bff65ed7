"""Build ``libdashkv.so`` in-tree with nvcc for sm_100a (B200).

The library is relocatable device code in several translation units compiled
in parallel: ``csrc/dashkv.cu`` (host side and every kernel but the step
kernel) and ``csrc/step_inst.cu`` once per (bits, head dim) pair, each holding
that pair's instantiations of the clustered step kernel; nvcc then links the
objects, device code included, into one shared library.
"""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdashkv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-rdc=true"]
STEP_PAIRS = [(b, d) for b in (32, 64, 128) for d in (64, 128)]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "dashkv.h")])


def _units() -> list[tuple[str, list[str]]]:
    """(object file, nvcc arguments) of every translation unit."""
    units = [(os.path.join(OBJ, "dashkv.o"), [os.path.join(CSRC, "dashkv.cu")])]
    for b, d in STEP_PAIRS:
        units.append((os.path.join(OBJ, f"step_{b}_{d}.o"),
                      [f"-DSTEP_BITS={b}", f"-DSTEP_D={d}", os.path.join(CSRC, "step_inst.cu")]))
    return units


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the translation units (in parallel) and link libdashkv.so."""
    newest = max(os.path.getmtime(s) for s in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    procs = []
    for obj, args in _units():
        cmd = [_nvcc(), *NVCC_FLAGS, "-c", "-o", obj, *args]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((cmd, subprocess.Popen(cmd)))
    failed = [cmd for cmd, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-rdc=true", "-o", tmp,
                           *[obj for obj, _ in _units()]])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
