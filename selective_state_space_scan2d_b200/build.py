"""Build the CUDA library in-tree: libscan2d_b200.so next to this file (sm_100a only).

    python -m selective_state_space_scan2d_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libscan2d_b200.so")
OBJDIR = os.path.join(HERE, "_build")
HEADER = os.path.join(ROOT, "include", "scan2d.h")
# each translation unit with the files it includes; they compile in parallel
UNITS = {
    os.path.join(HERE, "csrc", "scan2d.cu"): [os.path.join(HERE, "csrc", "scan2d_kernels.cuh"), HEADER],
    os.path.join(HERE, "csrc", "scan2d_bwd.cu"): [HEADER],
    os.path.join(HERE, "csrc", "scan2d_grid.cu"): [HEADER],
    os.path.join(HERE, "csrc", "scan2d_proj.cu"): [HEADER],
}
SOURCES = list(UNITS)
DEPS = SOURCES + sorted({d for deps in UNITS.values() for d in deps})
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _obj(src: str) -> str:
    return os.path.join(OBJDIR, os.path.splitext(os.path.basename(src))[0] + ".o")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in DEPS):
            return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2"]
    if verbose:
        flags.insert(0, "-Xptxas=-v")
    procs = []
    for src, deps in UNITS.items():
        obj = _obj(src)
        fresh = (not force and os.path.exists(obj) and
                 all(os.path.getmtime(d) <= os.path.getmtime(obj) for d in [src, *deps]))
        if fresh:
            continue
        tmp = obj + f".tmp{os.getpid()}"
        procs.append((obj, tmp, subprocess.Popen([nvcc(), *flags, "-c", "-o", tmp, src],
                                                 stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                                 text=True)))
    failed = []
    for obj, tmp, proc in procs:
        out, _ = proc.communicate()
        if proc.returncode != 0:
            failed.append(out)
        else:
            if verbose:
                sys.stderr.write(out)
            os.replace(tmp, obj)
    if failed:
        raise RuntimeError("nvcc failed:\n" + "\n".join(failed))
    tmp = LIB + f".tmp{os.getpid()}"
    res = subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *(_obj(s) for s in SOURCES)],
                         capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
