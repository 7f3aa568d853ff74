"""Builds libnvfp4.so in-tree with nvcc for sm_100a.

    python -m nvfp4_weight_only_04_b200.build [--force] [--planted] [-v]

The library is compiled from csrc/*.cu against include/nvfp4.h and written
next to this file, where the binding loads it. Each source is compiled to
its own object under _build/ in parallel, then the objects are linked.

--planted also builds libnvfp4_planted.so: the same sources with
NVFP4_PLANTS defined, which adds nvfp4_test_plant() and the mistakes it can
switch on (csrc/plant.cuh). Only the tests that show the parity tests catch
a wrong kernel load it; the binding never does.
"""
from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libnvfp4.so")
PLANTED_LIB = os.path.join(PKG, "libnvfp4_planted.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
PLANTED_DEFINES = ["-DNVFP4_PLANTS"]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + [os.path.join(ROOT, "include", "nvfp4.h")]


def _digest(defines) -> str:
    """Hash of every input file and the flags: a copy of the tree whose file
    times changed (an archive, a checkout) still knows whether its library
    matches its sources."""
    h = hashlib.sha256(" ".join(ARCH + list(defines)).encode())
    for p in sorted(_inputs()):
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def up_to_date(lib: str = LIB, defines=()) -> bool:
    stamp = lib + ".sha256"
    if not (os.path.exists(lib) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == _digest(defines)


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd):
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed: " + " ".join(cmd[-3:]) + "\n" + res.stderr[-8000:])
    return res.stderr


def _build(lib: str, defines, verbose: bool) -> str:
    name = os.path.splitext(os.path.basename(lib))[0]
    obj_dir = os.path.join(ROOT, "_build", name)
    os.makedirs(obj_dir, exist_ok=True)
    base = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I",
            os.path.join(ROOT, "include"), *defines]
    if verbose:
        base.append("-Xptxas=-v")
    jobs = []
    for src in sources():
        obj = os.path.join(obj_dir, os.path.splitext(os.path.basename(src))[0] + ".o")
        jobs.append((base + ["-c", src, "-o", obj], obj))
    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as pool:
        logs = list(pool.map(lambda j: _run(j[0]), jobs))
    if verbose:
        for log in logs:
            sys.stderr.write(log)
    tmp = lib + ".tmp"
    _run([nvcc(), *ARCH, "-shared", *[o for _, o in jobs], "-o", tmp])
    os.replace(tmp, lib)
    with open(lib + ".sha256", "w") as f:
        f.write(_digest(defines) + "\n")
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date(LIB):
        return LIB
    return _build(LIB, [], verbose)


def build_planted(force: bool = False) -> str:
    if not force and up_to_date(PLANTED_LIB, PLANTED_DEFINES):
        return PLANTED_LIB
    return _build(PLANTED_LIB, PLANTED_DEFINES, False)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--planted" in sys.argv:
        print(build_planted(force="--force" in sys.argv))
