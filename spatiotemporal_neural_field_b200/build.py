"""Builds the in-tree libraries for sm_100a with nvcc:

* ``libspin4d.so`` from ``csrc/*.cu``: the decoder (``include/spin4d.h``);
* ``libspin4d_checked.so`` from the same sources with ``-DSPIN4D_CHECKED``:
  the decoder with device-side bounds checks (``spin4d_checked_build``);
* ``libspin4d_probe.so`` from ``csrc/probe/*.cu``: the measurement probes
  and the bounded-wait self-test (``include/spin4d_probe.h``).

Usage: ``python -m spatiotemporal_neural_field_b200.build [--force]``.
A library is rebuilt when a source or header is newer than it.
"""
from __future__ import annotations

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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libspin4d.so")
PROBE_LIB = os.path.join(PKG, "libspin4d_probe.so")
CHECKED_LIB = os.path.join(PKG, "libspin4d_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=default",
              "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libspin4d.so")
    return cand


def sources(sub: str = ""):
    return sorted(glob.glob(os.path.join(CSRC, sub, "*.cu")))


def _deps(sub: str = ""):
    return sources(sub) + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = LIB, sub: str = "") -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps(sub))


def _build_one(lib: str, sub: str, verbose: bool, defines=(), obj_sub=None) -> str:
    nvcc = _nvcc()
    obj_sub = sub if obj_sub is None else obj_sub
    obj_dir = os.path.join(BUILD, obj_sub) if obj_sub else BUILD
    os.makedirs(obj_dir, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc] + ARCH + NVCC_FLAGS + ["-D" + d for d in defines] + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources(sub)))
    tmp = lib + ".tmp"
    cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds both libraries (each only when out of date); returns the decoder's path."""
    for lib, sub, defines, obj_sub in ((LIB, "", (), ""), (CHECKED_LIB, "", ("SPIN4D_CHECKED",), "checked"),
                                       (PROBE_LIB, "probe", (), "probe")):
        if force or not up_to_date(lib, sub):
            _build_one(lib, sub, verbose, defines, obj_sub)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
