"""Builds libtern.so (sm_100a) in-tree with nvcc.

    python -m ternary_weight_only_tern_b200.build [--force] [--verbose] [--debug]

--debug builds libtern_debug.so instead: the same sources with TERN_DEBUG defined, so the decode
kernels check their memory indices before each access and report a failed check through
tern_device_status (TERN_ERR_BOUNDS) instead of faulting; select it with TERN_LIBRARY=debug.

Every CUDA source is compiled for sm_100a only (-gencode arch=compute_100a,code=sm_100a)
with line info; the CUDA runtime is linked statically so the library shares the device's
primary context with whatever else the process uses (PyTorch included).
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libtern.so")
LIB_DEBUG = os.path.join(PKG, "libtern_debug.so")
SOURCES = ["tern_api.cu", "tern_pack.cu", "tern_elem.cu", "tern_gemv.cu", "tern_decode1.cu", "tern_decodem.cu", "tern_gemm_sm100.cu",
           "tern_rotate.cu", "tern_fit.cu", "tern_bits.cpp"]
HEADERS = ["tern_internal.cuh", "tern_device.cuh", "tern_stream.cuh", os.path.join("..", "..", "include", "tern.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _flags(extra_ptxas_v: bool, debug: bool = False) -> list[str]:
    f = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]
    if debug:
        f += ["-DTERN_DEBUG=1"]
    if extra_ptxas_v:
        f += ["-Xptxas", "-v"]
    return f


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS]
    objs, jobs = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(bdir, src + ".o")
        objs.append(obj)
        if force or _stale(obj, [path] + hdrs + [__file__]):
            cmd = [nvcc()] + ARCH + _flags(verbose, debug) + ["-c", path, "-o", obj]
            if src.endswith(".cpp"):
                cmd = [shutil.which("g++") or "g++", "-O2", "-std=c++17", "-fPIC",
                       "-I" + os.path.join(ROOT, "include"), "-c", path, "-o", obj]
                if debug:
                    cmd.insert(-4, "-DTERN_DEBUG=1")
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or r.returncode:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError(f"nvcc failed on {cmd[-3]}")
    if force or jobs or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs + ["-lpthread", "-ldl", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print nvcc output including -Xptxas -v")
    ap.add_argument("--debug", action="store_true", help="build libtern_debug.so (TERN_DEBUG bounds checks)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))


if __name__ == "__main__":
    main()
