"""Build libtpconv.so (sm_100a) in-tree.

Steps: compile and run the CG table emitter (host C++), compile every CUDA
translation unit for sm_100a (large template files are compiled several times,
one instantiation set each, in parallel), link one shared library next to this
file. Objects go to <repo>/_build; a unit is rebuilt only when a source or
header is newer than its object.
"""
from __future__ import annotations

import concurrent.futures
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
LIB = os.path.join(PKG, "libtpconv.so")
CG_LMAX = 6

# translation units and how many instantiation sets each one is split into
UNITS = {
    "uvu_fwd.cu": 10,
    "uvu_bwd.cu": 10,
    "uvw.cu": 10,
    "uvu_dbwd.cu": 10,
    "uvu_state.cu": 2,
    "gemm.cu": 1,
    "tc_gemm.cu": 1,
    "csr.cu": 1,
    "api.cu": 1,
    "noalloc.cu": 1,
    "plan.cpp": 1,
    "cg_host.cpp": 1,
}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"command failed ({r.returncode}): {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def _includes(path, found):
    """Local headers a source includes, directly or through other headers."""
    import re
    try:
        text = open(path).read()
    except OSError:
        return found
    for name in re.findall(r'^\s*#\s*include\s+"([^"]+)"', text, re.M):
        for d in (CSRC, INCLUDE, BUILD):
            cand = os.path.join(d, name)
            if os.path.exists(cand) and cand not in found:
                found.add(cand)
                _includes(cand, found)
                break
    return found


def build(jobs: int | None = None, verbose: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    # 1. compile-time CG table
    gen = os.path.join(BUILD, "cg_gen")
    table = os.path.join(BUILD, "cg_table.inc")
    gen_src = [os.path.join(CSRC, "cg_gen.cpp"), os.path.join(CSRC, "cg_host.cpp"),
               os.path.join(CSRC, "cg_host.h")]
    if force or not os.path.exists(table) or os.path.getmtime(table) < _newest(gen_src):
        _run(["g++", "-O2", "-std=c++17", "-o", gen, gen_src[0], gen_src[1]], verbose)
        _run([gen, str(CG_LMAX), table], verbose)
    # 2. objects
    nvcc = _nvcc()
    jobs_list = []
    for unit, nset in UNITS.items():
        src = os.path.join(CSRC, unit)
        stem = os.path.splitext(unit)[0]
        deps_time = _newest([src] + sorted(_includes(src, set())))
        for k in range(nset):
            obj = os.path.join(BUILD, f"{stem}_{k}.o" if nset > 1 else f"{stem}.o")
            cmd = [nvcc, "-std=c++17", "-O3", "-lineinfo", *ARCH, "-Xcompiler", "-fPIC",
                   "-I", CSRC, "-I", INCLUDE, "-I", BUILD, "-x", "cu", "-c", src, "-o", obj]
            if nset > 1:
                cmd.insert(1, f"-DTPC_SET={k}")
            stale = (force or not os.path.exists(obj)
                     or os.path.getmtime(obj) < max(deps_time, os.path.getmtime(src)))
            jobs_list.append((obj, cmd, stale))
    todo = [(o, c) for o, c, s in jobs_list if s]
    if todo:
        n = jobs or max(1, min(len(todo), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(n) as ex:
            futs = [ex.submit(_run, c, verbose) for _, c in todo]
            for f in futs:
                f.result()
    objs = [o for o, _, _ in jobs_list]
    # 3. link (static CUDA runtime: no dependency on a libcudart search path)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < _newest(objs):
        tmp = LIB + ".tmp"
        _run([nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-Xcompiler", "-fPIC"], verbose)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
