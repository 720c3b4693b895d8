"""Build libq4g.so (the CUDA library behind include/q4g.h) in-tree for sm_100a,
and the device fills of the seeded generators (datagen/libq4g_datagen.so).

    python -m int4_q4_gemv_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libq4g.so")
DG_SRC = os.path.join(ROOT, "datagen", "q4g_datagen_fill.cu")
DG_LIB = os.path.join(ROOT, "datagen", "libq4g_datagen.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]
# the library's objects are compiled with ptxas's resource report, kept per source file
# beside the object (registers, stack frame, spills of every kernel: kernel_resources())
RES_FLAGS = ["-Xptxas", "-v"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                     [os.path.join(ROOT, "include", "q4g.h")])
    nvcc = _nvcc()
    objs = []
    jobs = []
    for s in srcs:
        o = os.path.join(BUILD_DIR, os.path.basename(s) + ".o")
        objs.append(o)
        if force or _stale(o, [s] + headers) or not os.path.exists(o + ".resources.txt"):
            jobs.append((o, [nvcc, *ARCH, *FLAGS, *RES_FLAGS, "-c", s, "-o", o]))

    def compile_one(job):
        o, cmd = job
        log = _run(cmd, verbose)
        with open(o + ".resources.txt", "w") as f:
            f.write(log)

    with ThreadPoolExecutor(max_workers=min(8, len(jobs) or 1)) as ex:
        list(ex.map(compile_one, jobs))
    if force or jobs or _stale(LIB, objs):
        _run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB + ".tmp", *objs], verbose)
        os.replace(LIB + ".tmp", LIB)
    dg_deps = [DG_SRC, os.path.join(ROOT, "datagen", "q4g_datagen.h")]
    if force or _stale(DG_LIB, dg_deps):
        _run([nvcc, *ARCH, *FLAGS, "-shared", "-cudart", "static", "-o", DG_LIB + ".tmp", DG_SRC], verbose)
        os.replace(DG_LIB + ".tmp", DG_LIB)
    return LIB


def kernel_resources() -> dict:
    """Per kernel of libq4g.so, from the ptxas reports of the last build: demangled
    name -> {"registers", "stack", "spill_stores", "spill_loads"} (bytes, per thread)."""
    import re
    text = ""
    for f in sorted(glob.glob(os.path.join(BUILD_DIR, "*.o.resources.txt"))):
        with open(f) as fh:
            text += fh.read()
    out, cur = {}, None
    for line in text.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            cur = m.group(1)
            out[cur] = {}
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and cur is not None:
            out[cur].update(stack=int(m.group(1)), spill_stores=int(m.group(2)), spill_loads=int(m.group(3)))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and cur is not None:
            out[cur]["registers"] = int(m.group(1))
            cur = None
    names = list(out)
    try:  # demangle in one call
        r = subprocess.run(["c++filt"], input="\n".join(names), capture_output=True, text=True, check=True)
        pretty = r.stdout.splitlines()
    except (OSError, subprocess.CalledProcessError):
        pretty = names
    return {p: out[n] for n, p in zip(names, pretty) if len(pretty) == len(names)} or out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
