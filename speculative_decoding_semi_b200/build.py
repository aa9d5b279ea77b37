"""Build libdspark.so in-tree with nvcc for sm_100a (B200).

Usage: python speculative_decoding_semi_b200/build.py [--verbose] [--ptxas]
Each .cu under csrc/ is compiled in parallel to an object file under _build/,
then linked into speculative_decoding_semi_b200/libdspark.so with the CUDA
runtime linked statically (the library then needs only the driver at run time).
The L2 read probe under probe/ (not part of the library's path; the benchmark
loads it for its L2 denominator) becomes libdspark_probe.so the same way.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libdspark.so")
PROBE_SRC = os.path.join(HERE, "probe", "l2_read.cu")
PROBE_LIB = os.path.join(HERE, "libdspark_probe.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdspark")
    return path


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _needs_rebuild(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(ROOT, "include", "dspark.h"))
    objs, jobs = [], []
    for src in sources():
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if _needs_rebuild(obj, [src] + headers):
            cmd = [nvcc(), *ARCH, *FLAGS, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + p.stdout + p.stderr)
        return p.stdout + p.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for out in ex.map(run, jobs):
            if verbose and out.strip():
                print(out)
    if jobs or _needs_rebuild(LIB, objs):
        run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs])
    if _needs_rebuild(PROBE_LIB, [PROBE_SRC]):
        run([nvcc(), *ARCH, *FLAGS, "-shared", "-cudart", "static", "-o", PROBE_LIB, PROBE_SRC])
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, ptxas_verbose="--ptxas" in sys.argv))
