"""Build libkvq.so (CUDA for sm_100a) in-tree with nvcc.

Usage: python -m asymmetric_kv_cache_b200.build [--verbose-ptxas]

Objects go to _build/ at the repository root; the shared library is written
next to this file, where the Python binding loads it from.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libkvq.so")
# the same library with the decode kernels' range checks compiled in
# (-DKVQ_DEBUG): every cache, workspace, query and output index is checked
# before its access and a failure is recorded in the workspace error word
DEBUG_LIB = os.path.join(HERE, "libkvq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
          "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cpp")))


def _compile(src: str, verbose_ptxas: bool, debug: bool = False) -> tuple[str, str]:
    obj = os.path.join(BUILD, os.path.basename(src) + (".debug.o" if debug else ".o"))
    cmd = [_nvcc(), *ARCH, *COMMON, *(["-DKVQ_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if verbose_ptxas and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stdout}\n{res.stderr}")
    return obj, res.stderr


def _up_to_date(srcs) -> bool:
    if not os.path.exists(LIB) or not os.path.exists(DEBUG_LIB):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(DEBUG_LIB))
    deps = list(srcs) + [os.path.join(INCLUDE, "kvq.h"), __file__]
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return all(os.path.getmtime(d) <= t for d in deps)


def _link(objs, out: str) -> None:
    tmp = out + ".tmp"
    cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, out)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile every CUDA/C++ source of the library and link libkvq.so and
    its range-checked twin libkvq_debug.so."""
    srcs = _sources()
    if not force and not verbose_ptxas and _up_to_date(srcs):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    jobs = [(s, False) for s in srcs] + [(s, True) for s in srcs]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda j: _compile(j[0], verbose_ptxas and not j[1], j[1]), jobs))
    if verbose_ptxas:
        with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
            for (_, dbg), (_, log) in zip(jobs, results):
                if not dbg:
                    f.write(log)
    _link([o for (_, dbg), (o, _) in zip(jobs, results) if not dbg], LIB)
    _link([o for (_, dbg), (o, _) in zip(jobs, results) if dbg], DEBUG_LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true",
                    help="write per-kernel register/shared-memory use to _build/ptxas.log")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas))
    return 0


if __name__ == "__main__":
    sys.exit(main())
