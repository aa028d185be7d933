"""Build libtq.so in-tree with nvcc for sm_100a.

Usage: ``python kv_cache_vector_turboquant_b200/build.py [--force] [-j N]`` (run as a
script: importing the package would load the library being built).
Objects go to ``_build/`` at the repository root; the shared library is
written next to this file, and the test hooks' libtq_test.so beside it
(linked against libtq.so, found through $ORIGIN). CUDA runtime is linked
statically so the libraries do not depend on the runtime version that torch
ships.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libtq.so")
TEST_LIB = os.path.join(PKG, "libtq_test.so")

SOURCES = ["tq_host.cpp", "tq_device.cu", "tq_encode.cu", "tq_encode_tc.cu", "tq_decode.cu", "tq_decode_tc.cu", "tq_attend.cu", "tq_attend_fast.cu", "tq_attend_static.cu", "tq_mma_check.cu"]
# test hooks (include/tq_test.h): a separate library, linked against libtq.so,
# that the product path never loads
TEST_SOURCES = ["tq_test_hooks.cpp", "tq_test_umma.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers() -> list[str]:
    out = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    out += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return out


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, jobs: int | None = None, verbose: bool = False) -> str:
    """Compile every source for sm_100a, link libtq.so and libtq_test.so;
    return the path of libtq.so."""
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    headers = _headers()
    objs, test_objs, todo = [], [], []
    for srcs, out in ((SOURCES, objs), (TEST_SOURCES, test_objs)):
        for src in srcs:
            path = os.path.join(CSRC, src)
            obj = os.path.join(BUILD, src + ".o")
            out.append(obj)
            if force or _stale(obj, [path] + headers):
                todo.append((path, obj))

    def compile_one(item):
        path, obj = item
        cmd = [nvcc] + ARCH + FLAGS + ["-c", path, "-o", obj]
        if path.endswith(".cpp"):
            cmd = [nvcc] + FLAGS + ["-x", "c++", "-c", path, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"compile failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose:
            print("built", os.path.basename(obj), file=sys.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=jobs or os.cpu_count() or 4) as ex:
        list(ex.map(compile_one, todo))
    if force or todo or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-Xlinker", "-soname", "-Xlinker", "libtq.so", "-o",
                               tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    if force or todo or _stale(TEST_LIB, test_objs + [LIB]):
        tmp = TEST_LIB + ".tmp"
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + test_objs + [
            "-L" + PKG, "-ltq", "-Xlinker", "-rpath", "-Xlinker", "$ORIGIN"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, TEST_LIB)
    return LIB


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    args = ap.parse_args()
    print(build(force=args.force, jobs=args.j, verbose=True))


if __name__ == "__main__":
    main()
