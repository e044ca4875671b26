"""Build libvkv.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m kv_cache_attention_chunk_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled to an object in <repo>/_build/ (in parallel),
then linked into kv_cache_attention_chunk_b200/libvkv.so with the CUDA runtime
linked statically, so the library loads on machines without a GPU driver.
The same sources built with VKV_TEST_AIDS defined give libvkv_test.so, the
test build that also exports the test aids of include/vkv_test.h.
"""
from __future__ import annotations

import argparse
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
LIB = os.path.join(PKG, "libvkv.so")
LIB_TEST = os.path.join(PKG, "libvkv_test.so")
TEST_DEFINES = ("VKV_TEST_AIDS",)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-v",
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvkv")
    return cand


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def up_to_date(target: str = LIB) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, verbose: bool, defines=(), tag: str = "") -> tuple[str, str]:
    obj = os.path.join(BUILD, tag + os.path.basename(src).replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = r.stdout + r.stderr
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{log}")
    if verbose:
        print(log)
    return obj, log


def build(force: bool = False, verbose: bool = False, out: str | None = None, defines=()) -> str:
    """Compile every CUDA source for sm_100a and link libvkv.so and its test build
    libvkv_test.so; returns the path of libvkv.so.

    `out` / `defines` build one variant library (extra -D macros) at another path.
    """
    if out is None and not defines:
        _build_one(LIB, (), force, verbose)
        _build_one(LIB_TEST, TEST_DEFINES, force, verbose)
        return LIB
    return _build_one(out or LIB, tuple(defines), True, verbose)


def _build_one(target: str, defines, force: bool, verbose: bool) -> str:
    if not force and up_to_date(target):
        return target
    os.makedirs(BUILD, exist_ok=True)
    tag = "" if target == LIB else os.path.basename(target).replace(".so", "") + "_"
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, defines, tag), _sources()))
    objs = [o for o, _ in results]
    with open(os.path.join(BUILD, tag + "ptxas.log"), "w") as fh:
        for o, log in results:
            fh.write(f"== {os.path.basename(o)}\n{log}\n")
    tmp = target + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-lrt", "-ldl", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
