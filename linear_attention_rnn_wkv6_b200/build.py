"""Build libwkv.so (and its test variant) in-tree with nvcc for sm_100a (B200).

    python -m linear_attention_rnn_wkv6_b200.build [--force] [--verbose] [--variant NAME]

Variants (each a complete library with the same C ABI, include/wkv.h):
  default     libwkv.so            -- the product: every entry point runs its one
                                      fixed algorithm (the chunked tensor-core forms
                                      where they exist)
  recurrence  libwkv_recurrence.so -- built with -DWKV_RECURRENCE_PATHS: the entry
                                      points that have a chunked tensor-core form run
                                      the token-by-token recurrence kernels instead;
                                      for testing those kernels and timing the chunked
                                      forms against them
  debug       libwkv_debug.so      -- built with -DWKV_DEVICE_CHECKS=1: the product
                                      with an index check on every global store of
                                      every kernel, and entry points that wait for
                                      their kernels and report a failed check

The libraries are written next to this file so that they travel with the source
tree; the Python binding loads them from there.  Each .cu file is compiled to an
object of its own (in parallel, under _build/), then the objects are device-linked
into the shared library.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
VARIANTS = {
    "default": ("libwkv.so", []),
    "recurrence": ("libwkv_recurrence.so", ["-DWKV_RECURRENCE_PATHS=1"]),
    "debug": ("libwkv_debug.so", ["-DWKV_DEVICE_CHECKS=1"]),
}
LIB = os.path.join(HERE, VARIANTS["default"][0])


def lib_file(variant: str = "default") -> str:
    return os.path.join(HERE, VARIANTS[variant][0])


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(p) > t for p in _deps())


def _run(cmd: list[str], verbose: bool) -> None:
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)


def _build_variant(variant: str, verbose: bool) -> str:
    out = lib_file(variant)
    flags = VARIANTS[variant][1]
    nvcc = nvcc_path()
    objdir = os.path.join(OBJDIR, variant)
    os.makedirs(objdir, exist_ok=True)
    common = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-Xcompiler", "-fPIC", "-I", INCLUDE,
              *flags]
    if verbose:
        common.insert(1, "-Xptxas=-v")
    objs = []
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        jobs.append(common + ["-c", src, "-o", obj])
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        list(ex.map(lambda c: _run(c, verbose), jobs))
    _run([nvcc, *ARCH, "-rdc=true", "-shared", "-Xcompiler", "-fPIC", "-o", out + ".tmp", *objs, "-lcudart"], verbose)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False, verbose: bool = False, variants=("default", "recurrence", "debug")) -> str:
    """Build the requested variants (all by default) if their sources changed.
    Returns the path of the default library."""
    todo = [v for v in variants if force or _stale(lib_file(v))]
    if todo:
        with ThreadPoolExecutor(max_workers=len(todo)) as ex:
            list(ex.map(lambda v: _build_variant(v, verbose), todo))
    return LIB


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--variant", action="append", choices=sorted(VARIANTS))
    a = ap.parse_args()
    variants = a.variant or ["default", "recurrence", "debug"]
    build(force=a.force, verbose=a.verbose, variants=variants)
    for v in variants:
        print(lib_file(v))


if __name__ == "__main__":
    main()
