"""Build libkvc.so in-tree for sm_100a (nvcc cross-compiles without a GPU)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libkvc.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
SOURCES = ["api.cpp", "container.cu", "lossless.cu", "transform.cu"]
HEADERS = ["kvc_device.cuh", "kvc_internal.h", "tcgen05.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--fmad=false",                 # no fused multiply-add unless written explicitly
    "-Xcompiler", "-fPIC,-O2,-ffp-contract=off",
    "-I", INCLUDE,
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


# Test builds of the same sources with one compile-time setting changed; each
# links to libkvc_<name>.so beside libkvc.so. "wait0": the tensor stage's wait
# for its own MMAs gives up without polling, so the timeout status can be tested.
VARIANTS = {"wait0": ["-DKVC_MMA_WAIT_POLLS=0u"]}


def variant_path(name: str) -> str:
    return os.path.join(HERE, f"libkvc_{name}.so")


def build(verbose: bool = False, extra: list[str] | None = None, variant: str | None = None) -> str:
    bdir = BUILD if variant is None else os.path.join(BUILD, variant)
    lib = LIB if variant is None else variant_path(variant)
    extra = list(extra or []) + (VARIANTS[variant] if variant else [])
    os.makedirs(bdir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "kvc.h")]
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(bdir, src + ".o")
        objs.append(obj)
        if _stale(obj, [path] + headers + [__file__]):
            cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-c", path, "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.check_call(cmd)
    if _stale(lib, objs):
        cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs,
               "-Xcompiler", "-fPIC", "-lpthread"]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
    return lib


def build_all(verbose: bool = False) -> None:
    build(verbose)
    for name in VARIANTS:
        build(verbose, variant=name)


if __name__ == "__main__":
    if sys.argv[1:] == ["all"]:
        build_all(verbose=True)
    else:
        build(verbose=True, extra=sys.argv[1:])
    print(LIB)
