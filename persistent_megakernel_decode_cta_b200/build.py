"""Builds libamk.so (the C-ABI library: lowering, validator, launcher and the
sm_100a megakernel) in-tree with nvcc.

Every source compiles to its own object file, in parallel (the kernel's
template instances are spread over several amk_kernel_inst_*.cu files for
that reason), and the objects link into one shared library."""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libamk.so")
OBJ = os.path.join(ROOT, "_build", "amk")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) +
                  glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def _newer(deps, t) -> bool:
    return any(os.path.getmtime(d) > t for d in deps)


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    return _newer(sources() + _headers(), os.path.getmtime(out))


def _obj_for(src: str) -> str:
    return os.path.join(OBJ, os.path.basename(src) + ".o")


def _compile(nvcc: str, src: str, force: bool, verbose: bool) -> str:
    obj = _obj_for(src)
    if not force and os.path.exists(obj) and \
            not _newer([src] + _headers(), os.path.getmtime(obj)):
        return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA/C++ source into persistent_megakernel_decode_cta_b200/libamk.so."""
    if not force and not _stale(LIB):
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ, exist_ok=True)
    srcs = sources()
    workers = max(1, min(len(srcs), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        objs = list(ex.map(lambda s: _compile(nvcc, s, force, verbose), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                    *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
