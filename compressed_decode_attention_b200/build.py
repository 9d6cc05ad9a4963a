"""Build the library in-tree: csrc/*.cu, csrc/*.cpp -> libtq.so (sm_100a).

Usage: python -m compressed_decode_attention_b200.build [--force] [--verbose]
       [--waittest | --debug]
Objects go to _build/ beside this file; the shared library is written next
to this file so it travels with the source tree.

--waittest (build(variant="waittest")) builds libtq_waittest.so, a test-only
build of the same sources with TQ_TEST_INJECT_WAIT_FAULTS: short bounded
waits and two waits made to run out, for the test of the kernels' give-up
path (tests/test_gpu_wait_timeout.py). Only that test loads it.

--debug (build(variant="debug")) builds libtq_debug.so, the bounds-checked
build (TQ_DEBUG): the copy and store index checks of the kernels are live
and report TQ_DEV_DEBUG_CHECK instead of touching memory out of range
(tests/test_gpu_debug_build.py runs it).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libtq.so")
OBJ = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3",
          "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]
CUDA_ONLY = ["--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


VARIANTS = {None: ("libtq.so", "", []),
            "waittest": ("libtq_waittest.so", "waittest", ["-DTQ_TEST_INJECT_WAIT_FAULTS"]),
            "debug": ("libtq_debug.so", "debug", ["-DTQ_DEBUG"])}


def _compile(src, verbose, obj_dir=None, defines=()):
    obj = os.path.join(obj_dir or OBJ, os.path.basename(src) + ".o")
    if not _stale(obj, [src] + _headers()):
        return obj
    cmd = [NVCC] + ARCH + COMMON + list(defines) + \
        (CUDA_ONLY if src.endswith(".cu") else ["-x", "cu"] + CUDA_ONLY) + ["-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, variant=None) -> str:
    name, sub, defines = VARIANTS[variant]
    out = OUT if variant is None else os.path.join(HERE, name)
    obj_dir = os.path.join(OBJ, sub) if sub else OBJ
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    if force:
        for f in glob.glob(os.path.join(obj_dir, "*.o")):
            os.remove(f)
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, obj_dir, defines), srcs))
    if force or _stale(out, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", out] + objs + ["-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                variant="waittest" if "--waittest" in sys.argv else
                "debug" if "--debug" in sys.argv else None))
