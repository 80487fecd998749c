"""Build libkda.so in-tree with nvcc for sm_100a (B200).

    python -m gated_delta_rule_158_b200.build [--force]

Compiles every csrc/*.cu into one shared library next to this file, and the
same sources with -DKDA_DEBUG_CHECKS (device-side bounds checks that record
KDA_ERR_BOUNDS in the status word) into libkda_debug.so beside it.  nvcc
cross-compiles without a GPU; the CUDA runtime is linked statically and the
driver API entry points (tensor-map encoding) are resolved at run time, so
the libraries need only libcuda from the driver.  Translation units compile
in parallel.
"""
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libkda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


VARIANTS = {  # library -> (object directory, extra flags)
    "release": (LIB, BUILD_DIR, []),
    "debug": (os.path.join(HERE, "libkda_debug.so"), os.path.join(BUILD_DIR, "debug"),
              ["-DKDA_DEBUG_CHECKS"]),
}


def _build_variant(lib, obj_dir, extra, force, verbose, pool):
    os.makedirs(obj_dir, exist_ok=True)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    objs, jobs = [], []
    for src in _sources():
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers + [os.path.abspath(__file__)]):
            cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append(pool.submit(subprocess.run, cmd, check=True))
    for j in jobs:
        j.result()  # raises CalledProcessError on a failed compile
    if force or _stale(lib, objs + [CSRC]):  # the directory's mtime: a source removed
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs,
               "-Xcompiler", "-fvisibility=hidden"]
        subprocess.run(cmd, check=True)
    return lib


def build(force: bool = False, verbose: bool = False, variants=("release", "debug")) -> str:
    """Builds the listed variants; returns the release library's path."""
    with ThreadPoolExecutor(max_workers=max(2, min(16, os.cpu_count() or 2))) as pool:
        for name in variants:
            lib, obj_dir, extra = VARIANTS[name]
            _build_variant(lib, obj_dir, extra, force, verbose, pool)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
