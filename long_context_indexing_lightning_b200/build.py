"""Build ``libdsa.so`` in-tree with nvcc for sm_100a (B200).

Usage: ``python -m long_context_indexing_lightning_b200.build [--force]``.
Each CUDA source is compiled to an object in ``_build/`` (in parallel, only
when it or a header changed), then the objects are linked into the shared
library, which lands next to this file so it travels with the source tree.
"""
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libdsa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(INCLUDE, "dsa.h")]


def _obj(src):
    return os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in deps)


def up_to_date() -> bool:
    return not _stale(LIB, _sources() + _headers())


def _nvcc():
    nvcc = os.environ.get("NVCC", "nvcc")
    if nvcc == "nvcc":
        from shutil import which
        if which("nvcc") is None and os.path.exists("/usr/local/cuda/bin/nvcc"):
            nvcc = "/usr/local/cuda/bin/nvcc"
    return nvcc


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = _nvcc()
    os.makedirs(OBJDIR, exist_ok=True)
    headers = _headers()
    todo = [s for s in _sources() if force or _stale(_obj(s), [s] + headers)]

    def compile_one(src):
        tmp = _obj(src) + ".tmp"
        cmd = [nvcc, *NVCC_FLAGS, "-I" + INCLUDE, "-I" + CSRC, "-c", src, "-o", tmp]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        os.replace(tmp, _obj(src))

    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 1))) as ex:
        list(ex.map(compile_one, todo))
    tmp = LIB + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
           *[_obj(s) for s in _sources()], "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
