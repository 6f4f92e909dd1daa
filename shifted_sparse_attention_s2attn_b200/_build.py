"""Builds the CUDA library (csrc/*.cu) for sm_100a into libs2attn.so next to this file.

    python -m shifted_sparse_attention_s2attn_b200._build [--force] [-v] [--debug]

Each .cu is compiled to an object in _build/ (in parallel), then linked with nvcc
into one shared library with the CUDA runtime linked statically.  A source is
rebuilt when it, or any header it may include, is newer than its object.

--debug builds libs2attn_debug.so (objects in _build/debug/) with -DS2ATTN_DEBUG: every
computed global store or reduction index is checked against its tensor's extent, and an
out-of-range access is skipped and recorded in the device error word (site bit 0x80).
Select it with the environment variable S2ATTN_LIBRARY.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libs2attn.so")
DEBUG_LIB = os.path.join(PKG, "libs2attn_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-ffp-contract=off",
         "-I", INCLUDE, "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, obj, verbose, extra=()):
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stderr if verbose else ""


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = DEBUG_LIB if debug else LIB
    extra = ("-DS2ATTN_DEBUG",) if debug else ()
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    jobs = []
    objs = []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src, *headers]):
            jobs.append((src, obj))
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for log in ex.map(lambda a: _compile(*a, verbose, extra), jobs):
            if log:
                print(log, file=sys.stderr)
    if force or jobs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        r = subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
