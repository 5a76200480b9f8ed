"""Build libcsa.so in-tree from csrc/*.cu with nvcc for sm_100a.

Usage: python -m compressed_sparse_attention_16_b200.build [--force] [-v] [--check]
The shared library links the CUDA runtime statically, so it needs only the
NVIDIA driver at run time.  --check also builds libcsa_check.so, the
CSA_CHECK build (the C API file compiled with -DCSA_CHECK, every other
object shared), which checks every top-k list it writes on the device.
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libcsa.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
          "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    hdr = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hdr += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hdr


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    os.makedirs(OBJDIR, exist_ok=True)
    nvcc = _nvcc()
    hdrs = _deps()
    srcs = sources()
    flags = ARCH + CFLAGS + list(extra_flags or [])
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(OBJDIR, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            jobs.append([nvcc] + flags + ["-c", s, "-o", o])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _stale(LIB, objs):
        run([nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs)
    return LIB


CHECK_LIB = os.path.join(HERE, "libcsa_check.so")


def build_check(force: bool = False, verbose: bool = False) -> str:
    """The CSA_CHECK build: capi.cu with -DCSA_CHECK, linked with the default
    build's other objects (built first if needed)."""
    build(force=force, verbose=verbose)
    nvcc = _nvcc()
    capi = os.path.join(CSRC, "capi.cu")
    obj = os.path.join(OBJDIR, "capi_check.o")
    objs = [os.path.join(OBJDIR, os.path.basename(s)[:-3] + ".o") for s in sources() if s != capi]
    if force or _stale(obj, [capi] + _deps()):
        cmd = [nvcc] + ARCH + CFLAGS + ["-DCSA_CHECK", "-c", capi, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if force or _stale(CHECK_LIB, objs + [obj]):
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", CHECK_LIB] + objs + [obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + r.stdout + r.stderr)
    return CHECK_LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
    if "--check" in sys.argv:
        print(build_check(verbose="-v" in sys.argv))
