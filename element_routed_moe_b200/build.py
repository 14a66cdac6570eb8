"""Build libjanus.so (the C-ABI CUDA library) in-tree for sm_100a.

Each ``csrc/*.cu`` is compiled by nvcc to an object (in parallel), then
linked into ``element_routed_moe_b200/libjanus.so``.  ``-Xptxas -v`` output
(registers, spills, shared memory per kernel) is kept in
``_build/ptxas.txt`` for inspection.

``build(debug=True)`` (``--debug``) builds the same sources with
``-DJANUS_DEBUG`` into ``libjanus_debug.so``: every kernel then checks the
index arrays it is given before using them and records a data fault instead
of an out-of-range access (see janus_debug_check in include/janus.h).
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
LIB = os.path.join(PKG, "libjanus.so")
DEBUG_LIB = os.path.join(PKG, "libjanus_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(INCLUDE, "janus.h"), os.path.abspath(__file__)]


def _stale(lib) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def _compile(src, out_dir, extra):
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    r = subprocess.run([NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj],
                       capture_output=True, text=True)
    return src, obj, r


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    extra = ["-DJANUS_DEBUG"] if debug else []
    os.makedirs(out_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda src: _compile(src, out_dir, extra), _sources()))
    log = []
    for src, obj, r in results:
        log.append(f"==== {os.path.basename(src)}\n{r.stdout}{r.stderr}")
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {src}")
    with open(os.path.join(out_dir, "ptxas.txt"), "w") as f:
        f.write("\n".join(log))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *[o for _, o, _ in results]])
    os.replace(tmp, lib)
    if verbose:
        print("\n".join(log))
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
