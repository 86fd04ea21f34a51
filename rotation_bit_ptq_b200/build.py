"""Build librbq.so in-tree with nvcc for sm_100a.

Run ``python -m rotation_bit_ptq_b200.build`` (or call ``build()``).  Each
CUDA source compiles to an object under ``_build/`` (in parallel, rebuilt
when it or a header is newer than its object), then one shared library is
linked next to this file.  The CUDA runtime is linked statically.
"""

import concurrent.futures
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
LIB = os.path.join(PKG, "librbq.so")
# The same sources compiled with RBQ_DEBUG: device-side bounds checks on the
# indices the kernels compute (see dbg_index in csrc/rbq_sm100.cuh) record
# into the device error word instead of trapping.  Tests load it beside the
# release library; the product path never does.
LIB_DEBUG = os.path.join(PKG, "librbq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj, src, newest_header):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return os.path.getmtime(src) > t or newest_header > t


def build(verbose=False, ptxas_info=False, jobs=None, debug=False):
    """Compile every CUDA source for sm_100a and link librbq.so (or, with
    debug=True, librbq_debug.so with -DRBQ_DEBUG, objects under _build/debug)."""
    bdir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(bdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DRBQ_DEBUG"] if debug else [])
    cmds = []
    objs = []
    for src in srcs:
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        objs.append(obj)
        if ptxas_info or _stale(obj, src, newest_header):
            cmds.append([nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with concurrent.futures.ThreadPoolExecutor(max_workers=jobs or os.cpu_count()) as ex:
        for cmd, r in ex.map(run, cmds):
            if verbose or ptxas_info or r.returncode:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError(f"nvcc failed on {cmd[-3]}")
    if cmds or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        link = [nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-lcudart_static", "-lrt", "-lpthread", "-ldl"]
        r = subprocess.run(link, capture_output=True, text=True)
        if verbose or r.returncode:
            sys.stderr.write(" ".join(link) + "\n" + r.stdout + r.stderr)
        if r.returncode:
            raise RuntimeError(f"link of {os.path.basename(lib)} failed")
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv, debug="--debug" in sys.argv))
