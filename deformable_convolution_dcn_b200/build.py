"""Build step of libdcn_b200.so: nvcc for sm_100a, in-tree.

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel,
rebuilt only when a source or header is newer), then linked into
``deformable_convolution_dcn_b200/libdcn_b200.so`` with the CUDA runtime linked
statically, so the library does not depend on which libcudart a host process
has already loaded.

    python -m deformable_convolution_dcn_b200.build [--force] [-v] [--nvtx]
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdcn_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                 "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src: str, force: bool, verbose: bool, extra=(), build_dir=BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC, *CFLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed on %s:\n%s%s" % (src, r.stdout, r.stderr))
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False, defines=(), out: str = LIB,
          build_dir: str = BUILD) -> str:
    """Compile every CUDA source for sm_100a and link libdcn_b200.so; returns its path.

    ``defines`` (e.g. ["DCN_FWD_MAX_STAGES=3"]) override compile-time tuning
    constants; use them with a separate ``out`` and ``build_dir``.
    """
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = (["-Xptxas", "-v"] if ptxas_verbose else []) + ["-D" + d for d in defines]
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, force or ptxas_verbose, verbose or ptxas_verbose, extra, build_dir),
                           srcs))
    newest_obj = max(os.path.getmtime(o) for o in objs)
    LIBOUT = out
    if force or not os.path.exists(LIBOUT) or os.path.getmtime(LIBOUT) < newest_obj:
        tmp = LIBOUT + ".tmp%d" % os.getpid()
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIBOUT)
    return LIBOUT


CHECKED_LIB = os.path.join(os.path.dirname(LIB), "libdcn_b200_checked.so")
CHECKED_BUILD = os.path.join(BUILD, "checked")


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """The range-checked build (DCN_CHECKED): every indexed global access of the
    gather and scatter paths is checked against its buffer before it is made; an
    access outside is skipped (a load reads zeros) and recorded in the device
    status word, which dcn_check_status reports as DCN_ERR_RANGE. Load it with
    DCN_B200_LIB=libdcn_b200_checked.so."""
    return build(force=force, verbose=verbose, defines=["DCN_CHECKED"], out=CHECKED_LIB, build_dir=CHECKED_BUILD)


if __name__ == "__main__":
    # --nvtx: rebuild the library with NVTX ranges around its entry points (--force goes back)
    # --checked: build libdcn_b200_checked.so (range-checked accesses) beside the library
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv, verbose="-v" in sys.argv))
    else:
        print(build(force="--force" in sys.argv or "--nvtx" in sys.argv, verbose="-v" in sys.argv,
                    ptxas_verbose="--ptxas" in sys.argv, defines=["DCN_NVTX"] if "--nvtx" in sys.argv else ()))
