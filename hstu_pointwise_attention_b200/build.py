"""Build libhstu.so (sm_100a) in-tree with nvcc.

    python -m hstu_pointwise_attention_b200.build [--force] [--verbose] [--trace]

Compiles every csrc/*.cu for sm_100a only (-gencode arch=compute_100a,code=sm_100a)
and links one shared library, lib/libhstu.so, with the CUDA runtime linked
statically (the driver is reached through the runtime's entry-point query).
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIBDIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIBDIR, "libhstu.so")
INCLUDE = os.path.join(ROOT, "include")
# The phase-traced variant (-DHSTU_TRACE): its own objects and library, so the
# product library is never replaced by it.
TRACE_LIB = os.path.join(HERE, "lib_trace", "libhstu.so")
TRACE_OBJDIR = os.path.join(ROOT, "_build_trace")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA library cannot be built")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), trace: bool = False) -> str:
    """Build the library; with trace=True the phase-traced variant (TRACE_LIB)."""
    lib = TRACE_LIB if trace else LIB
    # objects are reused only when built with the same flags (the traced
    # objects live in their own folder)
    reuse = not force and not extra
    if trace:
        extra = tuple(extra) + ("-DHSTU_TRACE",)
    if not force and not trace and not _stale():
        return LIB
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    objdir = TRACE_OBJDIR if trace else os.path.join(ROOT, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs, procs = [], []
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    newest_header = max((os.path.getmtime(h) for h in headers), default=0.0)
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        # An object is reused only if it is newer than its source and every header.
        if (reuse and os.path.exists(obj) and
                os.path.getmtime(obj) > max(os.path.getmtime(src), newest_header)):
            continue
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((subprocess.Popen(cmd), src))
    failed = [src for p, src in procs if p.wait() != 0]
    if failed:
        raise RuntimeError("nvcc failed on: " + ", ".join(failed))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print register/smem usage")
    ap.add_argument("--trace", action="store_true",
                    help="build the phase-traced variant into lib_trace/ (product library untouched)")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_info else []
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose, extra=extra, trace=a.trace))
    return 0


if __name__ == "__main__":
    sys.exit(main())
