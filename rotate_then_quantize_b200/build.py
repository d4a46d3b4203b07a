"""Builds libsrftq.so in-tree with nvcc for sm_100a.

Each translation unit under csrc/ compiles in parallel to an object file in
_build/ at the repository root; the objects are linked into
rotate_then_quantize_b200/libsrftq.so. An object is rebuilt when it is older
than its source or any header it may include (all of csrc/*.cuh and
include/*.h). Usage:
``python -m rotate_then_quantize_b200.build [-j N] [--force] [--debug]``.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsrftq.so")
LIB_DEBUG = os.path.join(PKG, "libsrftq_debug.so")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -fno-gnu-unique and -Bsymbolic keep every function-local static (the
# per-kernel attribute and occupancy caches) private to its library: a
# process may load libsrftq.so and libsrftq_debug.so side by side, and GCC
# would otherwise emit those statics as STB_GNU_UNIQUE symbols, which the
# dynamic linker merges across libraries even when they are loaded locally.
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-Xcompiler", "-fno-gnu-unique", "-I", os.path.join(ROOT, "include")]
LINK_FLAGS = ["-Xlinker", "-Bsymbolic"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps_mtime():
    deps = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    deps.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in deps)


def _compile(src: str, force: bool, verbose_ptxas: bool, build_dir: str, flags: list):
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(src), _deps_mtime())):
        return obj, None
    cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr[-8000:]}")
    return obj, r.stderr if verbose_ptxas else None


def build(jobs: int | None = None, force: bool = False, verbose_ptxas: bool = False,
          debug: bool = False) -> str:
    """Compiles every csrc/*.cu for sm_100a and links the in-tree library; returns its path.

    debug=True builds libsrftq_debug.so instead (objects in _build/debug,
    -DSRFTQ_DEBUG_CHECKS=1): the same kernels with index checks that record
    an out-of-range access in the device guard word instead of making it."""
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = LIB_DEBUG if debug else LIB
    flags = FLAGS + (["-DSRFTQ_DEBUG_CHECKS=1"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    logs = []
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        futs = [ex.submit(_compile, s, force, verbose_ptxas, build_dir, flags) for s in srcs]
        objs = []
        for f in futs:
            obj, log = f.result()
            objs.append(obj)
            if log:
                logs.append(log)
    if (force or not os.path.exists(lib)
            or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs)):
        cmd = [NVCC, *ARCH, "-shared", *LINK_FLAGS, "-o", lib, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr[-8000:]}")
    if verbose_ptxas:
        with open(os.path.join(build_dir, "ptxas.log"), "w") as f:
            f.write("\n".join(logs))
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("-j", "--jobs", type=int, default=None)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true",
                    help="write ptxas register/spill reports to _build/ptxas.log")
    ap.add_argument("--debug", action="store_true",
                    help="build libsrftq_debug.so, the kernels with device-side index checks")
    args = ap.parse_args(argv)
    print(build(args.jobs, args.force, args.ptxas_verbose, args.debug))


if __name__ == "__main__":
    sys.exit(main())
