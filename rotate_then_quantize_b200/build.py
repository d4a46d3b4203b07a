"""Builds libsrftq.so in-tree with nvcc for sm_100a.

Each translation unit under csrc/ compiles in parallel to an object file in
_build/ at the repository root; the objects are linked into
rotate_then_quantize_b200/libsrftq.so. An object is rebuilt when it is older
than its source or any header it may include (all of csrc/*.cuh and
include/*.h). Usage: ``python -m rotate_then_quantize_b200.build [-j N] [--force]``.
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

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps_mtime():
    deps = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    deps.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in deps)


def _compile(src: str, force: bool, verbose_ptxas: bool):
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(src), _deps_mtime())):
        return obj, None
    cmd = [NVCC, *ARCH, *FLAGS, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr[-8000:]}")
    return obj, r.stderr if verbose_ptxas else None


def build(jobs: int | None = None, force: bool = False, verbose_ptxas: bool = False,
          defines: tuple = (), out_dir: str | None = None, src_dir: str | None = None) -> str:
    """Compiles every csrc/*.cu for sm_100a and links libsrftq.so; returns its path.

    `defines` (NAME=VALUE strings), `src_dir` and `out_dir` build a variant
    of the library in a separate directory instead of the in-tree one."""
    global BUILD, LIB, CSRC
    if src_dir:
        if not out_dir:
            raise ValueError("a build from other sources needs its own out_dir")
        CSRC = os.path.abspath(src_dir)
    if defines or out_dir:
        if not out_dir:
            raise ValueError("a variant build needs its own out_dir")
        BUILD, LIB = os.path.join(out_dir, "obj"), os.path.join(out_dir, "libsrftq.so")
        FLAGS.extend(f"-D{d}" for d in defines)
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    logs = []
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        futs = [ex.submit(_compile, s, force, verbose_ptxas) for s in srcs]
        objs = []
        for f in futs:
            obj, log = f.result()
            objs.append(obj)
            if log:
                logs.append(log)
    if (force or not os.path.exists(LIB)
            or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)):
        cmd = [NVCC, *ARCH, "-shared", "-o", LIB, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr[-8000:]}")
    if verbose_ptxas:
        with open(os.path.join(BUILD, "ptxas.log"), "w") as f:
            f.write("\n".join(logs))
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("-j", "--jobs", type=int, default=None)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true",
                    help="write ptxas register/spill reports to _build/ptxas.log")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="extra preprocessor definition (variant builds)")
    ap.add_argument("--out-dir", default=None, help="directory of a variant build")
    ap.add_argument("--src", default=None, help="build these sources instead of csrc/")
    args = ap.parse_args(argv)
    path = build(args.jobs, args.force, args.ptxas_verbose, tuple(args.defines), args.out_dir,
                 args.src)
    print(path)


if __name__ == "__main__":
    sys.exit(main())
