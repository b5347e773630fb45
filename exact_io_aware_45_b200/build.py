"""Builds libfa.so (the C-ABI attention library) for sm_100a with nvcc.

    python -m exact_io_aware_45_b200.build [--verbose-ptxas]

Every ``csrc/*.cu`` file is compiled to an object under ``_build/`` (in
parallel) and linked into ``exact_io_aware_45_b200/_lib/libfa.so``. The CUDA
runtime is linked statically, so the library needs only the driver at run
time. Objects are rebuilt when a source or header is newer.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(OUT_DIR, "libfa.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "-I" + os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose_ptxas: bool = False, force: bool = False, defines=(), out_dir: str = None) -> str:
    """Compiles and links libfa.so. ``defines`` are extra ``NAME=VALUE``
    build-time tuning macros (e.g. FA_FWD_SLOTS_D128=4); a build with defines
    goes to its own object and output directories (``out_dir``, default
    ``_build/<defines>/``) so the default library is untouched."""
    lib_path, build_dir = LIB, BUILD_DIR
    if defines:
        tag = "_".join(d.replace("=", "-") for d in defines)
        build_dir = os.path.join(BUILD_DIR, tag)
        lib_path = os.path.join(out_dir or build_dir, "libfa.so")
    os.makedirs(os.path.dirname(lib_path), exist_ok=True)
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = _headers()
    cc = nvcc()
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + ["-D" + d for d in defines]

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        if force or verbose_ptxas or _stale(obj, [src] + hdrs):
            cmd = [cc] + ARCH + FLAGS + extra + ["-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
            if verbose_ptxas:
                sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(compile_one, srcs))
    if force or _stale(lib_path, objs):
        cmd = [cc] + ARCH + ["-shared", "-o", lib_path] + objs + ["-lcudart_static", "-ldl",
                                                                  "-lpthread", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="build-time tuning macro NAME=VALUE (separate output directory)")
    ap.add_argument("--out-dir", default=None)
    a = ap.parse_args()
    print(build(a.verbose_ptxas, a.force, tuple(a.defines), a.out_dir))
