"""Build libstarattn.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_attention_phase_b200.build [--force] [-v] [--debug]

Objects go to _build/ at the repository root; the shared library is written
next to this file so that it travels with the source tree. --debug builds
libstarattn_debug.so instead: the same library with -DSTAR_DEBUG (index checks
on every global store of the kernels, see include/star_attn.h).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_NAME = "libstarattn.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
DEBUG_LIB_PATH = os.path.join(HERE, "libstarattn_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-I", INCLUDE, "-I", CSRC,
          "-Xcompiler", "-fPIC,-fvisibility=hidden", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libstarattn")
    return path


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def _compile(src: str, verbose: bool, extra, obj_dir: str = BUILD_DIR) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [nvcc()] + ARCH + COMMON + list(extra) + ["-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    """Compile every source under csrc/ and link libstarattn.so (or, with debug,
    libstarattn_debug.so with -DSTAR_DEBUG). Returns the library's path."""
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    obj_dir = os.path.join(BUILD_DIR, "debug") if debug else BUILD_DIR
    extra = list(extra) + (["-DSTAR_DEBUG=1"] if debug else [])
    if not force and (debug or not extra) and up_to_date(lib_path):
        return lib_path
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, obj_dir), srcs))
    tmp = lib_path + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    ap.add_argument("--debug", action="store_true",
                    help="build libstarattn_debug.so (index checks on every store)")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="NAME=VALUE passed to the compiler (tuning constants)")
    args = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if args.ptxas_info else []
    extra += [f"-D{d}" for d in args.defines]
    path = build(force=args.force or args.ptxas_info or bool(args.defines),
                 verbose=args.verbose or args.ptxas_info, extra=extra, debug=args.debug)
    print(path)
    return 0


if __name__ == "__main__":
    sys.exit(main())
