"""Builds libusp.so in-tree with nvcc for sm_100a.

    python -m ulysses_sequence_attention_sp_b200.build [--force] [--verbose]

Objects go to ``_build/`` at the repository root; the shared library is
written next to this file, where the ctypes binding loads it. The CUDA
runtime is linked statically (nvcc's default), so the library does not depend
on which libcudart PyTorch loaded.
"""

from __future__ import annotations

import argparse
import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(PKG_DIR, "libusp.so")
# The bounds-checking build (-DUSP_BOUNDS_CHECK): every global offset of the copy
# kernels and the attention epilogues is range-checked; a debugging aid, loaded
# through $USP_LIBRARY.
CHECKED_LIB_PATH = os.path.join(PKG_DIR, "libusp_checked.so")

SOURCES = ["plan.cpp", "tensor_map.cpp", "permute.cu", "pack_tma.cu", "rows.cu", "attn_tc.cu", "attn_pp.cu", "attn_simt.cu", "noalloc.cu", "dist.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libusp.so")
    return path


def _deps() -> list[str]:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "usp.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    lib_mtime = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= lib_mtime for f in _deps())


def _compile(src: str, extra: list[str], verbose: bool, build_dir: str = BUILD_DIR) -> str:
    obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *COMMON, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    if src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"] if verbose else []
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}")
    return obj


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    """Compiles every source for sm_100a and links libusp.so (or `out`, for a
    variant built with `extra` flags such as -DUSP_TRACE); returns its path."""
    lib_path = out or LIB_PATH
    if not force and not extra and out is None and up_to_date():
        return LIB_PATH
    build_dir = BUILD_DIR if out is None else os.path.join(BUILD_DIR, "variant")
    os.makedirs(build_dir, exist_ok=True)
    extra = list(extra or [])
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, verbose, build_dir), SOURCES))
    tmp = lib_path + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        raise RuntimeError("linking libusp.so failed")
    os.replace(tmp, lib_path)
    return lib_path


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """Builds the bounds-checking variant into CHECKED_LIB_PATH; returns its path."""
    if (not force and os.path.exists(CHECKED_LIB_PATH)
            and all(os.path.getmtime(f) <= os.path.getmtime(CHECKED_LIB_PATH) for f in _deps())):
        return CHECKED_LIB_PATH
    return build(force=True, verbose=verbose, extra=["-DUSP_BOUNDS_CHECK"], out=CHECKED_LIB_PATH)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    main()
