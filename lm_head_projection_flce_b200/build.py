"""Build libflce.so (the sm_100a CUDA kernels and their C ABI) in-tree with nvcc.

    python -m lm_head_projection_flce_b200.build [--force]

nvcc cross-compiles for sm_100a without a GPU.  The library links the CUDA
runtime statically and resolves cuTensorMapEncodeTiled from the driver at run
time, so it loads on a machine without a GPU (its calls then return an error).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libflce.so")
DIGEST_PATH = LIB_PATH + ".sources"  # sha256 of the sources the library was built from
MAIN_SOURCE = os.path.join(CSRC, "flce.cu")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libflce.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def source_digest() -> str:
    h = hashlib.sha256()
    for p in sources():
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    h.update(" ".join(ARCH_FLAGS + NVCC_FLAGS).encode())
    return h.hexdigest()


def is_stale() -> bool:
    """True when the library is missing or was built from other sources or flags
    (compared by content, so copying the tree does not force a rebuild)."""
    if not os.path.exists(LIB_PATH) or not os.path.exists(DIGEST_PATH):
        return True
    with open(DIGEST_PATH) as f:
        return f.read().strip() != source_digest()


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libflce.so if missing or older than its sources; return its path."""
    if not force and not is_stale():
        return LIB_PATH
    tmp = f"{LIB_PATH}.tmp{os.getpid()}"  # concurrent builders never share a temp file
    cmd = [_nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, f"-I{INCLUDE}", "-o", tmp, MAIN_SOURCE]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    digest = source_digest()
    os.replace(tmp, LIB_PATH)
    with open(f"{DIGEST_PATH}.tmp{os.getpid()}", "w") as f:
        f.write(digest + "\n")
    os.replace(f"{DIGEST_PATH}.tmp{os.getpid()}", DIGEST_PATH)
    return LIB_PATH


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))
    return 0


if __name__ == "__main__":
    sys.exit(main())
