"""Build the in-tree CUDA library ``libkroquant.so`` for sm_100a.

    python -m w4a4_dit_post_b200.build [--force] [--verbose]

Compiles ``csrc/*.cu`` and ``csrc/*.cpp`` with nvcc
(``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3``) and links a
shared library next to this file.  The library links the CUDA runtime
statically and talks to the driver through the runtime only, so it loads on
a machine without a GPU (nothing runs until a function is called).  A hash of
the sources is stored beside the library; an unchanged tree is not rebuilt.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_NAME = "libkroquant.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
HASH_PATH = LIB_PATH + ".srchash"
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def sources() -> list[str]:
    out = []
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cpp")):
            out.append(os.path.join(CSRC, name))
    return out


def _hash_inputs() -> str:
    h = hashlib.sha256()
    files = sorted(
        [os.path.join(CSRC, n) for n in os.listdir(CSRC)]
        + [os.path.join(INCLUDE, n) for n in os.listdir(INCLUDE)]
        + [os.path.abspath(__file__)]
    )
    for f in files:
        if os.path.isfile(f):
            h.update(os.path.relpath(f, ROOT).encode())
            with open(f, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def source_hash() -> str:
    """Hash of everything the library is built from."""
    return _hash_inputs()


# the translation unit of the streaming kernels and everything it includes
STREAM_KERNEL_FILES = ("csrc/kq_stream.cu", "csrc/kq_device.cuh", "csrc/kq_host.h", "../include/kq.h")


def stream_kernel_hash() -> str:
    """Hash of the sources the streaming kernels (kq_quantize, sq_quantize,
    kq_transform) are compiled from, and of the compile flags."""
    h = hashlib.sha256()
    h.update(" ".join(ARCH_FLAGS).encode())
    for rel in STREAM_KERNEL_FILES:
        path = os.path.normpath(os.path.join(os.path.dirname(os.path.abspath(__file__)), rel))
        h.update(rel.encode())
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def is_current() -> bool:
    if not os.path.exists(LIB_PATH) or not os.path.exists(HASH_PATH):
        return False
    with open(HASH_PATH) as f:
        return f.read().strip() == _hash_inputs()


def _compile(nvcc: str, src: str, verbose: bool) -> tuple[str, str]:
    obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
    cmd = [nvcc, "-c", src, "-o", obj, "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo",
           "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC]
    if src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    log = res.stdout + res.stderr
    if verbose:
        print(log)
    return obj, log


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile and link the library if the sources changed; return its path."""
    if not force and is_current():
        return LIB_PATH
    nvcc = nvcc_path()
    os.makedirs(BUILD_DIR, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        results = list(ex.map(lambda s: _compile(nvcc, s, verbose), srcs))
    objs = [o for o, _ in results]
    with open(os.path.join(BUILD_DIR, "ptxas.log"), "w") as f:
        for (_, log), s in zip(results, srcs):
            f.write(f"== {os.path.basename(s)}\n{log}\n")
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc, "-shared", "-o", tmp, *objs, *ARCH_FLAGS, "-cudart", "static"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, LIB_PATH)
    with open(HASH_PATH, "w") as f:
        f.write(_hash_inputs())
    return LIB_PATH


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    path = build(force=a.force, verbose=a.verbose)
    print(path)
    return 0


if __name__ == "__main__":
    sys.exit(main())
