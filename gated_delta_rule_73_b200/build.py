"""Build the CUDA library ``libkda_b200.so`` in-tree for sm_100a.

``python -m gated_delta_rule_73_b200.build`` (or ``build()``) compiles every
``csrc/*.cu`` with nvcc for ``sm_100a`` and links one shared library next to
this file.  Objects go to ``_build/`` at the repository root.

Staleness is decided by content, not by file times: the library and each object
carry a stamp file with the SHA-256 of every source and header they depend on and
of the compiler flags.  A library copied from elsewhere, or built from other
sources, is rebuilt; ``LAST_BUILD`` says what the last ``build()`` did.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INC = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkda_b200.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-I" + INC, "-I" + CSRC]


def _nvcc():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libkda_b200.so")
    return cand


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INC, "*.h")))


LAST_BUILD = {"compiled": None, "objects_compiled": []}


def _digest(files, flags):
    h = hashlib.sha256()
    # flags with this checkout's absolute paths made relative, so a copy elsewhere matches
    h.update(" ".join(f.replace(ROOT, "<root>") for f in flags).encode())
    for f in files:
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _fresh(target, digest):
    stamp = target + ".stamp"
    if not (os.path.exists(target) and os.path.exists(stamp)):
        return False
    with open(stamp) as fh:
        return fh.read().strip() == digest


def _stamp(target, digest):
    with open(target + ".stamp", "w") as fh:
        fh.write(digest + "\n")


def build(verbose: bool = False, extra_flags=()) -> str:
    """Compile what is stale and return the path of the shared library.

    Sets ``LAST_BUILD["compiled"]`` to True when the library was (re)linked and to False
    when the stamped library already matched every source, header and flag."""
    deps = _deps() + [os.path.abspath(__file__)]
    flags = [*ARCH, *NVCC_FLAGS, *extra_flags]
    lib_digest = _digest(deps, flags)
    if _fresh(LIB, lib_digest):
        LAST_BUILD.update(compiled=False, objects_compiled=[])
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    nvcc = _nvcc()
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = [d for d in deps if not d.endswith(".cu")]
    compiled = []

    def compile_one(src):
        obj = os.path.join(OBJDIR, os.path.basename(src) + ".o")
        dg = _digest([src] + headers, flags)
        if not _fresh(obj, dg):
            cmd = [nvcc, *flags, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
            if verbose and r.stderr:
                print(r.stderr, file=sys.stderr)
            _stamp(obj, dg)
            compiled.append(os.path.basename(src))
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(compile_one, srcs))
    cmd = [nvcc, *ARCH, "-shared", "-o", LIB, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    _stamp(LIB, lib_digest)
    LAST_BUILD.update(compiled=True, objects_compiled=sorted(compiled))
    print(f"built {os.path.relpath(LIB, ROOT)} (compiled: {', '.join(sorted(compiled)) or 'none, relinked'})",
          file=sys.stderr)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
