"""Build the sm_100a CUDA library ``libtcq.so`` in-tree with nvcc.

    python -m trellis_coded_weight_tcq_b200.build [--verbose] [--debug]

The library links the CUDA runtime statically, so it loads next to PyTorch's
own runtime without a version clash; device pointers and streams are shared
through the primary context.  ``--debug`` also builds ``libtcq_debug.so``: the
same sources with TCQ_DEBUG defined (every global-memory index of the encode,
decode and matrix-vector kernels checked against its buffer, a failure
recorded in the device error word and the access skipped) and relocatable
device code, so that one error word serves every kernel file.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libtcq.so")
DEBUG_LIB = os.path.join(PKG, "libtcq_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the TCQ library needs the CUDA toolkit to build")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "tcq.h"),
        os.path.abspath(__file__),
    ]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every .cu under csrc/ into libtcq.so, or with ``debug`` into the
    bounds-checked libtcq_debug.so (skipped when up to date)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    common = [
        "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
        "-I", os.path.join(ROOT, "include"),
    ]
    if debug:
        common += ["-DTCQ_DEBUG", "-rdc=true"]
    if verbose:
        common += ["-Xptxas", "-v"]
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append((src, subprocess.Popen([nvcc, *common, "-c", src, "-o", obj],
                                            stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if verbose or p.returncode != 0:
            sys.stdout.write(f"--- {os.path.basename(src)}\n{text}")
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed on {failed}")
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc, *ARCH, "-shared", *(["-rdc=true"] if debug else []), "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="pass -Xptxas -v")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="also build the bounds-checked libtcq_debug.so")
    args = ap.parse_args()
    print(build(force=args.force or args.verbose, verbose=args.verbose))
    if args.debug:
        print(build(force=args.force, verbose=args.verbose, debug=True))


if __name__ == "__main__":
    main()
