"""Build libjlkey.so (the CUDA library behind include/jlkey.h) in-tree.

    python -m bit_jl_key_b200.build [--force] [--verbose] [--debug-index]

Compiles every csrc/*.cu for sm_100a with nvcc and links one shared library
next to this file.  Objects go to bit_jl_key_b200/_build/ (ignored by git).
Rebuilds only what changed (sources are compared by mtime against their
object and every header in csrc/ and include/).

--debug-index builds the index-checking variant libjlkey_debug.so instead
(objects in _build/debug/, compiled with -DJL_DEBUG_INDEX): every global
access the kernels make through a raw pointer is checked against the extent
the call's shapes give that buffer, and one outside it is skipped and
reported as JL_DERR_INDEX through jl_device_error.  Load it by setting
JLKEY_LIBRARY to its path.
"""
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libjlkey.so")
DEBUG_OBJ_DIR = os.path.join(OBJ_DIR, "debug")
DEBUG_LIB = os.path.join(HERE, "libjlkey_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
              "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"),
                 "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libjlkey")


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def build(force: bool = False, verbose: bool = False, extra_flags=(),
          debug_index: bool = False) -> str:
    obj_dir, lib = (DEBUG_OBJ_DIR, DEBUG_LIB) if debug_index else (OBJ_DIR, LIB)
    if debug_index:
        extra_flags = (*extra_flags, "-DJL_DEBUG_INDEX")
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    objs, procs = [], []
    for src in srcs:
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_mtime)):
            continue
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            sys.stdout.write(out)
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    newest_obj = max(os.path.getmtime(o) for o in objs)
    if force or procs or not os.path.exists(lib) or os.path.getmtime(lib) < newest_obj:
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                debug_index="--debug-index" in sys.argv))
