"""Build librq.so in-tree with nvcc for sm_100a.

    python -m kv_quantization_b200.build [--force]

Each .cu under csrc/ compiles to an object in parallel (nvcc -gencode
arch=compute_100a,code=sm_100a -lineinfo -O3, position-independent), then the
objects link into kv_quantization_b200/librq.so.  No fast-math and no
multiply-add contraction: the kernels rely on IEEE-rounded fp32 adds,
multiplies, reciprocals and square roots, each rounded on its own.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "librq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# --fmad=false: no multiply-add contraction anywhere.  The canonical arithmetic
# rounds every product and every sum separately; the packed f32x2 intrinsics
# were measured to be contracted otherwise (the residual x - w * s came out
# with a single rounding).  Explicit fma intrinsics are unaffected.
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-rdc=true", "-Xcompiler", "-fPIC", "-Xcompiler", "-fno-fast-math",
              "--ftz=false", "--prec-div=true", "--prec-sqrt=true", "--fmad=false", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build librq")
    return path


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


_INCLUDE_RE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _closure(src):
    """The source and every local header it includes, transitively."""
    seen, todo = set(), [src]
    while todo:
        f = todo.pop()
        if f in seen or not os.path.exists(f):
            continue
        seen.add(f)
        with open(f, encoding="utf-8", errors="replace") as fh:
            for name in _INCLUDE_RE.findall(fh.read()):
                for d in (os.path.dirname(f), CSRC, INCLUDE):
                    cand = os.path.join(d, name)
                    if os.path.exists(cand):
                        todo.append(os.path.normpath(cand))
                        break
    return seen


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(OBJ, os.path.basename(src) + ".o")
        if not force and not extra_flags and os.path.exists(obj) and \
                all(os.path.getmtime(p) <= os.path.getmtime(obj) for p in _closure(src)):
            return obj                              # nothing it depends on changed
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, file=sys.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-rdc=true", "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    t0 = __import__("time").time()
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else ()))
    print(f"built in {__import__('time').time() - t0:.1f}s")
