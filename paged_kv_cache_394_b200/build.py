"""Build ``libpagedkv.so`` in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_394_b200.build [--verbose-ptxas] [-j N] [--force]
                                            [--define NAME=VALUE ...]

Each source under ``csrc/`` is compiled to an object in ``_build/`` (in
parallel, skipped when up to date), then linked into
``paged_kv_cache_394_b200/libpagedkv.so`` with the CUDA runtime linked
statically, so the library does not depend on which libcudart the host
process has loaded.  ``--define`` passes a preprocessor definition to every
source (the tuning and comparison switches the sources document); objects
built with other definitions are rebuilt.
"""

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3,-Wall",
          "-I", INCLUDE, "-I", CSRC]


def nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found")
    return exe


def sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def headers_mtime():
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    paths.append(os.path.join(INCLUDE, "pagedkv.h"))
    return max(os.path.getmtime(p) for p in paths)


def compile_one(src, verbose_ptxas, force, defines=()):
    obj = os.path.join(BUILD, src + ".o")
    srcp = os.path.join(CSRC, src)
    stamp = obj + ".defines"
    tag = " ".join(defines)
    same_defines = os.path.exists(stamp) and open(stamp).read() == tag
    if (not force and same_defines and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(srcp), headers_mtime())):
        return obj, ""
    cmd = [nvcc()] + ARCH + COMMON + ["-D" + d for d in defines] + ["-c", srcp, "-o", obj]
    if verbose_ptxas and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    if src.endswith(".cpp"):
        cmd += ["-x", "c++"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
    with open(stamp, "w") as f:
        f.write(tag)
    return obj, r.stderr


def build(verbose_ptxas=False, jobs=None, force=False, quiet=True, defines=()):
    os.makedirs(BUILD, exist_ok=True)
    srcs = sources()
    defines = tuple(sorted(defines))
    with ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: compile_one(s, verbose_ptxas, force, defines), srcs))
    objs = [o for o, _ in results]
    if verbose_ptxas:
        for _, log in results:
            if log:
                sys.stderr.write(log)
    if (force or not os.path.exists(LIB)
            or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)):
        tmp = LIB + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + \
              ["-lpthread", "-ldl", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIB)
    if not quiet:
        print("built", LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("--define", action="append", default=[], metavar="NAME=VALUE")
    a = ap.parse_args()
    build(a.verbose_ptxas, a.j, a.force, quiet=False, defines=a.define)


if __name__ == "__main__":
    main()
