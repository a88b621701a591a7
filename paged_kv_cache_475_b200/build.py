"""Build libpa.so in-tree with nvcc for sm_100a (B200).

python paged_kv_cache_475_b200/build.py [--force] [--verbose]
(run it as a script: importing the package loads libpa.so, which may not exist yet)

Sources are compiled in parallel into _build/ (git-ignored) and linked into
paged_kv_cache_475_b200/libpa.so. A rebuild happens only when a source or the
public header is newer than the library.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpa.so")
HEADER = os.path.join(ROOT, "include", "pa.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpa.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _flags_file(lib: str) -> str:
    return lib + ".defines"


def _stale(defines=()) -> bool:
    if not os.path.exists(LIB):
        return True
    # a library built with other -D macros (e.g. a --trace build) is rebuilt
    try:
        with open(_flags_file(LIB)) as f:
            built_with = f.read().split()
    except OSError:
        built_with = []
    if sorted(built_with) != sorted(defines):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, defines=None, lib: str = LIB, objdir: str = BUILD) -> str:
    """Compile every CUDA source for sm_100a and link libpa.so; returns its path.

    defines: extra -D macros (tuning variants), written to `lib` with objects in `objdir`; None takes
    them from the PA_BUILD_DEFINES environment variable (space-separated, empty by default), so that
    a variant built that way is not rebuilt by a later plain build() in the same environment.
    """
    if defines is None:
        defines = tuple(os.environ.get("PA_BUILD_DEFINES", "").split())
    if not force and os.path.abspath(lib) == LIB and not _stale(tuple(defines)):
        return LIB
    os.makedirs(objdir, exist_ok=True)
    cc = nvcc()
    procs = []
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        log = obj + ".log"
        objs.append(obj)
        cmd = [cc, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-c", src, "-o", obj]
        f = open(log, "w")
        procs.append((src, subprocess.Popen(cmd, stdout=f, stderr=subprocess.STDOUT), f, log))
    failed = []
    for src, pr, f, log in procs:
        rc = pr.wait()
        f.close()
        text = open(log).read()
        if verbose or rc:
            sys.stderr.write(f"--- {os.path.basename(src)} (rc={rc})\n{text}\n")
        if rc:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for: {', '.join(os.path.basename(s) for s in failed)}")
    tmp = lib + ".tmp"
    link = [cc, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(link, capture_output=True, text=True)
    if r.returncode:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    with open(_flags_file(lib), "w") as f:
        f.write(" ".join(defines))
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true",
                    help="build with per-CTA timeline records (PA_TRACE=1; pa_trace_read), off by default")
    a = ap.parse_args()
    print(build(force=a.force or a.trace, verbose=a.verbose, defines=("PA_TRACE=1",) if a.trace else ()))
