"""Builds libmsda.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m scale_deformable_attention_msdeformattn_b200.build [--verbose]

The library links only the CUDA runtime (statically, nvcc's default); it has
no PyTorch dependency.  Its .cu files compile in parallel.  The build is
skipped when the .so is newer than every source file.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmsda.so")
CHECKED = os.path.join(PKG, "libmsda_checked.so")  # MSDA_BOUNDS_CHECK=1 variant (tests)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -static-global-template-stub=false: msda_api.cu launches kernel templates
# that other units instantiate (extern template), which whole-program mode
# supports only with non-static template stubs
COMPILE_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                 "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
                 "-static-global-template-stub=false"]
LINK_FLAGS = ["-shared", "-Xcompiler", "-fPIC"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def up_to_date(path: str = LIB) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build_checked(force: bool = False) -> str:
    """The checked variant: every corner row a kernel reads or reduces into is
    tested against its tensor (MSDA_BOUNDS_CHECK=1); the tests run it."""
    if not force and up_to_date(CHECKED):
        return CHECKED
    return build(force=True, out=CHECKED, defines=("MSDA_BOUNDS_CHECK=1",))


def _compile(args):
    cmd, verbose = args
    res = subprocess.run(cmd, capture_output=True, text=True)
    return cmd, res.returncode, res.stdout, res.stderr


def build(force: bool = False, verbose: bool = False, out: str = LIB, defines=()) -> str:
    """Compiles the library to `out`; `defines` are extra -D tuning knobs.

    Each .cu file (the C ABI and one file per group of kernel instantiations)
    compiles to an object in parallel; nvcc then links the shared library."""
    if not force and out == LIB and not defines and up_to_date():
        return LIB
    objdir = out + ".%d.obj" % os.getpid()
    os.makedirs(objdir, exist_ok=True)
    try:
        jobs = []
        for src in sources():
            obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
            cmd = [nvcc()] + ARCH + COMPILE_FLAGS + ["-D" + d for d in defines] + \
                ["-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append((cmd, verbose))
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        objs = []
        with concurrent.futures.ThreadPoolExecutor(workers) as pool:
            for cmd, rc, so, se in pool.map(_compile, jobs):
                if verbose or rc != 0:
                    print(" ".join(cmd))
                    sys.stdout.write(so)
                    sys.stderr.write(se)
                if rc != 0:
                    raise RuntimeError("nvcc failed (exit %d)" % rc)
                objs.append(cmd[cmd.index("-o") + 1])
        tmp = out + ".%d.tmp" % os.getpid()
        link = [nvcc()] + ARCH + LINK_FLAGS + ["-o", tmp] + objs
        res = subprocess.run(link, capture_output=True, text=True)
        if verbose or res.returncode != 0:
            sys.stdout.write(res.stdout)
            sys.stderr.write(res.stderr)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed (exit %d)" % res.returncode)
        os.replace(tmp, out)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
