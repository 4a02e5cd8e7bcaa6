"""Build libsalad.so in-tree with nvcc for sm_100a.

    python -m sparse_linear_hybrid_b200.build [--force] [--verbose] [--profile | --debug]

Each translation unit compiles in parallel to an object under _build/, then one
shared library is linked next to this file.  The CUDA runtime is linked
statically; the driver is reached through cudaGetDriverEntryPoint, so the
library loads (and its symbols can be inspected) on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libsalad.so")
# variants: (object directory, library, extra nvcc flags)
#   profile: the attention kernel writes phase stamps (SALAD_PROFILE)
#   debug:   kernels check every mask row before using it (SALAD_DEBUG)
VARIANTS = {
    "release": (OBJ, LIB, []),
    "profile": (os.path.join(OBJ, "profile"), os.path.join(HERE, "libsalad_profile.so"), ["-DSALAD_PROFILE"]),
    "debug": (os.path.join(OBJ, "debug"), os.path.join(HERE, "libsalad_debug.so"), ["-DSALAD_DEBUG"]),
}
PROF_LIB = VARIANTS["profile"][1]
DEBUG_LIB = VARIANTS["debug"][1]
SOURCES = ["api.cu", "mask.cu", "linear.cu", "attn.cu", "noalloc.cu", "topk.cu", "gate.cu", "bwd.cu", "bwd_linear.cu"]
HEADERS = ["ptx.cuh", "internal.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", f"-I{os.path.join(ROOT, 'include')}"]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose, variant="release"):
    obj_dir, _, extra = VARIANTS[variant]
    obj = os.path.join(obj_dir, os.path.splitext(src)[0] + ".o")
    deps = [os.path.join(CSRC, src)] + [os.path.join(CSRC, h) for h in HEADERS] + \
        [os.path.join(ROOT, "include", "salad.h")]
    if not _stale(obj, deps):
        return obj, ""
    cmd = [NVCC, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    return obj, res.stderr


def build(force: bool = False, verbose: bool = False, profile: bool = False, debug: bool = False) -> str:
    """Builds libsalad.so, or with profile=True libsalad_profile.so (the
    attention kernel's phase stamps compiled in), or with debug=True
    libsalad_debug.so (mask rows checked on the device before use)."""
    if profile and debug:
        raise ValueError("one variant at a time")
    variant = "profile" if profile else "debug" if debug else "release"
    obj_dir, lib, _ = VARIANTS[variant]
    os.makedirs(obj_dir, exist_ok=True)
    if force:
        for f in os.listdir(obj_dir):
            if f.endswith(".o"):
                os.remove(os.path.join(obj_dir, f))
    with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, variant), SOURCES))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    if force or _stale(lib, objs):
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs]
        subprocess.check_call(cmd)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--profile", action="store_true", help="the profiling build (libsalad_profile.so)")
    ap.add_argument("--debug", action="store_true", help="the checking build (libsalad_debug.so)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.profile, a.debug))
