"""Build liblcsa.so (sm_100a) in-tree from csrc/*.cu with nvcc.

    python -m block_sparse_video_lcsa_b200.build [--force] [--verbose] [--nvtx] [--stalltest]

Objects go to _build/ (ignored by git); the library lands next to this file,
where the binding loads it. Rebuilds only when a source or header is newer,
or when the flags differ from the last build's. --nvtx compiles in NVTX
ranges around the kernel launches of each call (csrc/nvtx_range.h).

--stalltest builds the test-only variant liblcsa_stalltest.so instead
(-DLCSA_TEST_STALL: bounded waits give up after 100 ms, and an exported
lcsa_test_arm_stall makes the next attention launch give up a wait on
purpose). Only the device-timeout test loads it; the binding never does.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "liblcsa.so")
STALL_LIB = os.path.join(PKG, "liblcsa_stalltest.so")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, nvtx: bool = False, stalltest: bool = False) -> str:
    srcs = _sources()
    hdrs = _headers()
    extra = (["-DLCSA_NVTX"] if nvtx else []) + (["-DLCSA_TEST_STALL"] if stalltest else [])
    flags = FLAGS + extra
    lib_path = STALL_LIB if stalltest else LIB
    build_dir = os.path.join(BUILD, "stalltest") if stalltest else BUILD
    # the optional flags of the last build (no stamp: a default build)
    stamp = os.path.join(build_dir, "extra_flags.txt")
    want = " ".join(extra)
    have = ""
    if os.path.exists(stamp):
        with open(stamp) as f:
            have = f.read()
    if have != want:
        force = True  # the objects were built with other optional flags
    if not force and not _stale(lib_path, srcs + hdrs + [__file__]):
        return lib_path
    os.makedirs(build_dir, exist_ok=True)
    objs = []

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        if force or _stale(obj, [src] + hdrs + [__file__]):
            cmd = [NVCC] + ARCH + flags + (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
            if verbose:
                sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib_path + ".tmp%d" % os.getpid()
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs + (["-ldl"] if nvtx else [])
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib_path)
    with open(stamp, "w") as f:
        f.write(want)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, nvtx="--nvtx" in sys.argv,
                stalltest="--stalltest" in sys.argv))
