"""Build libgva.so in-tree with nvcc for sm_100a (B200).

    python -m compressed_kv_cache_gva_b200._build [--force]

Each .cu under csrc/ is compiled to an object in parallel, then linked into
compressed_kv_cache_gva_b200/libgva.so (static CUDA runtime, no torch symbols).
A rebuild happens only when a source or header is newer than the library.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgva.so")
OBJDIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-O2", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


# Test-only variant for the failure-detection test: bounded pipeline waits give up
# after 50 ms, and the split kernel's producer never requests the second tile of
# each CTA, so a consumer wait runs out (no copy is ever in flight for that tile).
WAIT_TEST_LIB = os.path.join(PKG, "libgva_waittest.so")
WAIT_TEST_FLAGS = ("-DGVA_WAIT_NS=50000000ull", "-DGVA_TEST_WITHHOLD_TILE=1")


def up_to_date(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), out: str = LIB) -> str:
    """Compile every csrc/*.cu and link them into `out` (default: the package's
    libgva.so).  `extra_flags` go to every nvcc compile (e.g. -DGVA_TRACE)."""
    if not force and up_to_date(out) and (not extra_flags or out != LIB):
        return out
    os.makedirs(OBJDIR, exist_ok=True)
    srcs = _sources()

    tag = "" if not extra_flags else "_" + hashlib.sha1(" ".join(extra_flags).encode()).hexdigest()[:12]
    def compile_one(src):
        obj = os.path.join(OBJDIR, os.path.basename(src) + tag + ".o")
        cmd = [NVCC, *FLAGS, *extra_flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = out + ".tmp"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, out)
    return out


def build_wait_test(force: bool = False) -> str:
    """The failure-detection test's library (see WAIT_TEST_FLAGS)."""
    return build(force=force, extra_flags=WAIT_TEST_FLAGS, out=WAIT_TEST_LIB)


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build with -DGVA_TRACE")
    ap.add_argument("--out", default=LIB)
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.v, extra_flags=["-DGVA_TRACE"] if a.trace else [], out=a.out))
