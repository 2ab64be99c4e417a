"""Build libpa.so (sm_100a) in-tree with nvcc.

``python -m paged_kv_cache_388_b200.build`` compiles every ``csrc/*.cu`` to an
object and links them into ``paged_kv_cache_388_b200/libpa.so``.  Objects are
rebuilt only when a source or header is newer than them.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
BUILD = os.environ.get("PA_BUILD_DIR", os.path.join(PKG, "_build"))
LIB = os.environ.get("PA_LIB_OUT", os.path.join(PKG, "libpa.so"))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills", "-I", INCLUDE] + os.environ.get("PA_NVCC_DEFINES", "").split()


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


# The test build of the decode kernel: a 50 ms wait limit and one ring use of
# CTA 0 announced but never copied, so that a test can watch a wait expire and
# the kernel unwind with PA_DEVERR_TIMEOUT (tests/test_wait_timeout.py).
WAITTEST_LIB = os.path.join(PKG, "libpa_waittest.so")
WAITTEST_SRC = "decode_mma.cu"
WAITTEST_DEFINES = ["-DPA_WAIT_LIMIT_NS=50000000ull", "-DPA_TEST_LOST_COPY=3"]


def _compile(src, verbose=False, defines=(), tag=""):
    obj = os.path.join(BUILD, os.path.basename(src) + tag + ".o")
    if not _stale(obj, [src] + _headers()):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *defines, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose or r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(verbose: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if force:
        for o in glob.glob(os.path.join(BUILD, "*.o")):
            os.remove(o)
    wt_src = os.path.join(CSRC, WAITTEST_SRC)
    jobs = [(s, (), "") for s in srcs] + [(wt_src, WAITTEST_DEFINES, ".waittest")]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        built = list(ex.map(lambda j: _compile(j[0], verbose, j[1], j[2]), jobs))
    objs, wt_obj = built[:-1], built[-1]
    _link(LIB, objs)
    _link(WAITTEST_LIB, [o for o in objs if os.path.basename(o) != WAITTEST_SRC + ".o"] + [wt_obj])
    return LIB


def _link(out, objs):
    if _stale(out, objs):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
