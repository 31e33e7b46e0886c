"""Build libcpattn.so in-tree with nvcc for sm_100a.

    python -m context_attention_cp_b200.build [--force] [--debug-bounds]

Each .cu under csrc/ is compiled to an object in _build/ (in parallel), then all
are linked into context_attention_cp_b200/libcpattn.so with the static CUDA
runtime.  The driver API entry point for TMA descriptors is fetched at run time
(cudaGetDriverEntryPointByVersion), so nothing links libcuda directly.

--debug-bounds builds libcpattn_debug.so instead (objects in _build_debug/): the
same library compiled with CP_DEBUG_BOUNDS=1, whose tensor-core kernels check every
TMA coordinate and global index before the access and report a failed check
through cp_stream_check (CP_ERR_BOUNDS) instead of trapping.  The package loads it
when the environment variable CP_LIBRARY is set to "debug".

    python -m context_attention_cp_b200.build --define NAME=VALUE ... --out PATH

builds a variant with extra preprocessor definitions (the kernels' compile-time
knobs, e.g. CP_ATTN_PINGPONG=1) into PATH (objects beside it); CP_LIBRARY=PATH
makes the package load it, so a variant is timed with the same bench.py command.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libcpattn.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libcpattn_debug.so")
HEADER = os.path.join(ROOT, "include", "cpattn.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hdrs + [HEADER, __file__]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, extra, bdir=BUILD):
    obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
    if _stale(obj, [src] + _deps()):
        cmd = [nvcc()] + ARCH + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
        if r.stderr.strip():
            sys.stderr.write(r.stderr)
    return obj


def build(force=False, verbose_ptxas=False, debug_bounds=False, defines=(), out=None):
    """Compile (if stale) and return the path of libcpattn.so (libcpattn_debug.so
    with debug_bounds; `out` with extra `defines`)."""
    bdir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug_bounds else (BUILD, LIB)
    if out:
        lib = os.path.abspath(out)
        bdir = lib + ".objs"
    os.makedirs(bdir, exist_ok=True)
    if force:
        for f in os.listdir(bdir):
            os.remove(os.path.join(bdir, f))
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if debug_bounds:
        extra = extra + ["-DCP_DEBUG_BOUNDS=1"]
    extra = extra + ["-D" + d for d in defines]
    srcs = sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, bdir), srcs))
    if force or _stale(lib, objs):
        tmp = lib + ".tmp%d" % os.getpid()
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + ["-ldl"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, lib)
    return lib


def _main(argv):
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    ap.add_argument("--define", action="append", default=[])
    ap.add_argument("--out")
    a = ap.parse_args(argv)
    if a.define and not a.out:
        ap.error("--define needs --out (a variant never replaces the default library)")
    return build(force=a.force, verbose_ptxas=a.ptxas_v, debug_bounds=a.debug_bounds, defines=a.define, out=a.out)


if __name__ == "__main__":
    print(_main(sys.argv[1:]))
