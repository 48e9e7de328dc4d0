"""Build liblt2gdr.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m gated_delta_rule_looped_b200.build        # or build() from Python
    python -m gated_delta_rule_looped_b200.build debug  # also liblt2gdr_debug.so

Every .cu under csrc/ is compiled with -gencode arch=compute_100a,code=sm_100a and linked
(static CUDA runtime) into gated_delta_rule_looped_b200/liblt2gdr.so.  build(debug=True) compiles
the same sources with LT2_DEBUG into liblt2gdr_debug.so: device-side index checks, a short bound
on the in-kernel waits and the fault-injection hooks of include/lt2_gdr_debug.h.  Only the
tests load the debug library.
"""
import concurrent.futures as cf
import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "liblt2gdr.so")
DEBUG_LIB = os.path.join(PKG, "liblt2gdr_debug.so")
# The debug build's bound on every in-kernel wait: long enough for any wait that a correct run
# makes on a small problem, short enough for its fault-injection test to end in milliseconds.
DEBUG_FLAGS = ["-DLT2_DEBUG", "-DLT2_WAIT_TIMEOUT_NS=20000000ull"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def needs_build(debug=False):
    lib = DEBUG_LIB if debug else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def _compile(src, extra, obj_dir=OBJ_DIR):
    obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *ARCH, *CFLAGS, *extra, "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{res.stdout}{res.stderr}")
    return obj, res.stderr


def build(verbose=False, extra_flags=(), debug=False):
    """Compile and link the library; returns the path of liblt2gdr.so (liblt2gdr_debug.so with
    debug=True)."""
    obj_dir = os.path.join(OBJ_DIR, "debug") if debug else OBJ_DIR
    lib = DEBUG_LIB if debug else LIB
    flags = list(extra_flags) + (DEBUG_FLAGS if debug else [])
    os.makedirs(obj_dir, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, flags, obj_dir), srcs))
    objs = [r[0] for r in results]
    if verbose:
        for _, log in results:
            if log:
                print(log)
    tmp = lib + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{res.stdout}{res.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(verbose=True))
    if "debug" in sys.argv[1:]:
        print(build(verbose=True, debug=True))
