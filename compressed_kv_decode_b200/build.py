"""Build ``libtq.so`` (the C-ABI library) in-tree with nvcc for sm_100a, and
``libtq_debug.so``, the same sources compiled with ``TQ_DEBUG`` (computed
indices range-checked on the device; a violation records TQ_ERR_RANGE and
skips the access)."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq.so")
LIB_DEBUG = os.path.join(HERE, "libtq_debug.so")
SOURCES = ["tq_api.cu", "tq_decode.cu", "tq_compress.cu", "tq_topk.cu", "tq_params.cpp",
           "tq_noalloc.cu", "tq_compress_tc.cu", "tq_monarch.cu",
           "tq_stage1.cu", "tq_tensor_cache.cu", "tq_self_index.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "tq.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose=False, debug=False):
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(HERE, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *(["-DTQ_DEBUG"] if debug else []), "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
