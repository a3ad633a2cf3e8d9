"""Builds the CUDA library (csrc/*.cu) into libmqa_logits.so in this folder.

nvcc, sm_100a only (-gencode arch=compute_100a,code=sm_100a), static CUDA
runtime, -lineinfo for the profiler. Objects go to _build/ at the repo root.
With debug=True (--debug) the same sources are built with -DMQA_DEBUG into
libmqa_logits_debug.so (objects in _build/debug/): the kernels then check
their pipeline invariants and report a failure as MQA_STATUS_DEBUG_INVARIANT
(the binding loads that library when MQA_LOGITS_DEBUG=1).
Run: python -m paged_mqa_logits_b200.build [--force] [--debug]
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmqa_logits.so")
LIB_DEBUG = os.path.join(HERE, "libmqa_logits_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    dep = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    inc = os.path.join(ROOT, "include")
    dep += [os.path.join(inc, f) for f in os.listdir(inc) if f.endswith(".h")]
    return dep


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    obj_dir = os.path.join(OBJ, "debug") if debug else OBJ
    flags = FLAGS + (["-DMQA_DEBUG"] if debug else [])
    srcs = sources()
    newest = max(os.path.getmtime(p) for p in srcs + _deps() + [__file__])
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    os.makedirs(obj_dir, exist_ok=True)
    exe = nvcc()

    def compile_one(src):
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        cmd = [exe, *ARCH, *flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp"
    cmd = [exe, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
