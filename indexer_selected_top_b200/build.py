"""Builds libsa.so (the CUDA library behind include/sa.h) in-tree with nvcc
for sm_100a. Usage: python indexer_selected_top_b200/build.py [--force]
[--debug-checks: libsa_debug.so, with device-side invariant checks]

Run it by path (or load it with load_build below): importing the package
itself loads libsa.so, which must already exist."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["sa_api.cu", "indexer.cu", "topk.cu", "attn.cu", "pool.cu", "noalloc.cu", "topk_warp.cu", "stream.cu", "topk_fast.cu", "group.cu", "attn_tc.cu", "quant.cu", "expand.cu", "lsa.cu", "lsa_attn.cu"]
LIB = os.path.join(HERE, "libsa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills",
         "-I", os.path.join(ROOT, "include")]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "sa.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, out: str = None, defines=(), bdir: str = None) -> str:
    """Compiles every source and links libsa.so (or `out`); `defines` are
    extra -D flags (tuning knobs), built in `bdir`."""
    lib = out or LIB
    if not force and out is None and not defines and not _stale():
        return LIB
    objs = []
    bdir = bdir or os.path.join(HERE, "_build")
    os.makedirs(bdir, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, *[f"-D{d}" for d in defines], "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd))
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        objs.append(obj)
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            sys.stdout.write(out.decode())
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs]
    subprocess.check_call(cmd)
    return lib


DEBUG_LIB = os.path.join(HERE, "libsa_debug.so")


def build_debug(verbose: bool = False) -> str:
    """The debug build: the same sources with -DSA_DEBUG_CHECKS (device-side
    invariant checks that record errors for sa_debug_errors), as
    libsa_debug.so beside libsa.so. Load it with SA_LIB=<path>."""
    return build(force=True, verbose=verbose, out=DEBUG_LIB, defines=("SA_DEBUG_CHECKS",),
                 bdir=os.path.join(HERE, "_build_debug"))


if __name__ == "__main__":
    if "--debug-checks" in sys.argv:
        print(build_debug(verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True))
