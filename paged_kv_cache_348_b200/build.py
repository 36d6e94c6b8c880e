"""Build libpagedkv.so in-tree with nvcc for sm_100a (no JIT, no torch extension)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpagedkv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
    "-I", CSRC,
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(ROOT, "include", "pagedkv.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every source to an object in parallel (the decode kernel instances are
    spread over several translation units), then link libpagedkv.so."""
    if not force and not _stale():
        return LIB
    import concurrent.futures
    import tempfile

    compile_flags = [f for f in FLAGS if f != "-shared"]
    with tempfile.TemporaryDirectory(prefix="pagedkv_build_") as tmpdir:
        def compile_one(src):
            obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
            cmd = [NVCC, *compile_flags, *extra, "-c", "-o", obj, src]
            r = subprocess.run(cmd, capture_output=True, text=True)
            return src, obj, cmd, r
        srcs = sources()
        workers = max(1, min(len(srcs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            results = list(ex.map(compile_one, srcs))
        for src, obj, cmd, r in results:
            if verbose:
                print(" ".join(cmd), flush=True)
                sys.stdout.write(r.stdout)
                sys.stderr.write(r.stderr)
            if r.returncode != 0:
                if not verbose:
                    sys.stderr.write(r.stderr)
                raise subprocess.CalledProcessError(r.returncode, cmd)
        tmp = LIB + ".tmp%d" % os.getpid()
        link = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp,
                *[obj for _, obj, _, _ in results]]
        if verbose:
            print(" ".join(link), flush=True)
        subprocess.check_call(link)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
