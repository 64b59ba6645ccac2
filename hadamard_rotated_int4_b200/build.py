"""Build libhbl.so (the sm_100a CUDA library behind include/hbl.h) in-tree.

Each .cu file under csrc/ is compiled with nvcc for sm_100a only
(-gencode arch=compute_100a,code=sm_100a), without fast-math and with FMA
contraction off (--fmad=false): the kernels rely on every fp32 operation being
one IEEE round-to-nearest operation.  Objects are linked into one shared
library with the CUDA runtime linked statically.
"""
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INC = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libhbl.so")
BUILD = os.path.join(ROOT, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "--fmad=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", INC, "-I", CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps_mtime():
    files = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                         if f.endswith((".cuh", ".h"))] + [os.path.join(INC, "hbl.h")]
    return max(os.path.getmtime(f) for f in files)


_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _src_mtime(path, seen=None):
    """Latest mtime of a source and the local headers it includes (recursively)."""
    seen = set() if seen is None else seen
    if path in seen or not os.path.exists(path):
        return 0.0
    seen.add(path)
    t = os.path.getmtime(path)
    with open(path, errors="replace") as f:
        for name in _INCLUDE.findall(f.read()):
            for d in (os.path.dirname(path), CSRC, INC):
                cand = os.path.join(d, name)
                if os.path.exists(cand):
                    t = max(t, _src_mtime(cand, seen))
                    break
    return t


def build(force=False, verbose=False, ptxas_info=False):
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= _deps_mtime():
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    flags_key = " ".join(FLAGS)
    stamp = os.path.join(BUILD, "flags.txt")
    same_flags = os.path.exists(stamp) and open(stamp).read() == flags_key

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        # objects newer than their source and its headers (same flags) are kept
        if (not force and not ptxas_info and same_flags and os.path.exists(obj) and
                os.path.getmtime(obj) >= _src_mtime(src)):
            return obj
        cmd = [NVCC] + FLAGS + extra + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose or ptxas_info:
            sys.stderr.write(r.stderr)
        return obj

    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, sources()))
    with open(stamp, "w") as f:
        f.write(flags_key)
    tmp = OUT + ".tmp%d" % os.getpid()
    cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
           "-o", tmp] + objs
    subprocess.check_call(cmd)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                ptxas_info="--ptxas" in sys.argv))
