"""Builds libzdit.so (the sm_100a CUDA library behind include/zdit.h) in-tree.

Each .cu file under csrc/ is compiled for sm_100a with nvcc, in parallel, then the
objects are linked into a shared library next to this file.  Rebuilds only what is
older than its sources, or everything when the compile flags changed.

ZDIT_WAIT_LIMIT_MS in the environment sets the limit of the kernels' bounded waits
(default 2000 ms; see include/zdit.h).
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libzdit.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, extra_flags=()) -> str:
    os.makedirs(OBJ, exist_ok=True)
    nvcc = _nvcc()
    extra_flags = list(extra_flags)
    if os.environ.get("ZDIT_WAIT_LIMIT_MS"):
        extra_flags.append(f"-DZDIT_WAIT_LIMIT_MS={int(os.environ['ZDIT_WAIT_LIMIT_MS'])}")
    # objects built with other code-affecting flags are stale (-Xptxas -v only reports)
    stamp = os.path.join(OBJ, "flags.txt")
    code_flags = " ".join(f for f in extra_flags if f.startswith("-D"))
    if not os.path.exists(stamp) or open(stamp).read() != code_flags:
        for o in glob.glob(os.path.join(OBJ, "*.o")):
            os.remove(o)
        with open(stamp, "w") as fh:
            fh.write(code_flags)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    jobs = []
    for src in sources:
        obj = os.path.join(OBJ, os.path.basename(src) + ".o")
        if _stale(obj, [src] + headers):
            cmd = [nvcc, *ARCH, *FLAGS, *extra_flags, "-c", src, "-o", obj]
            jobs.append((src, cmd))

    def run(job):
        src, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr)
        return src

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(run, jobs))
    objs = [os.path.join(OBJ, os.path.basename(s) + ".o") for s in sources]
    if jobs or _stale(LIB, objs):
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    import sys
    print(build(verbose="-v" in sys.argv, extra_flags=["-Xptxas", "-v"] if "-v" in sys.argv else []))
