"""Build libmad.so (the CUDA library behind include/mad.h) in-tree with nvcc.

Compiles every .cu / .cpp under csrc/ for sm_100a only and links a shared
library with the CUDA runtime linked statically, so the library needs no
CUDA toolkit at run time beyond the driver.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmad.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", f"-I{os.path.join(HERE, '..', 'include')}"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps():
    return _sources() + _headers()


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(HERE, "..", "include", "mad.h")]


def _compile(src: str, extra: list[str], bdir: str, force: bool) -> str:
    obj = os.path.join(bdir, os.path.basename(src) + ".o")
    # an object newer than its source and every header is reused (every unit
    # is treated as depending on every header)
    if not force and os.path.exists(obj):
        t = os.path.getmtime(obj)
        if all(os.path.getmtime(d) <= t for d in [src, *_headers()]):
            return obj
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, extra: list[str] | None = None, jobs: int | None = None,
          out: str | None = None, build_dir: str | None = None) -> str:
    """Compile and link; `extra` nvcc flags and `out` select a variant build."""
    lib = out or LIB
    if not force and not extra and out is None and up_to_date():
        return LIB
    bdir = build_dir or BUILD
    os.makedirs(bdir, exist_ok=True)
    extra = list(extra or [])
    # variant builds (extra flags) compile everything into their own folder
    fresh = force or bool(extra)
    srcs = _sources()
    # the longest units first, so that they do not finish last
    srcs.sort(key=lambda s: -os.path.getsize(s) - (1 << 20) * s.endswith("_d3.cu"))
    with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, bdir, fresh), srcs))
    tmp = lib + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    extra = sys.argv[1:]
    print(build(force=True, extra=extra))
