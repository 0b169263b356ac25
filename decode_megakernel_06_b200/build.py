"""Build ``libmk.so`` (the C-ABI decode-step library) in-tree for sm_100a.

Each ``.cu`` file is compiled to an object with nvcc (in parallel; the step
kernels twice, with and without the timeline trace), then
linked into a shared library next to this file.  Only the ``MK_API``
symbols of ``include/mk.h`` are exported.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmk.so")
# (source, object name, extra flags): the step kernels are built twice, the
# second time with the timeline trace compiled in.
UNITS = [("mk_kernel.cu", "mk_kernel", []), ("mk_kernel.cu", "mk_kernel_trace", ["-DMK_TRACE=1"]),
         ("mk_api.cu", "mk_api", []), ("mk_wide.cu", "mk_wide", []), ("mk_sample.cu", "mk_sample", []),
         ("mk_probe.cu", "mk_probe", [])]
SOURCES = sorted({u[0] for u in UNITS})
HEADERS = ["mk_internal.h", os.path.join("..", "..", "include", "mk.h")]

NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-Xptxas", "-v",
         "-diag-suppress", "177"]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(unit) -> str:
    src, name, extra = unit
    obj = os.path.join(BUILD, name + ".o")
    deps = [os.path.join(CSRC, src)] + [os.path.join(CSRC, h) for h in HEADERS]
    if _stale(obj, deps):
        cmd = [NVCC, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        log = os.path.join(BUILD, name + ".ptxas.txt")
        with open(log, "w") as fh:
            fh.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src} ({name}):\n{r.stderr[-4000:]}")
    return obj


def build(force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    if force:
        for _, name, _ in UNITS:
            o = os.path.join(BUILD, name + ".o")
            if os.path.exists(o):
                os.remove(o)
    with cf.ThreadPoolExecutor(len(UNITS)) as ex:
        objs = list(ex.map(_compile, UNITS))
    if _stale(LIB, objs):
        cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
               "-o", LIB + ".tmp", "-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
