"""Build libsa.so (sm_100a) and the synthetic-input generator library in-tree.

    python -m cross_layer_shared_b200.build

Each .cu is compiled on its own (in parallel) and linked with nvcc; objects
go to _build/, the shared libraries next to the sources that use them.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsa.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "synth.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libsasynth.so")
HEADER = os.path.join(ROOT, "include", "sa.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr"]
SOURCES = ["api.cu", "indexer.cu", "indexer_prefill.cu", "topk.cu", "topk_split.cu", "topk_dynamic.cu", "attn.cu",
           "attn_small.cu", "attn_mid.cu", "union.cu", "kap.cu", "route_attn.cu", "cp.cu"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _deps() -> list:
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hdrs + [HEADER]


def _stale(out: str, inputs: list) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(i) > t for i in inputs)


def _compile(src: str, obj: str, extra=()) -> None:
    cmd = [nvcc(), *NVFLAGS, *extra, "-c", src, "-o", obj + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)


TIMELINE_LIB = os.path.join(PKG, "libsa_timeline.so")


def _build_lib(out: str, objdir: str, extra, force: bool) -> None:
    os.makedirs(objdir, exist_ok=True)
    deps = _deps()
    jobs = []
    objs = []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(objdir, s.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [src] + deps):
            jobs.append((src, obj))
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for f in [ex.submit(_compile, s, o, extra) for s, o in jobs]:
            f.result()
    if force or _stale(out, objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", out + ".tmp", *objs]
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)


def build_timeline(force: bool = False) -> str:
    """The tracing build (-DSA_TIMELINE, see csrc/timeline.cuh) as a library
    of its own; the library proper is not touched."""
    _build_lib(TIMELINE_LIB, os.path.join(BUILD, "timeline"), ("-DSA_TIMELINE",), force)
    return TIMELINE_LIB


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    _build_lib(LIB, BUILD, (), force)
    if force or _stale(SYNTH_LIB, [SYNTH_SRC]):
        cmd = [nvcc(), *NVFLAGS, "-shared", "-o", SYNTH_LIB + ".tmp", SYNTH_SRC]
        subprocess.check_call(cmd)
        os.replace(SYNTH_LIB + ".tmp", SYNTH_LIB)
    if verbose:
        print("built", LIB, "and", SYNTH_LIB)
    return LIB


def ptxas_report(source: str) -> str:
    """Registers / spills / shared memory of one source (ptxas -v)."""
    src = os.path.join(CSRC, source)
    r = subprocess.run([nvcc(), *NVFLAGS, "-Xptxas", "-v", "-c", src, "-o", os.devnull],
                       capture_output=True, text=True)
    return r.stderr


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    if "--ptxas" in sys.argv:
        for s in SOURCES:
            print(ptxas_report(s))
