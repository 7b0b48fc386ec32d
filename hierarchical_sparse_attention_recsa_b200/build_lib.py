"""Compile the RecSA CUDA library (librecsa.so) in-tree for sm_100a.

Run as ``python -m hierarchical_sparse_attention_recsa_b200.build_lib``; the
shared library lands next to this file, where the binding loads it from.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librecsa.so")
OBJ_DIR = os.path.join(HERE, "_build")
SOURCES = ["recsa_api.cu", "build.cu", "attend.cu", "decode_cluster.cu",
           "prefill_warp.cu", "prefill_window.cu",
           "prefill_static.cu", "zha_attend.cu", "prefill_leaf.cu",
           "prefill_tree.cu", "window_tc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(HERE, "..", "include", "recsa.h"))
    return [h for h in hs if os.path.exists(h)]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in sources() + headers())


def _compile(src: str, obj: str, verbose: bool) -> None:
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
           "-c", "-o", obj + ".tmp", src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(obj + ".tmp", obj)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every translation unit (in parallel, only those older than their
    source or a header) and link librecsa.so."""
    if not force and not needs_build():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    newest_header = max(os.path.getmtime(h) for h in headers())
    jobs = []
    objs = []
    for src in sources():
        obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or \
                os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header):
            jobs.append((src, obj))
    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    if jobs:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            for f in [ex.submit(_compile, s_, o_, verbose) for s_, o_ in jobs]:
                f.result()
    tmp = LIB + ".tmp"
    subprocess.run([nvcc_path(), *ARCH, "-shared", "-cudart", "shared", "-o", tmp, *objs],
                   check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
