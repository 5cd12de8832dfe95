"""Builds libpagedkv.so in-tree for sm_100a with nvcc (no JIT, no torch extension).

    python -m paged_kv_cache_393_b200.build [--force] [--ptxas-verbose]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build", "pagedkv")
LIB = os.path.join(HERE, "libpagedkv.so")

SOURCES = ["api.cu", "attention_simt.cu", "attention_mma.cu", "split_merge.cu", "cache_ops.cu",
           "block_manager.cpp", "noalloc.cu", "prefix_groups.cpp"]
HEADERS = [os.path.join(CSRC, h) for h in ("common.cuh", "kernels.h")] + [
    os.path.join(ROOT, "include", "pagedkv.h")]

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "-Xcompiler", "-fvisibility=hidden"]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, ptxas_verbose: bool) -> str:
    obj = os.path.join(BUILD, src + ".o")
    cmd = [NVCC] + FLAGS + ["-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src), "-o", obj]
    if ptxas_verbose and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed on %s:\n%s%s" % (src, res.stdout, res.stderr))
    if ptxas_verbose:
        sys.stderr.write(res.stderr)
    return obj


def source_digest() -> str:
    """Hash of every source, header and flag that goes into the library."""
    h = hashlib.sha256(" ".join(FLAGS).encode())
    for path in [os.path.join(CSRC, s) for s in SOURCES] + HEADERS:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + b"\0" + f.read())
    return h.hexdigest()


def build(force: bool = False, ptxas_verbose: bool = False, verbose: bool = False) -> str:
    digest = source_digest()
    stamp = LIB + ".sha256"
    if not force and not ptxas_verbose and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                if verbose:
                    print("up to date:", LIB)
                return LIB
    os.makedirs(BUILD, exist_ok=True)
    hdr_time = _newest(HEADERS)
    todo = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src + ".o")
        if force or ptxas_verbose or not os.path.exists(obj) or os.path.getmtime(obj) < max(
                hdr_time, os.path.getmtime(os.path.join(CSRC, src))):
            todo.append(src)
    if todo:
        with cf.ThreadPoolExecutor(max(1, min(len(todo), os.cpu_count() or 4))) as ex:
            list(ex.map(lambda s: _compile(s, ptxas_verbose), todo))
    objs = [os.path.join(BUILD, s + ".o") for s in SOURCES]
    if todo or not os.path.exists(LIB) or os.path.getmtime(LIB) < _newest(objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("link failed:\n%s%s" % (res.stdout, res.stderr))
        os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    if verbose:
        print("built", LIB, "(recompiled: %s)" % (", ".join(todo) or "nothing"))
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    build(force=a.force, ptxas_verbose=a.ptxas_verbose, verbose=True)
