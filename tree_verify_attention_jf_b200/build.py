"""Builds libjf.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension machinery), and the debug
build libjf_debug.so (JF_DEBUG: 50 ms wait limit and the jf_debug.h test hooks).

Usage: python -m tree_verify_attention_jf_b200.build [--debug] [-v]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libjf.so")
DEBUG_LIB = os.path.join(PKG, "libjf_debug.so")
SOURCES = ["jf_api.cu", "tree_attention.cu", "build_tree.cu", "frontier.cu", "accept.cu", "commit_kv.cu",
           "kv_append.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def needs_rebuild(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", f)
                                                               for f in os.listdir(os.path.join(ROOT, "include"))]
    return any(os.path.getmtime(d) > t for d in deps if os.path.isfile(d))


def build(verbose: bool = False, force: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not needs_rebuild(lib):
        return lib
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
           "-cudart", "static", "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DJF_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += list(extra or [])
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True, debug="--debug" in sys.argv))
