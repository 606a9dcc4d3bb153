"""ctypes binding of libjf.so (include/jf.h).  Argument marshalling only: every step of the hot path
runs in the library's CUDA kernels.  There is no fallback: if the library is missing or cannot be
loaded, :func:`lib` raises."""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjf.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libjf_debug.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "jf.h")
DEBUG_HEADER = os.path.join(os.path.dirname(_PKG), "include", "jf_debug.h")

JF_OK = 0
JF_ERR_INVALID_ARG = 1
JF_ERR_UNSUPPORTED = 2
JF_ERR_CUDA = 3
JF_ERR_DEVICE_CHECK = 4
JF_ERR_TIMEOUT = 5

_c_i32p = ctypes.c_void_p  # device pointers travel as integers
_lib = None


class JFError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def lib() -> ctypes.CDLL:
    """The loaded libjf.so.  Raises if it was not built (``python -m tree_verify_attention_jf_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _load(LIB_PATH)
    return _lib


_debug_lib = None


def debug_lib() -> ctypes.CDLL:
    """The debug build libjf_debug.so (50 ms wait limit, jf_debug.h hooks), for the failure-detection tests."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
        _debug_lib.jf_debug_hold.argtypes = [ctypes.c_int]
        _debug_lib.jf_debug_hold.restype = ctypes.c_int
    return _debug_lib


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m tree_verify_attention_jf_b200.build`")
    L = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.jf_status_string.argtypes = [i]
    L.jf_status_string.restype = ctypes.c_char_p
    L.jf_version.argtypes = []
    L.jf_version.restype = i
    L.jf_tree_attention_workspace_size.argtypes = [i, i, i, i]
    L.jf_tree_attention_workspace_size.restype = sz
    L.jf_tree_attention.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp, sz, vp, vp]
    L.jf_tree_attention.restype = i
    L.jf_tree_attention_fp8.argtypes = [vp, vp, vp, f, f, vp, i, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp, vp, sz,
                                        vp, vp]
    L.jf_tree_attention_fp8.restype = i
    L.jf_build_tree_workspace_size.argtypes = [i, i, i, i]
    L.jf_build_tree_workspace_size.restype = sz
    L.jf_build_tree.argtypes = [vp, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp, sz, vp, vp]
    L.jf_build_tree.restype = i
    L.jf_expand_frontier_state_size.argtypes = [i, i, i]
    L.jf_expand_frontier_state_size.restype = sz
    L.jf_expand_frontier_workspace_size.argtypes = [i, i, i]
    L.jf_expand_frontier_workspace_size.restype = sz
    L.jf_expand_frontier.argtypes = [vp, vp, i, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp, vp]
    L.jf_expand_frontier.restype = i
    L.jf_accept.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp, vp]
    L.jf_accept.restype = i
    L.jf_commit_kv.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, vp]
    L.jf_commit_kv.restype = i
    L.jf_tree_kv_append.argtypes = [vp, vp, vp, vp, vp, vp, i, vp, vp, vp, i, i, i, i, i, i, i, f, vp, vp]
    L.jf_tree_kv_append.restype = i
    return L


def status_string(code: int) -> str:
    return lib().jf_status_string(int(code)).decode()


def declared_functions(header: str = HEADER) -> list[str]:
    """Names of the functions a header declares (used to check the library's exports)."""
    text = open(header).read()
    return sorted(set(re.findall(r"JF_API\s+[\w\s\*]+?\b(jf_\w+)\s*\(", text)))


def check(fn: str, code: int) -> None:
    if code != JF_OK:
        raise JFError(fn, code)
