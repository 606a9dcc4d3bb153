"""CPU checks of the C ABI: libjf.so loads, exports every function include/jf.h declares, and rejects
bad arguments on the host before any CUDA call (so these run without a GPU)."""

import pytest

from tree_verify_attention_jf_b200 import _lib

NULL = None


@pytest.fixture(scope="module")
def L():
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    names = _lib.declared_functions()
    assert set(names) == {"jf_status_string", "jf_version", "jf_tree_attention_workspace_size", "jf_tree_attention",
                          "jf_build_tree_workspace_size", "jf_build_tree", "jf_build_tree_noalloc", "jf_accept",
                          "jf_commit_kv", "jf_tree_kv_append", "jf_expand_frontier_state_size",
                          "jf_expand_frontier_workspace_size", "jf_expand_frontier", "jf_tree_attention_fp8"}
    for n in names:
        assert hasattr(L, n), n


def test_debug_build_exports_every_declared_symbol():
    D = _lib.debug_lib()
    for n in _lib.declared_functions() + _lib.declared_functions(_lib.DEBUG_HEADER):
        assert hasattr(D, n), n
    assert _lib.declared_functions(_lib.DEBUG_HEADER) == ["jf_debug_hold"]
    assert not hasattr(_lib.lib(), "jf_debug_hold")  # the release build has no test hooks


def test_status_strings(L):
    assert _lib.status_string(0) == "JF_OK"
    assert _lib.status_string(4) == "JF_ERR_DEVICE_CHECK"
    assert _lib.status_string(99) == "JF_ERR_UNKNOWN"
    assert L.jf_version() >= 10000


def attn(L, **over):
    a = dict(q=8, k=16, v=32, bt=64, maxp=4, pl=128, off=256, par=512, batch=1, T=16, hq=4, hkv=1, d=128, page=16,
             pages=8, scale=0.088, out=1024, lse=NULL, ws=4096, wsb=L.jf_tree_attention_workspace_size(1, 4, 1, 16),
             st=NULL, stream=NULL)
    a.update(over)
    return L.jf_tree_attention(a["q"], a["k"], a["v"], a["bt"], a["maxp"], a["pl"], a["off"], a["par"], a["batch"],
                               a["T"], a["hq"], a["hkv"], a["d"], a["page"], a["pages"], a["scale"], a["out"],
                               a["lse"], a["ws"], a["wsb"], a["st"], a["stream"])


def test_attention_host_validation(L):
    assert attn(L, d=64) == _lib.JF_ERR_UNSUPPORTED
    assert attn(L, page=32) == _lib.JF_ERR_UNSUPPORTED
    assert attn(L, hq=6, hkv=4) == _lib.JF_ERR_UNSUPPORTED
    assert attn(L, hq=96, hkv=3) == _lib.JF_ERR_UNSUPPORTED  # group 32 > 16
    assert attn(L, batch=-1) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, scale=0.0) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, scale=float("nan")) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, q=NULL) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, q=9) == _lib.JF_ERR_INVALID_ARG          # misaligned
    assert attn(L, wsb=100) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, ws=4097) == _lib.JF_ERR_INVALID_ARG
    assert attn(L, batch=5000) == _lib.JF_ERR_UNSUPPORTED
    assert attn(L, batch=0) == _lib.JF_OK                   # nothing to do, nothing launched
    assert attn(L, T=0) == _lib.JF_OK


def test_build_host_validation(L):
    def call(**o):
        a = dict(x=16, roots=32, B=2, depths=16, V=1000, topk=4, budget=256, md=16, par=64, tok=128, sc=256, dep=NULL,
                 ws=512, wsb=L.jf_build_tree_workspace_size(2, 16, 1000, 4), st=NULL, stream=NULL)
        a.update(o)
        return L.jf_build_tree(a["x"], a["roots"], a["B"], a["depths"], a["V"], a["topk"], a["budget"], a["md"],
                               a["par"], a["tok"], a["sc"], a["dep"], a["ws"], a["wsb"], a["st"], a["stream"])
    assert call(topk=9) == _lib.JF_ERR_UNSUPPORTED
    assert call(budget=2000) == _lib.JF_ERR_UNSUPPORTED
    assert call(md=17) == _lib.JF_ERR_INVALID_ARG
    assert call(topk=2, md=3, budget=16) == _lib.JF_ERR_INVALID_ARG   # full tree holds 15
    assert call(topk=2, md=3, budget=15, B=0) == _lib.JF_OK
    assert call(V=3, topk=4) == _lib.JF_ERR_INVALID_ARG
    assert call(wsb=10) == _lib.JF_ERR_INVALID_ARG
    assert call(x=NULL) == _lib.JF_ERR_INVALID_ARG
    assert call(B=0) == _lib.JF_OK


def test_accept_host_validation(L):
    def call(**o):
        a = dict(tok=16, par=32, x=64, B=2, N=256, V=1000, md=16, acc=128, path=256, bonus=512, st=NULL, stream=NULL)
        a.update(o)
        return L.jf_accept(a["tok"], a["par"], a["x"], a["B"], a["N"], a["V"], a["md"], a["acc"], a["path"],
                           a["bonus"], a["st"], a["stream"])
    assert call(N=0) == _lib.JF_ERR_INVALID_ARG
    assert call(N=2000) == _lib.JF_ERR_UNSUPPORTED
    assert call(md=-1) == _lib.JF_ERR_INVALID_ARG
    assert call(x=68 + 4) == _lib.JF_ERR_INVALID_ARG     # target logits not 16-byte aligned
    assert call(tok=NULL) == _lib.JF_ERR_INVALID_ARG
    assert call(B=0) == _lib.JF_OK


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_commit_kv_host_validation(L):
    def call(**o):
        a = dict(k=16, v=32, bt=64, maxp=4, pl=128, off=256, path=512, acc=1024, B=2, md=16, hkv=8, d=128, page=16,
                 pages=64, newp=2048, st=NULL, stream=NULL)
        a.update(o)
        return L.jf_commit_kv(a["k"], a["v"], a["bt"], a["maxp"], a["pl"], a["off"], a["path"], a["acc"], a["B"],
                              a["md"], a["hkv"], a["d"], a["page"], a["pages"], a["newp"], a["st"], a["stream"])
    assert call(d=64) == _lib.JF_ERR_UNSUPPORTED
    assert call(page=32) == _lib.JF_ERR_UNSUPPORTED
    assert call(hkv=65) == _lib.JF_ERR_UNSUPPORTED
    assert call(md=1024) == _lib.JF_ERR_UNSUPPORTED
    assert call(hkv=0) == _lib.JF_ERR_INVALID_ARG
    assert call(B=-1) == _lib.JF_ERR_INVALID_ARG
    assert call(md=-1) == _lib.JF_ERR_INVALID_ARG
    assert call(k=NULL) == _lib.JF_ERR_INVALID_ARG
    assert call(newp=NULL) == _lib.JF_ERR_INVALID_ARG
    assert call(k=24) == _lib.JF_ERR_INVALID_ARG         # not 16-byte aligned
    assert call(B=0) == _lib.JF_OK                       # nothing to do, nothing launched


def test_tree_kv_append_host_validation(L):
    def call(**o):
        a = dict(kn=16, vn=32, q=48, k=64, v=80, bt=96, maxp=4, pl=128, off=256, dep=512, B=2, T=20, hq=32, hkv=8,
                 d=128, page=16, pages=64, theta=1e6, st=NULL, stream=NULL)
        a.update(o)
        return L.jf_tree_kv_append(a["kn"], a["vn"], a["q"], a["k"], a["v"], a["bt"], a["maxp"], a["pl"], a["off"],
                                   a["dep"], a["B"], a["T"], a["hq"], a["hkv"], a["d"], a["page"], a["pages"],
                                   a["theta"], a["st"], a["stream"])
    assert call(d=64) == _lib.JF_ERR_UNSUPPORTED
    assert call(page=8) == _lib.JF_ERR_UNSUPPORTED
    assert call(B=2000) == _lib.JF_ERR_UNSUPPORTED
    assert call(theta=0.0) == _lib.JF_ERR_INVALID_ARG
    assert call(theta=float("inf")) == _lib.JF_ERR_INVALID_ARG
    assert call(hkv=0) == _lib.JF_ERR_INVALID_ARG
    assert call(hq=0) == _lib.JF_ERR_INVALID_ARG             # q given without heads
    assert call(kn=NULL) == _lib.JF_ERR_INVALID_ARG
    assert call(q=40) == _lib.JF_ERR_INVALID_ARG             # not 16-byte aligned
    assert call(T=0) == _lib.JF_OK                           # nothing to do, nothing launched
    assert call(B=0) == _lib.JF_OK


def test_expand_frontier_host_validation(L):
    # every pointer is null: a call that passed the size checks would stop at the null-pointer check
    def call(**over):
        a = dict(batch=2, rows=4, V=1000, topk=4, budget=64, max_depth=8, width=16)
        a.update(over)
        return L.jf_expand_frontier(None, None, a["batch"], a["rows"], a["V"], a["topk"], a["budget"],
                                    a["max_depth"], a["width"], None, None, None, None, None, None, None, 0, None, 0,
                                    None, None)
    assert call() == _lib.JF_ERR_INVALID_ARG  # null pointers
    assert call(batch=0) == _lib.JF_OK
    assert call(topk=9) == _lib.JF_ERR_UNSUPPORTED
    assert call(budget=257) == _lib.JF_ERR_UNSUPPORTED
    assert call(rows=257) == _lib.JF_ERR_UNSUPPORTED
    assert call(batch=300, rows=256) == _lib.JF_ERR_UNSUPPORTED  # grid rows > 65535
    assert call(topk=5, V=4) == _lib.JF_ERR_INVALID_ARG
    for bad in (dict(width=0), dict(max_depth=0), dict(rows=0), dict(budget=0), dict(topk=0), dict(V=0),
                dict(batch=-1)):
        assert call(**bad) == _lib.JF_ERR_INVALID_ARG, bad
    assert L.jf_expand_frontier_state_size(2, 64, 4) >= 2 * 64 * (8 + 4 * 8 + 4 * 4 + 4)
    assert L.jf_expand_frontier_workspace_size(2, 4, 4096) == 2 * 4 * 1 * 80


def test_tree_attention_fp8_host_validation(L):
    def call(**over):
        a = dict(ks=0.01, vs=0.02, batch=1, T=16, hq=4, hkv=1, d=128, page=16, pages=8, scale=0.088)
        a.update(over)
        return L.jf_tree_attention_fp8(None, None, None, a["ks"], a["vs"], None, 4, None, None, None, a["batch"],
                                       a["T"], a["hq"], a["hkv"], a["d"], a["page"], a["pages"], a["scale"], None, None,
                                       None, 0, None, None)
    assert call() == _lib.JF_ERR_INVALID_ARG  # null pointers
    for bad in (dict(ks=0.0), dict(vs=-1.0), dict(ks=float("inf")), dict(vs=float("nan")), dict(scale=0.0)):
        assert call(**bad) == _lib.JF_ERR_INVALID_ARG, bad
    assert call(d=64) == _lib.JF_ERR_UNSUPPORTED
    assert call(page=32) == _lib.JF_ERR_UNSUPPORTED
    assert call(hq=6, hkv=4) == _lib.JF_ERR_UNSUPPORTED
    assert call(batch=0) == _lib.JF_OK
