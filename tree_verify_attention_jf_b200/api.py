"""Torch-facing calls of the tree-verify hot path.  PyTorch only supplies device memory and the stream;
each function checks dtypes/shapes/devices, passes raw pointers to libjf.so (:mod:`._lib`) and returns.
Nothing here computes any part of the method."""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib

PAGE_SIZE = 16
HEAD_DIM = 128


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, device: torch.device) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must live on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class AttentionWorkspace:
    """Scratch for :func:`tree_attention` (partial results of split work units).  One per stream;
    needs no initialisation and is reusable across calls."""

    def __init__(self, device: torch.device):
        n = _lib.lib().jf_tree_attention_workspace_size(0, 0, 0, 0)
        self.buf = torch.empty(n, dtype=torch.uint8, device=device)

    @property
    def nbytes(self) -> int:
        return self.buf.numel()


def tree_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                   prefix_lens: torch.Tensor, tree_offsets: torch.Tensor, parent: torch.Tensor, sm_scale: float,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   workspace: Optional[AttentionWorkspace] = None, dev_status: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """jf_tree_attention: q bf16 [T, Hq, 128]; k/v_cache bf16 [pages, 16, Hkv, 128]; block_table int32
    [B, max_pages]; prefix_lens int32 [B]; tree_offsets int32 [B+1]; parent int32 [T].  Returns out."""
    dev = q.device
    T, Hq, D = q.shape
    num_pages, page, Hkv, D2 = k_cache.shape
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    for name, t in (("block_table", block_table), ("prefix_lens", prefix_lens), ("tree_offsets", tree_offsets),
                    ("parent", parent)):
        _need(t, name, torch.int32, dev)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    B = prefix_lens.numel()
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if workspace is None:
        workspace = AttentionWorkspace(dev)
    code = _lib.lib().jf_tree_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1] if block_table.dim() == 2 else 0,
        _ptr(prefix_lens), _ptr(tree_offsets), _ptr(parent), B, T, Hq, Hkv, D, page, num_pages, float(sm_scale),
        _ptr(out), _ptr(lse), _ptr(workspace.buf), workspace.nbytes, _ptr(dev_status), _stream(stream))
    _lib.check("jf_tree_attention", code)
    return out


def tree_attention_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: float,
                       v_scale: float, block_table: torch.Tensor, prefix_lens: torch.Tensor, tree_offsets: torch.Tensor,
                       parent: torch.Tensor, sm_scale: float, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, workspace: Optional[AttentionWorkspace] = None,
                       dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """jf_tree_attention_fp8: as :func:`tree_attention`, with k/v_cache uint8 E4M3 codes [pages, 16, Hkv, 128]
    standing for decode(code) * k_scale / v_scale.  Returns out (bf16)."""
    dev = q.device
    T, Hq, D = q.shape
    num_pages, page, Hkv, D2 = k_cache.shape
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.uint8, dev)
    _need(v_cache, "v_cache", torch.uint8, dev)
    for name, t in (("block_table", block_table), ("prefix_lens", prefix_lens), ("tree_offsets", tree_offsets),
                    ("parent", parent)):
        _need(t, name, torch.int32, dev)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    B = prefix_lens.numel()
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if workspace is None:
        workspace = AttentionWorkspace(dev)
    code = _lib.lib().jf_tree_attention_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale), _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else 0, _ptr(prefix_lens), _ptr(tree_offsets), _ptr(parent), B,
        T, Hq, Hkv, D, page, num_pages, float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace.buf), workspace.nbytes,
        _ptr(dev_status), _stream(stream))
    _lib.check("jf_tree_attention_fp8", code)
    return out


def build_tree_workspace(batch: int, depths: int, vocab: int, topk: int, device) -> torch.Tensor:
    n = _lib.lib().jf_build_tree_workspace_size(batch, depths, vocab, topk)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def build_tree(draft_logits: torch.Tensor, root_tokens: torch.Tensor, topk: int, budget: int, max_depth: int,
               workspace: Optional[torch.Tensor] = None, out: Optional[dict] = None,
               dev_status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """jf_build_tree: draft_logits fp32 [B, depths, V], root_tokens int32 [B] -> dict of parent, token,
    depth (int32 [B, budget]) and score (fp32 [B, budget])."""
    dev = draft_logits.device
    B, depths, V = draft_logits.shape
    _need(draft_logits, "draft_logits", torch.float32, dev)
    _need(root_tokens, "root_tokens", torch.int32, dev)
    if out is None:
        out = dict(parent=torch.empty(B, budget, dtype=torch.int32, device=dev),
                   token=torch.empty(B, budget, dtype=torch.int32, device=dev),
                   score=torch.empty(B, budget, dtype=torch.float32, device=dev),
                   depth=torch.empty(B, budget, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = build_tree_workspace(B, depths, V, topk, dev)
    code = _lib.lib().jf_build_tree(
        _ptr(draft_logits), _ptr(root_tokens), B, depths, V, topk, budget, max_depth, _ptr(out["parent"]),
        _ptr(out["token"]), _ptr(out["score"]), _ptr(out.get("depth")), _ptr(workspace), workspace.numel(),
        _ptr(dev_status), _stream(stream))
    _lib.check("jf_build_tree", code)
    return out


class FrontierTree:
    """A batch of trees grown round by round with :func:`expand_frontier`: the tree arrays (parent, token, depth
    int32 [B, budget], score fp32 [B, budget]), the node counts and frontier starts (int32 [B]) and the state the
    library carries between rounds.  ``reset()`` starts new trees (the next round creates the roots)."""

    def __init__(self, batch: int, budget: int, topk: int, device):
        self.batch, self.budget, self.topk = batch, budget, topk
        self.parent = torch.full((batch, budget), -1, dtype=torch.int32, device=device)
        self.token = torch.zeros(batch, budget, dtype=torch.int32, device=device)
        self.depth = torch.zeros(batch, budget, dtype=torch.int32, device=device)
        self.score = torch.zeros(batch, budget, dtype=torch.float32, device=device)
        self.num_nodes = torch.zeros(batch, dtype=torch.int32, device=device)
        self.frontier_begin = torch.zeros(batch, dtype=torch.int32, device=device)
        n = _lib.lib().jf_expand_frontier_state_size(batch, budget, topk)
        self.state = torch.empty(max(n, 256), dtype=torch.uint8, device=device)

    def reset(self) -> None:
        self.num_nodes.zero_()
        self.frontier_begin.zero_()


def expand_frontier_workspace(batch: int, frontier_rows: int, vocab: int, device) -> torch.Tensor:
    n = _lib.lib().jf_expand_frontier_workspace_size(batch, frontier_rows, vocab)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def expand_frontier(node_logits: torch.Tensor, root_tokens: torch.Tensor, tree: FrontierTree, max_depth: int,
                    width: int, workspace: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                    stream=None) -> FrontierTree:
    """jf_expand_frontier: one round.  node_logits fp32 [B, F, V] (row j of sequence b = the draft head's logits at
    node tree.frontier_begin[b] + j); root_tokens int32 [B].  Updates ``tree`` in place and returns it."""
    dev = node_logits.device
    B, F, V = node_logits.shape
    _need(node_logits, "node_logits", torch.float32, dev)
    _need(root_tokens, "root_tokens", torch.int32, dev)
    if B != tree.batch:
        raise ValueError("node_logits and tree have different batch sizes")
    if workspace is None:
        workspace = expand_frontier_workspace(B, F, V, dev)
    code = _lib.lib().jf_expand_frontier(
        _ptr(node_logits), _ptr(root_tokens), B, F, V, tree.topk, tree.budget, max_depth, width, _ptr(tree.parent),
        _ptr(tree.token), _ptr(tree.score), _ptr(tree.depth), _ptr(tree.num_nodes), _ptr(tree.frontier_begin),
        _ptr(tree.state), tree.state.numel(), _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream))
    _lib.check("jf_expand_frontier", code)
    return tree


def accept(token: torch.Tensor, parent: torch.Tensor, target_logits: torch.Tensor, max_depth: int,
           out: Optional[dict] = None, dev_status: Optional[torch.Tensor] = None, stream=None) -> dict:
    """jf_accept: token, parent int32 [B, N]; target_logits fp32 [B, N, V] -> dict of accepted_len int32 [B],
    path int32 [B, max_depth + 1], bonus int32 [B]."""
    dev = target_logits.device
    B, N, V = target_logits.shape
    _need(token, "token", torch.int32, dev)
    _need(parent, "parent", torch.int32, dev)
    _need(target_logits, "target_logits", torch.float32, dev)
    if out is None:
        out = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=dev),
                   path=torch.empty(B, max_depth + 1, dtype=torch.int32, device=dev),
                   bonus=torch.empty(B, dtype=torch.int32, device=dev))
    code = _lib.lib().jf_accept(_ptr(token), _ptr(parent), _ptr(target_logits), B, N, V, max_depth,
                                _ptr(out["accepted_len"]), _ptr(out["path"]), _ptr(out["bonus"]), _ptr(dev_status),
                                _stream(stream))
    _lib.check("jf_accept", code)
    return out


def commit_kv(k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor, prefix_lens: torch.Tensor,
              tree_offsets: torch.Tensor, path: torch.Tensor, accepted_len: torch.Tensor,
              new_prefix_lens: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """jf_commit_kv: moves the accepted path's K/V (path, accepted_len as :func:`accept` returns them) to slots
    P + 1 .. P + L of each sequence, in place in k_cache / v_cache bf16 [pages, 16, Hkv, 128].  Returns
    new_prefix_lens int32 [B] (= P + L + 1; it may be prefix_lens itself)."""
    dev = k_cache.device
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    for t, name in ((block_table, "block_table"), (prefix_lens, "prefix_lens"), (tree_offsets, "tree_offsets"),
                    (path, "path"), (accepted_len, "accepted_len")):
        _need(t, name, torch.int32, dev)
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4:
        raise ValueError("k_cache and v_cache must both be [pages, 16, Hkv, 128]")
    num_pages, page, Hkv, D = k_cache.shape
    B = prefix_lens.shape[0]
    if path.dim() != 2 or path.shape[0] != B:
        raise ValueError("path must be [B, max_depth + 1]")
    if new_prefix_lens is None:
        new_prefix_lens = torch.empty(B, dtype=torch.int32, device=dev)
    _need(new_prefix_lens, "new_prefix_lens", torch.int32, dev)
    code = _lib.lib().jf_commit_kv(_ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
                                   _ptr(prefix_lens), _ptr(tree_offsets), _ptr(path), _ptr(accepted_len), B,
                                   path.shape[1] - 1, Hkv, D, page, num_pages, _ptr(new_prefix_lens), _ptr(dev_status),
                                   _stream(stream))
    _lib.check("jf_commit_kv", code)
    return new_prefix_lens


def tree_kv_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_table: torch.Tensor, prefix_lens: torch.Tensor, tree_offsets: torch.Tensor,
                   depth: torch.Tensor, rope_theta: float, q: Optional[torch.Tensor] = None,
                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """jf_tree_kv_append: k_new, v_new bf16 [T, Hkv, 128] of the tree tokens go to cache slots P + j of their
    sequences, K rotated at position P + depth; q bf16 [T, Hq, 128], when given, is rotated in place."""
    dev = k_cache.device
    for t, name in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, name, torch.bfloat16, dev)
    for t, name in ((block_table, "block_table"), (prefix_lens, "prefix_lens"), (tree_offsets, "tree_offsets"),
                    (depth, "depth")):
        _need(t, name, torch.int32, dev)
    if q is not None:
        _need(q, "q", torch.bfloat16, dev)
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4 or k_new.shape != v_new.shape or k_new.dim() != 3:
        raise ValueError("caches must be [pages, 16, Hkv, 128] and k_new / v_new [T, Hkv, 128]")
    num_pages, page, Hkv, D = k_cache.shape
    T = k_new.shape[0]
    if depth.numel() != T or (q is not None and q.shape[0] != T):
        raise ValueError("depth must have one entry per tree node, q one row per node")
    B = prefix_lens.shape[0]
    code = _lib.lib().jf_tree_kv_append(_ptr(k_new), _ptr(v_new), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_table), block_table.shape[1], _ptr(prefix_lens), _ptr(tree_offsets),
                                        _ptr(depth), B, T, q.shape[1] if q is not None else 0, Hkv, D, page, num_pages,
                                        float(rope_theta), _ptr(dev_status), _stream(stream))
    _lib.check("jf_tree_kv_append", code)
