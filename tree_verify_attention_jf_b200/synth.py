"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle's tests.

This module only draws random numbers and lays them out; it holds none of the method's
arithmetic (no masks, no softmax, no scores, no tree search, no acceptance walk).  Every
generator takes an explicit seed and uses numpy's PCG64 (``numpy.random.default_rng``), so the
oracle and the GPU see identical inputs.

Workload shapes follow the JetFlow/JetSpec pages: the Qwen3-8B and Qwen3-30B-A3B attention
shapes and the 151936-token vocabulary ("4. Experimental results"), a tree-causal verify pass over
a paged KV cache ("2. Method: tree-causal attention mask", "3. Contributions: vLLM integration"),
and best-first trees of up to 256 tokens ("2. Method: tree construction").  The benchmark suites the
pages measure on are not available here; these seeded tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

PAGE_SIZE = 16
HEAD_DIM = 128
VOCAB = 151936


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even) and return them as float32."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def to_bf16_tensor(x: np.ndarray) -> torch.Tensor:
    """float32 array holding bf16-representable values -> torch.bfloat16 CPU tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# ----------------------------------------------------------------------------------------------
# Trees (topological parent lists; -1 = child of the cached prefix / the tree root's parent)
# ----------------------------------------------------------------------------------------------

def uniform_parent_tree(rng: np.random.Generator, n: int, max_depth: int) -> np.ndarray:
    """parent[i] drawn uniformly from {-1, 0..i-1}, restricted so that no node is deeper than
    ``max_depth`` (a node whose parent is -1 has depth 1).  Returns int32[n]."""
    parent = np.empty(n, dtype=np.int32)
    depth = np.empty(n, dtype=np.int32)
    for i in range(n):
        allowed = [-1] + [j for j in range(i) if depth[j] < max_depth]
        p = allowed[int(rng.integers(len(allowed)))]
        parent[i] = p
        depth[i] = 1 if p < 0 else depth[p] + 1
    return parent


def bushy_tree(rng: np.random.Generator, n: int, max_branch: int = 4, max_levels: int = 16) -> np.ndarray:
    """A rooted tree: node 0 is the root (parent -1); each later node attaches to a uniformly drawn
    earlier node that still has fewer than ``max_branch`` children and lies fewer than
    ``max_levels`` edges below the root.  Returns int32[n] in topological order."""
    parent = np.full(n, -1, dtype=np.int32)
    level = np.zeros(n, dtype=np.int32)
    nchild = np.zeros(n, dtype=np.int32)
    for i in range(1, n):
        cand = [j for j in range(i) if nchild[j] < max_branch and level[j] < max_levels]
        p = cand[int(rng.integers(len(cand)))]
        parent[i] = p
        level[i] = level[p] + 1
        nchild[p] += 1
    return parent


def chain_tree(n: int) -> np.ndarray:
    """0 <- 1 <- 2 ... : node 0 hangs off the prefix, every later node off the previous one."""
    return np.arange(-1, n - 1, dtype=np.int32)


def star_tree(n: int) -> np.ndarray:
    """Every node hangs directly off the prefix."""
    return np.full(n, -1, dtype=np.int32)


# ----------------------------------------------------------------------------------------------
# Paged KV cache
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class AttentionInputs:
    q: np.ndarray             # float32 [T, Hq, D], bf16-representable
    k_cache: np.ndarray       # float32 [num_pages, PAGE, Hkv, D], bf16-representable
    v_cache: np.ndarray       # float32 [num_pages, PAGE, Hkv, D]
    block_table: np.ndarray   # int32 [B, max_pages]
    prefix_lens: np.ndarray   # int32 [B]
    tree_offsets: np.ndarray  # int32 [B+1]
    parent: np.ndarray        # int32 [T]  (local indices, -1 = child of the prefix)
    sm_scale: float
    num_q_heads: int
    num_kv_heads: int

    @property
    def batch(self) -> int:
        return int(self.prefix_lens.shape[0])

    @property
    def total_nodes(self) -> int:
        return int(self.tree_offsets[-1])


def page_pool(rng: np.random.Generator, pages_per_seq: list[int], interleave: bool,
              extra_pages: int = 0) -> tuple[np.ndarray, int]:
    """Physical page ids for each sequence's logical pages.  ``interleave`` draws one permutation
    over the whole pool (all sequences' pages randomly interleaved); otherwise sequence b owns a
    contiguous physical range, permuted within itself.  Returns (block_table[B, max_pages], pool size).
    Unused block-table entries are set to -1."""
    total = int(sum(pages_per_seq)) + extra_pages
    maxp = max(1, max(pages_per_seq) if pages_per_seq else 1)
    bt = np.full((len(pages_per_seq), maxp), -1, dtype=np.int32)
    if interleave:
        perm = rng.permutation(total).astype(np.int32)
        pos = 0
        for b, n in enumerate(pages_per_seq):
            bt[b, :n] = perm[pos:pos + n]
            pos += n
    else:
        base = 0
        for b, n in enumerate(pages_per_seq):
            bt[b, :n] = base + rng.permutation(n).astype(np.int32)
            base += n
    return bt, total


def attention_inputs(seed: int, num_q_heads: int, num_kv_heads: int, prefix_lens: list[int],
                     parents: list[np.ndarray], interleave: bool = False, scale: float = 0.5,
                     extra_pages: int = 0, head_dim: int = HEAD_DIM) -> AttentionInputs:
    """q, k, v ~ bf16(N(0,1) * scale); tree node i of sequence b has its K/V at logical slot
    prefix_lens[b] + i of that sequence's pages."""
    rng = np.random.default_rng(seed)
    B = len(prefix_lens)
    ns = [int(p.shape[0]) for p in parents]
    pages_per_seq = [(int(P) + n + PAGE_SIZE - 1) // PAGE_SIZE for P, n in zip(prefix_lens, ns)]
    bt, num_pages = page_pool(rng, pages_per_seq, interleave, extra_pages)
    num_pages = max(num_pages, 1)
    T = int(sum(ns))
    offs = np.zeros(B + 1, dtype=np.int32)
    offs[1:] = np.cumsum(ns)
    q = bf16_round(rng.standard_normal((T, num_q_heads, head_dim), dtype=np.float32) * scale)
    k = bf16_round(rng.standard_normal((num_pages, PAGE_SIZE, num_kv_heads, head_dim), dtype=np.float32) * scale)
    v = bf16_round(rng.standard_normal((num_pages, PAGE_SIZE, num_kv_heads, head_dim), dtype=np.float32) * scale)
    parent = np.concatenate(parents).astype(np.int32) if T else np.zeros(0, np.int32)
    return AttentionInputs(q=q, k_cache=k, v_cache=v, block_table=bt,
                           prefix_lens=np.asarray(prefix_lens, dtype=np.int32), tree_offsets=offs,
                           parent=parent, sm_scale=1.0 / float(np.sqrt(head_dim)),
                           num_q_heads=num_q_heads, num_kv_heads=num_kv_heads)


def e4m3_cache(values: np.ndarray, scale: float) -> np.ndarray:
    """8-bit E4M3 codes (uint8) of a synthetic cache: values / scale converted by torch's float8_e4m3fn cast
    (round to nearest even).  Values must stay within +-448 * scale."""
    x = np.ascontiguousarray(values, dtype=np.float32) / np.float32(scale)
    if np.abs(x).max(initial=0.0) > 448.0:
        raise ValueError("values / scale exceed the E4M3 range (448)")
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def plant_tree_values(inp: AttentionInputs, magnitude: float = 8.0, base_scale: float = 0.5,
                      seed: int = 0) -> AttentionInputs:
    """Planted-V probe: every tree slot j of every sequence gets V = magnitude * e_(j mod D) in each
    kv head, all prefix slots get bf16(N(0, base_scale)) values.  Each ancestor's contribution then
    lands in its own coordinate of the output."""
    rng = np.random.default_rng(seed)
    v = bf16_round(rng.standard_normal(inp.v_cache.shape, dtype=np.float32) * base_scale)
    D = v.shape[-1]
    for b in range(inp.batch):
        P = int(inp.prefix_lens[b])
        n = int(inp.tree_offsets[b + 1] - inp.tree_offsets[b])
        for j in range(n):
            t = P + j
            page = int(inp.block_table[b, t // PAGE_SIZE])
            v[page, t % PAGE_SIZE] = 0.0
            v[page, t % PAGE_SIZE, :, j % D] = magnitude
    return dataclasses.replace(inp, v_cache=v)


# ----------------------------------------------------------------------------------------------
# Draft and target logits
# ----------------------------------------------------------------------------------------------

def draft_logits(seed: int, batch: int, depths: int, vocab: int, sigma: float = 2.0,
                 plant: int = 8) -> tuple[np.ndarray, np.ndarray]:
    """fp32 [batch, depths, vocab] ~ N(0, sigma^2), with a planted Zipf-peaked head per row: ``plant``
    distinct token ids t_1..t_plant get x[t_r] = max(noise row) + c - s*ln(r), with c ~ U(4, 10) and
    s ~ U(0.8, 1.5) drawn per row.  Also returns seeded root tokens int32[batch]."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, depths, vocab), dtype=np.float32) * np.float32(sigma)
    if plant:
        for b in range(batch):
            for k in range(depths):
                row = x[b, k]
                toks = rng.choice(vocab, size=min(plant, vocab), replace=False)
                c = rng.uniform(4.0, 10.0)
                s = rng.uniform(0.8, 1.5)
                top = float(row.max())
                for r, t in enumerate(toks, start=1):
                    row[t] = np.float32(top + c - s * np.log(r))
    roots = rng.integers(0, vocab, size=batch).astype(np.int32)
    return x, roots


def path_logits(seed: int, path: tuple, vocab: int, sigma: float = 2.0, plant: int = 8) -> np.ndarray:
    """Draft logits fp32 [vocab] at one tree node, drawn from a generator seeded by ``seed`` and the node's root
    path (its token ids, root first), so that the same path always gets the same row: the stand-in for a draft
    head whose output at a node depends on that node's path.  Same recipe as :func:`draft_logits` rows:
    N(0, sigma^2) with ``plant`` distinct ids lifted to rowmax + c - s*ln(r), c ~ U(4, 10), s ~ U(0.8, 1.5)."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), len(path)] + [int(t) for t in path]))
    x = rng.standard_normal(vocab, dtype=np.float32) * np.float32(sigma)
    if plant:
        toks = rng.choice(vocab, size=min(plant, vocab), replace=False)
        c = rng.uniform(4.0, 10.0)
        s = rng.uniform(0.8, 1.5)
        top = float(x.max())
        for r, t in enumerate(toks, start=1):
            x[t] = np.float32(top + c - s * np.log(r))
    return x


def target_logits_with_path(seed: int, parent: np.ndarray, token: np.ndarray, vocab: int,
                            path_len: Optional[list[int]] = None, sigma: float = 2.0,
                            lift: float = 4.0) -> tuple[np.ndarray, list[list[int]]]:
    """Target logits fp32 [B, N, vocab] ~ N(0, sigma^2) that agree with a given tree along a seeded
    path.  ``parent``/``token`` are [B, N] with node 0 the root.  For each sequence a path length
    L ~ U{1..16} is drawn (or taken from ``path_len``); an end node at depth L is drawn among the
    tree's nodes at that depth (if none exists, the deepest node shallower than L is used).  At the
    root and at every path node the logit of the next path node's token is lifted to rowmax + lift;
    at the end node a token that none of its children carries is lifted the same way.

    Returns the logits and, per sequence, the planted node path [0, ..., end]."""
    rng = np.random.default_rng(seed)
    B, N = parent.shape
    x = rng.standard_normal((B, N, vocab), dtype=np.float32) * np.float32(sigma)
    paths = []
    for b in range(B):
        par = parent[b]
        lvl = np.zeros(N, dtype=np.int64)
        for i in range(1, N):
            lvl[i] = lvl[par[i]] + 1
        L = int(rng.integers(1, 17)) if path_len is None else int(path_len[b])
        cand = np.nonzero(lvl == L)[0]
        if cand.size == 0:
            shallower = np.nonzero(lvl < L)[0]
            deepest = lvl[shallower].max()
            cand = np.nonzero(lvl == deepest)[0]
        end = int(cand[int(rng.integers(cand.size))])
        path = [end]
        while path[-1] != 0:
            path.append(int(par[path[-1]]))
        path.reverse()
        for a, c in zip(path[:-1], path[1:]):
            row = x[b, a]
            row[token[b, c]] = np.float32(float(row.max()) + lift)
        row = x[b, end]
        child_toks = set(int(token[b, c]) for c in range(N) if par[c] == end)
        t = int(rng.integers(vocab))
        while t in child_toks:
            t = int(rng.integers(vocab))
        row[t] = np.float32(float(row.max()) + lift)
        paths.append(path)
    return x, paths
