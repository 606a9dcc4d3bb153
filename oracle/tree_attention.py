"""Oracle: tree-causal attention over a paged KV cache (float64).

Definition followed ([JF] technical summary section 2, "tree-causal attention mask"): every node of
the draft tree attends to the original input prefix and to its own ancestors inside the tree, never
to its descendants or to unrelated sibling branches.  The same section states the branch
factorisation q(pi(v)|x) = prod_{u in pi(v)} q(y_u | x, h_x, pi_<u), i.e. node v is conditioned on
exactly the prefix plus the tokens on its own root path.

Readings where the pages are silent (each also listed in the design notes):
  * a node sees itself (its own slot is part of its path);
  * the tree nodes' K/V sit in the same paged cache, node i of sequence b at logical slot
    prefix_lens[b] + i;
  * parent -1 means "child of the cached prefix" (forests allowed); parent[i] < i;
  * GQA: query head h reads kv head h // (Hq / Hkv);
  * softmax scale ``sm_scale`` (1/sqrt(128) in every workload), natural-log LSE.

Pinned by tests/test_oracle_attention.py: chain tree == causal attention (torch SDPA), star tree ==
prefix-plus-self (closed form at P=0, SDPA otherwise), path extraction == causal SDPA over
prefix ++ path(v) for every node, zero queries give lse = ln|visible set| and out = mean of visible
V, physical-page permutation invariance, node relabelling, unrelated-branch invariance.
"""
from __future__ import annotations

import numpy as np

PAGE_SIZE = 16


def ancestor_sets(parent: np.ndarray) -> list[set[int]]:
    """anc(n) = {n} U anc(parent(n)); parent -1 ends the walk.  Requires parent[i] < i."""
    anc: list[set[int]] = []
    for i, p in enumerate(parent.tolist()):
        if not (-1 <= p < i):
            raise ValueError(f"parent[{i}] = {p} is not in [-1, {i - 1}]")
        anc.append({i} | (anc[p] if p >= 0 else set()))
    return anc


def visible_slots(prefix_len: int, anc_n: set[int]) -> np.ndarray:
    """Logical key slots visible to a node: the whole prefix, then its ancestors' (and its own) slots."""
    return np.concatenate([np.arange(prefix_len, dtype=np.int64),
                           prefix_len + np.array(sorted(anc_n), dtype=np.int64)])


def gather_slots(cache: np.ndarray, block_row: np.ndarray, slots: np.ndarray, kv_head: int) -> np.ndarray:
    """Logical slot t lives in physical page block_row[t // 16], row t % 16."""
    pages = block_row[slots // PAGE_SIZE]
    return cache[pages, slots % PAGE_SIZE, kv_head, :].astype(np.float64)


def visibility_mask(prefix_len: int, anc: list[set[int]]) -> np.ndarray:
    """bool [N, prefix_len + N]: row n is True exactly on visible_slots(prefix_len, anc[n])."""
    n_nodes = len(anc)
    mask = np.zeros((n_nodes, prefix_len + n_nodes), dtype=bool)
    for n in range(n_nodes):
        mask[n, visible_slots(prefix_len, anc[n])] = True
    return mask


def tree_attention(q, k_cache, v_cache, block_table, prefix_lens, tree_offsets, parent, sm_scale,
                   num_kv_heads=None, rows=None):
    """Returns (out float64 [T, Hq, D], lse float64 [T, Hq]).

    Per (sequence, node, q head): s_t = sm_scale * <q, K[t]> for every visible slot t,
    out = sum_t softmax(s)_t V[t], lse = ln sum_t exp(s_t).  Invisible slots take weight exactly 0, so
    the weighted sum is written as one matrix product over all slots of the sequence.

    ``rows`` optionally restricts the work to a list of (global node index, q head) pairs; the other
    entries are left as NaN."""
    q = np.asarray(q)
    T, Hq, D = q.shape
    Hkv = k_cache.shape[2] if num_kv_heads is None else num_kv_heads
    group = Hq // Hkv
    out = np.full((T, Hq, D), np.nan)
    lse = np.full((T, Hq), np.nan)
    want = None
    if rows is not None:
        want = np.zeros((T, Hq), dtype=bool)
        for t, h in rows:
            want[int(t), int(h)] = True
    for b in range(len(prefix_lens)):
        P = int(prefix_lens[b])
        o0, o1 = int(tree_offsets[b]), int(tree_offsets[b + 1])
        if o1 == o0:
            continue
        anc = ancestor_sets(np.asarray(parent[o0:o1]))
        mask = visibility_mask(P, anc)
        slots = np.arange(P + (o1 - o0), dtype=np.int64)
        for h in range(Hq):
            sel = np.arange(o1 - o0) if want is None else np.nonzero(want[o0:o1, h])[0]
            if sel.size == 0:
                continue
            kvh = h // group
            K = gather_slots(k_cache, block_table[b], slots, kvh)
            V = gather_slots(v_cache, block_table[b], slots, kvh)
            s = sm_scale * (q[o0 + sel, h].astype(np.float64) @ K.T)
            s = np.where(mask[sel], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            w = np.exp(s - m)
            l = w.sum(axis=1, keepdims=True)
            out[o0 + sel, h] = (w @ V) / l
            lse[o0 + sel, h] = (m + np.log(l))[:, 0]
    return out, lse


def tree_attention_inputs(inp, rows=None):
    """Convenience wrapper taking a ``synth.AttentionInputs``-like object."""
    return tree_attention(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.prefix_lens,
                          inp.tree_offsets, inp.parent, inp.sm_scale, inp.num_kv_heads, rows)
