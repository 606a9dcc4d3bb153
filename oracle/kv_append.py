"""Oracle: writing the tree tokens' K/V into the paged cache with rotary positions (TEST INFRASTRUCTURE).

What it restates: the target model verifies the whole tree in one forward pass ([JF] technical summary section 1),
inside a paged-KV serving engine (section 3); each tree token's key and value must sit in the cache where tree
attention reads them, and the key (and query) carry the token's position.  The pages leave the details open; the
readings used:

  * node j of sequence b is written at cache slot P_b + j (where tree attention reads it);
  * its position is P_b + depth_j with the root at depth 0: a node's position is that of the last prefix token
    plus its depth, so siblings share a position and every root path reads as consecutive positions;
  * rotary embedding over the whole head in the split-half layout: element i and element i + d/2 form a pair
    rotated by the angle pos * theta^(-2i/d), for i < d/2 (theta is a parameter of the call);
  * V is written unrotated; the query, when given, is rotated in place with the same position.

Pinned by tests/test_oracle_kv_append.py: position 0 is the identity, pair norms are kept, scores depend only on
relative position, a hand-worked d = 4 example, the same result from a complex-number formulation, and the slots
the nodes land in.
"""
from __future__ import annotations

import numpy as np

PAGE = 16


def rope(x, pos, theta):
    """x float [..., d] (d even); pos scalar or [...] broadcastable over x[..., 0].  Returns float64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = np.power(float(theta), -2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def node_positions(prefix_lens, tree_offsets, depth):
    """Position of every node of the flattened tree batch: P_b + depth."""
    pos = np.zeros(int(tree_offsets[-1]), dtype=np.int64)
    for b in range(len(prefix_lens)):
        o0, o1 = int(tree_offsets[b]), int(tree_offsets[b + 1])
        pos[o0:o1] = int(prefix_lens[b]) + np.asarray(depth[o0:o1], dtype=np.int64)
    return pos


def tree_kv_append(k_new, v_new, q, k_cache, v_cache, block_table, prefix_lens, tree_offsets, depth, theta):
    """k_new, v_new [T, Hkv, d]; q [T, Hq, d] or None; caches [pages, 16, Hkv, d]; block_table [B, max_pages];
    prefix_lens [B]; tree_offsets [B + 1]; depth [T] (root 0).  Returns float64 (k_cache, v_cache, q) with the
    rotated keys, the values and the rotated queries in place of the inputs (which are not modified)."""
    k = np.array(k_cache, dtype=np.float64, copy=True)
    v = np.array(v_cache, dtype=np.float64, copy=True)
    pos = node_positions(prefix_lens, tree_offsets, depth)
    q_out = None if q is None else rope(q, pos[:, None], theta)
    kr = rope(k_new, pos[:, None], theta)
    for b in range(len(prefix_lens)):
        P = int(prefix_lens[b])
        for t in range(int(tree_offsets[b]), int(tree_offsets[b + 1])):
            s = P + (t - int(tree_offsets[b]))
            pg, off = int(block_table[b][s // PAGE]), s % PAGE
            k[pg, off] = kr[t]
            v[pg, off] = v_new[t]
    return k, v, q_out
