"""Oracle: committing the accepted path's K/V into the paged cache (TEST INFRASTRUCTURE).

What it restates: [JF] technical summary section 1 (the target verifies all drafted tokens in one pass and keeps
the longest agreeing prefix) and section 3 (the method runs inside a paged-KV serving engine).  The pages leave the
cache update itself open; this is the plainest reading that the rest supports:

  * during verification, tree node j of sequence b sits at cache slot P_b + j (where tree attention reads it);
  * after the walk accepts the path [0, n_1, ..., n_L], the sequence continues with the root and the L accepted
    tokens, so slot P_b + i (i = 1 .. L) receives the K and V of slot P_b + n_i, for every kv head and all 128
    dimensions, while slot P_b (the root) keeps its own;
  * the prefix length becomes P_b + L + 1; slots past it are free and their contents are unspecified;
  * a sequence with an empty tree is left as it is.

Slot s of sequence b lives in page block_table[b, s // 16] at offset s % 16.

Pinned by tests/test_oracle_commit.py: a hand-worked example with values fixed by hand, the same result from a
dense formulation (gather the sequence, slice, scatter back), the committed cache reading as the accepted text
(token ids riding along as cache values), and the edge cases (nothing accepted, empty tree, a path whose sources
are destinations of later copies).
"""
from __future__ import annotations

import numpy as np

PAGE = 16


def locate(block_row, s):
    """(page, offset) of slot s of a sequence whose block-table row is block_row."""
    return int(block_row[s // PAGE]), s % PAGE


def commit_kv(k_cache, v_cache, block_table, prefix_lens, tree_offsets, path, accepted_len):
    """k_cache, v_cache [pages, 16, Hkv, D]; block_table int [B, max_pages]; prefix_lens int [B];
    tree_offsets int [B + 1]; path int [B, >= L + 1] (node indices, path[b, 0] = 0); accepted_len int [B].
    Returns (k, v, new_prefix_lens): new arrays, the inputs are not modified."""
    k = np.array(k_cache, copy=True)
    v = np.array(v_cache, copy=True)
    B = len(prefix_lens)
    new_p = np.array(prefix_lens, dtype=np.int64).copy()
    for b in range(B):
        P = int(prefix_lens[b])
        N = int(tree_offsets[b + 1]) - int(tree_offsets[b])
        if N == 0:
            continue
        L = int(accepted_len[b])
        # read every source before any write: a destination slot may be the source of a later copy
        srcs = []
        for i in range(1, L + 1):
            pg, off = locate(block_table[b], P + int(path[b][i]))
            srcs.append((k_cache[pg, off].copy(), v_cache[pg, off].copy()))
        for i in range(1, L + 1):
            pg, off = locate(block_table[b], P + i)
            k[pg, off], v[pg, off] = srcs[i - 1]
        new_p[b] = P + L + 1
    return k, v, new_p.astype(np.int32)
