"""Oracle: greedy acceptance walk over a verified draft tree.

Definition followed ([JF] technical summary section 1 and the lay section: the target checks all
drafted tokens at once and keeps the longest agreeing prefix; section 4 reports tau, the accepted
tokens per step): starting at the root, take the target's argmax at the current node; if a child of
the current node carries that token, move to it and repeat; otherwise stop.  The argmax at the last
accepted node is the bonus token the target contributes for free.

Readings: ties in the argmax go to the lowest token id; if several children carry the argmax token,
the lowest node index wins; accepted_len counts accepted draft nodes (root excluded) and never
exceeds ``max_depth``; path[0] = 0 (root), unused entries are -1.

Pinned by tests/test_oracle_accept.py: planted paths (closed form), root mismatch -> 0, a fully
agreeing chain -> max depth, brute force over all root paths on small trees, a hand-worked example
in tests/golden/.
"""
from __future__ import annotations

import numpy as np


def first_argmax(row) -> int:
    """Index of the largest entry; the lowest index among equal maxima."""
    return int(np.argmax(row))


def accept(token, parent, target_logits, max_depth):
    """token, parent int [B, N]; target_logits float [B, N, V].  Returns (accepted_len int32[B],
    path int32[B, max_depth + 1], bonus int32[B])."""
    token = np.asarray(token)
    parent = np.asarray(parent)
    B, N = token.shape
    acc = np.zeros(B, dtype=np.int32)
    path = np.full((B, max_depth + 1), -1, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    for b in range(B):
        cur, L = 0, 0
        path[b, 0] = 0
        while True:
            a = first_argmax(target_logits[b, cur])
            if L == max_depth:
                break
            nxt = -1
            for c in range(N):
                if parent[b, c] == cur and token[b, c] == a:
                    nxt = c
                    break
            if nxt < 0:
                break
            L += 1
            path[b, L] = nxt
            cur = nxt
        acc[b] = L
        bonus[b] = a
    return acc, path, bonus
