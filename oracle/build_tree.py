"""Oracle: best-first draft-tree construction under a token budget (float64 keys).

Definition followed ([JF] technical summary section 2, "tree construction"; [JF] section 4 for the
budgets 16..256): the draft head emits logits for all tree depths in parallel; a branch score,
by default the cumulative draft log-probability along the path, ranks nodes; a best-first expansion
grows the candidate tree until it holds the budget.

Readings (the pages give no pseudo-code):
  * the input is per-depth logits [B, depths, V]; row k-1 scores every child at depth k, so all
    depth-(k-1) nodes share the same top-k children (the pages do not say how one pass yields
    path-conditioned logits; per-depth rows are the plainest reading);
  * log-prob of token v at depth k: lp = x_v - lse_k with lse_k = m + ln sum_v exp(x_v - m), computed
    in float64;
  * each node may have up to ``topk`` children: the top-k tokens of its depth's row, ordered by
    (logit descending, token id ascending);
  * the budget counts the root (node 0 = ``root_tokens[b]``, parent -1, depth 0, score 0), so a
    budget-256 tree has 256 rows of target logits;
  * best-first = a priority queue of candidates (parent p, rank r) keyed by score(p) + lp[depth(p)+1][r];
    pops are ordered by (key descending, depth ascending, parent index ascending, rank ascending);
    a popped candidate becomes the next node; then its next sibling (p, r+1) and its first child
    (i, 0) (if depth(i) < max_depth) join the queue;
  * scores are stored as float32 (rounded from the float64 key).

Pinned by tests/test_oracle_build.py: row statistics against scipy.special.logsumexp and a stable
argsort; brute-force enumeration of every node of small full trees; topk = 1 gives the chain of
per-depth argmaxes; a flat depth-1 row with budget 1 + topk gives the star of depth-1 tokens; a
hand-worked example in tests/golden/; structural invariants (parent[i] < i, scores non-increasing,
score(child) - score(parent) = lp, distinct sibling tokens, branching <= topk, depth <= max_depth).
"""
from __future__ import annotations

import heapq

import numpy as np


def row_stats(x: np.ndarray) -> tuple[float, float]:
    """(max, natural-log LSE) of one logits row; exp and sum in float64."""
    xd = np.asarray(x, dtype=np.float64)
    m = float(xd.max())
    return m, m + float(np.log(np.sum(np.exp(xd - m))))


def topk_tokens(x: np.ndarray, k: int) -> np.ndarray:
    """Token ids of the k largest logits, ordered by (logit descending, token id ascending)."""
    ids = np.arange(x.shape[0])
    order = np.lexsort((ids, -np.asarray(x, dtype=np.float64)))
    return order[:k].astype(np.int64)


def build_tree(draft_logits, root_tokens, topk, budget, max_depth, return_margin=False):
    """Returns dict(parent int32[B, budget], token int32[B, budget], score float32[B, budget],
    depth int32[B, budget], key float64[B, budget]) and, with ``return_margin``, the smallest gap
    between a popped key and the best key left in the queue at that moment, per sequence."""
    x = np.asarray(draft_logits)
    B, depths, V = x.shape
    if not (1 <= max_depth <= depths) or not (1 <= topk <= V) or budget < 1:
        raise ValueError("bad build arguments")
    parent = np.full((B, budget), -1, dtype=np.int32)
    token = np.zeros((B, budget), dtype=np.int32)
    score = np.zeros((B, budget), dtype=np.float32)
    depth = np.zeros((B, budget), dtype=np.int32)
    key = np.zeros((B, budget), dtype=np.float64)
    margins = np.full(B, np.inf)
    for b in range(B):
        tok = np.zeros((max_depth + 1, topk), dtype=np.int64)
        lp = np.zeros((max_depth + 1, topk), dtype=np.float64)
        for k in range(1, max_depth + 1):
            row = x[b, k - 1]
            _, lse = row_stats(row)
            tok[k] = topk_tokens(row, topk)
            lp[k] = row[tok[k]].astype(np.float64) - lse
        token[b, 0] = root_tokens[b]
        heap = []
        if max_depth >= 1 and budget > 1:
            heapq.heappush(heap, (-(0.0 + lp[1][0]), 1, 0, 0))
        n = 1
        while n < budget:
            if not heap:
                raise ValueError("budget exceeds the number of nodes of the full tree")
            negk, d, p, r = heapq.heappop(heap)
            if heap:
                margins[b] = min(margins[b], heap[0][0] - negk)
            i = n
            n += 1
            parent[b, i] = p
            token[b, i] = tok[d][r]
            depth[b, i] = d
            key[b, i] = -negk
            score[b, i] = np.float32(-negk)
            if r + 1 < topk:
                heapq.heappush(heap, (-(key[b, p] + lp[d][r + 1]), d, p, r + 1))
            if d < max_depth:
                heapq.heappush(heap, (-(key[b, i] + lp[d + 1][0]), d + 1, i, 0))
    res = dict(parent=parent, token=token, score=score, depth=depth, key=key)
    if return_margin:
        return res, margins
    return res
