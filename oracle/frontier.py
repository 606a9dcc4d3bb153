"""Oracle: best-first tree expansion from per-node (path-conditioned) draft logits, one frontier at a time
(TEST INFRASTRUCTURE).

What it restates ([JF] technical summary section 2): the draft head conditions every node on the tokens of its
own root path -- the branch factorisation q(pi(v)|x) = prod_{u in pi(v)} q(y_u | x, h, pi_<u) -- and the
candidate tree is grown best-first by cumulative draft log-probability until it holds the budget.  With
path-conditioned logits a node's children can be scored only after the draft head has run on that node, so the
tree grows in rounds: the draft head scores the current frontier, then the best untaken children of every node
scored so far join the tree and become the next frontier.

Readings (the pages give no pseudo-code for this variant):
  * one round scores the frontier nodes (row j of the round's logits belongs to frontier node
    frontier_begin + j) and then adds at most ``width`` nodes, and never more than the budget allows;
  * a node's candidate children are the top-``topk`` tokens of its own row, ordered by (logit desc, id asc),
    with lp = x_tok - lse computed in float64 (the per-depth build's row statistics); a node at
    ``max_depth`` has none;
  * the candidate (parent u, rank r) has key = key(u) + lp_u[r] in float64; the round takes the best untaken
    candidates of all scored nodes in the per-depth build's order (key desc, depth asc, parent index asc, rank
    asc) and appends them in that order; a parent's ranks are taken in rank order;
  * a new tree (no nodes yet) starts with its root (node 0: the root token, parent -1, depth 0, key 0), which is
    the first round's frontier;
  * scores are the float64 keys rounded to float32, as in the per-depth build.

With width 1 every round adds one node and scores it before the next pop: that is exactly the per-depth build's
priority-queue expansion when each node's row is its depth's row.

Pinned by tests/test_oracle_frontier.py: width 1 with per-depth rows equals oracle.build_tree; width 1 with
path-conditioned rows equals a brute-force enumeration of the full tree's keys; an unlimited width grows the tree
level by level (closed form); invariants (parent[i] < i, round sizes, child key - parent key = the child's lp
from scipy's logsumexp of the parent's row, distinct sibling tokens).
"""
from __future__ import annotations

import numpy as np

from .build_tree import row_stats, topk_tokens


class FrontierState:
    """One sequence's tree under construction: the nodes so far and every scored node's candidate children."""

    def __init__(self, budget: int):
        self.budget = budget
        self.parent: list[int] = []
        self.token: list[int] = []
        self.depth: list[int] = []
        self.key: list[float] = []
        self.cand_tok: list[np.ndarray] = []   # per node: its top-k tokens (empty until scored)
        self.cand_lp: list[np.ndarray] = []    # per node: their float64 log-probabilities
        self.next_rank: list[int] = []         # per node: first rank not yet taken
        self.frontier_begin = 0

    @property
    def num_nodes(self) -> int:
        return len(self.parent)

    def frontier(self) -> range:
        return range(self.frontier_begin, self.num_nodes)

    def path_tokens(self, i: int) -> tuple[int, ...]:
        """Tokens on the root path of node i, root first."""
        toks = []
        while i >= 0:
            toks.append(self.token[i])
            i = self.parent[i]
        return tuple(reversed(toks))


def _append(state: FrontierState, parent: int, token: int, depth: int, key: float) -> None:
    state.parent.append(parent)
    state.token.append(int(token))
    state.depth.append(depth)
    state.key.append(key)
    state.cand_tok.append(np.zeros(0, np.int64))
    state.cand_lp.append(np.zeros(0))
    state.next_rank.append(0)


def node_children(row, topk: int):
    """A scored node's candidate children: its row's top-k tokens (logit desc, id asc) and their float64
    log-probabilities lp = x - lse."""
    row = np.asarray(row)
    _, lse = row_stats(row)
    tok = topk_tokens(row, topk)
    return tok, row[tok].astype(np.float64) - lse


def candidate_key(parent_key: float, lp: float) -> float:
    """Cumulative draft log-probability of a child: its parent's plus its own (float64)."""
    return parent_key + lp


def untaken(state: FrontierState, u: int) -> range:
    """Ranks of node u's candidates not yet in the tree (ranks are taken in order)."""
    return range(state.next_rank[u], len(state.cand_tok[u]))


def start_tree(state: FrontierState, root_token: int) -> None:
    """A new tree: the root alone, which is the first frontier."""
    if state.num_nodes == 0:
        _append(state, -1, root_token, 0, 0.0)
        state.frontier_begin = 0


def expand_frontier(state: FrontierState, rows, root_token: int, topk: int, max_depth: int, width: int) -> int:
    """One round: score the frontier with ``rows`` (row j = logits at node frontier_begin + j), then append the
    best untaken candidates.  Returns the number of nodes added."""
    start_tree(state, root_token)
    # 1. score the frontier: each node's candidate children from its own row
    for j, i in enumerate(state.frontier()):
        if state.depth[i] >= max_depth:
            state.cand_tok[i] = np.zeros(0, np.int64)
            state.cand_lp[i] = np.zeros(0)
            continue
        state.cand_tok[i], state.cand_lp[i] = node_children(rows[j], topk)
        state.next_rank[i] = 0
    # 2. the round's picks: the best untaken candidates of every scored node, in the total order
    n0 = state.num_nodes
    want = min(width, state.budget - n0)
    cands = []
    for u in range(n0):
        for r in untaken(state, u):
            k = candidate_key(state.key[u], state.cand_lp[u][r])
            cands.append((-k, state.depth[u] + 1, u, r))
    cands.sort()
    picks = cands[:max(want, 0)]
    # 3. append them in that order; they are the next frontier
    for negk, d, u, r in picks:
        _append(state, u, state.cand_tok[u][r], d, -negk)
        state.next_rank[u] = r + 1
    state.frontier_begin = n0
    return len(picks)


def grow_tree(row_for, root_tokens, topk, budget, max_depth, width, max_rounds=10_000):
    """Runs rounds until every sequence holds ``budget`` nodes or has no candidate left.  ``row_for(b, state, i)``
    returns the logits row of node i of sequence b (the draft head's output at that node).  Returns dict of
    parent, token, depth (int32 [B, budget], -1 / 0 past the end), score (float32), key (float64), num_nodes
    (int32 [B]) and the list of per-round frontier sizes per sequence."""
    B = len(root_tokens)
    states = [FrontierState(budget) for _ in range(B)]
    rounds = [[] for _ in range(B)]
    for b in range(B):
        start_tree(states[b], root_tokens[b])
        for _ in range(max_rounds):
            st = states[b]
            fr = list(st.frontier())
            if not fr or st.num_nodes >= budget:
                break
            rows = [row_for(b, st, i) for i in fr]
            added = expand_frontier(st, rows, root_tokens[b], topk, max_depth, width)
            rounds[b].append(added)
            if added == 0:
                break
    out = dict(parent=np.full((B, budget), -1, np.int32), token=np.zeros((B, budget), np.int32),
               depth=np.zeros((B, budget), np.int32), score=np.zeros((B, budget), np.float32),
               key=np.zeros((B, budget)), num_nodes=np.zeros(B, np.int32), rounds=rounds)
    for b, st in enumerate(states):
        n = st.num_nodes
        out["parent"][b, :n] = st.parent
        out["token"][b, :n] = st.token
        out["depth"][b, :n] = st.depth
        out["key"][b, :n] = st.key
        out["score"][b, :n] = np.asarray(st.key, dtype=np.float32)
        out["num_nodes"][b] = n
    return out
