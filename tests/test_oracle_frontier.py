"""Pins for oracle.frontier (round-by-round best-first expansion from per-node draft logits): equality with the
per-depth build at width 1 when every node's row is its depth's row, brute-force enumeration of the full tree's
keys at width 1 with path-conditioned rows, the level-by-level closed form at unlimited width, and invariants."""
import itertools

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle.build_tree import build_tree
from oracle.frontier import FrontierState, expand_frontier, grow_tree
from tree_verify_attention_jf_b200 import synth


def per_depth_rows(x):
    """Node i's row is its depth's row: x[b, d] scores the children at depth d + 1 (a node at the last depth has no
    children; the row it is given is never read)."""
    return lambda b, st, i: x[b, min(st.depth[i], x.shape[1] - 1)]


def path_rows(seed, vocab, plant=8):
    return lambda b, st, i: synth.path_logits(seed + 1000 * b, st.path_tokens(i), vocab, plant=plant)


@pytest.mark.parametrize("seed,topk,budget,max_depth,V", [(1, 4, 60, 6, 64), (2, 2, 31, 8, 40), (3, 3, 40, 4, 30),
                                                          (4, 1, 9, 8, 16), (5, 8, 100, 5, 200)])
def test_width_one_equals_the_per_depth_build(seed, topk, budget, max_depth, V):
    x, roots = synth.draft_logits(seed, 3, max_depth, V)
    ref = build_tree(x, roots, topk, budget, max_depth)
    got = grow_tree(per_depth_rows(x), roots, topk, budget, max_depth, width=1)
    for k in ("parent", "token", "depth", "key", "score"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    assert all(r == [1] * (budget - 1) for r in got["rounds"])


def test_width_one_equals_tied_per_depth_build():
    # integer logits: many exact ties between keys, broken by (depth, parent, rank)
    rng = np.random.default_rng(7)
    x = rng.integers(0, 3, size=(2, 5, 12)).astype(np.float32)
    roots = np.array([3, 4], np.int32)
    ref = build_tree(x, roots, 3, 50, 5)
    got = grow_tree(per_depth_rows(x), roots, 3, 50, 5, width=1)
    for k in ("parent", "token", "depth", "key"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def brute_force(row_of_path, root, topk, max_depth):
    """Every node of the full topk-ary tree with path-conditioned rows: (key, token path)."""
    out = []

    def visit(path, key, depth):
        out.append((key, path))
        if depth == max_depth:
            return
        row = row_of_path(path).astype(np.float64)
        lse = logsumexp(row)
        order = np.lexsort((np.arange(row.size), -row))[:topk]
        for t in order:
            visit(path + (int(t),), key + (row[t] - lse), depth + 1)

    visit((int(root),), 0.0, 0)
    return out


@pytest.mark.parametrize("seed,topk,max_depth,budget", [(11, 2, 4, 20), (12, 3, 3, 30), (13, 3, 4, 9)])
def test_width_one_with_path_conditioned_rows_is_exact_best_first(seed, topk, max_depth, budget):
    V = 12
    roots = np.array([5], np.int32)
    rows = path_rows(seed, V, plant=0)  # continuous draws: no two keys tie
    got = grow_tree(rows, roots, topk, budget, max_depth, width=1)
    allnodes = brute_force(lambda p: synth.path_logits(seed, p, V, plant=0), roots[0], topk, max_depth)
    allnodes.sort(key=lambda kp: -kp[0])
    want = allnodes[:budget]
    st_paths = []
    for i in range(budget):
        path, j = [], i
        while j >= 0:
            path.append(int(got["token"][0, j]))
            j = int(got["parent"][0, j])
        st_paths.append(tuple(reversed(path)))
    assert st_paths == [p for _, p in want]
    np.testing.assert_allclose(got["key"][0], [k for k, _ in want], rtol=0, atol=1e-12)


def level_by_level(row_of_path, root, topk, budget, max_depth):
    """Closed form at unlimited width: round t adds every depth-t child, sorted by (key desc, parent, rank), until
    the budget; returns (paths, keys) in node order."""
    paths, keys = [(int(root),)], [0.0]
    level = [0]
    while len(paths) < budget and level:
        cands = []
        for u in level:
            if len(paths[u]) - 1 >= max_depth:
                continue
            row = row_of_path(paths[u]).astype(np.float64)
            lse = logsumexp(row)
            order = np.lexsort((np.arange(row.size), -row))[:topk]
            for r, t in enumerate(order):
                cands.append((-(keys[u] + row[t] - lse), u, r, int(t)))
        cands.sort()
        nxt = []
        for negk, u, r, t in cands[:budget - len(paths)]:
            nxt.append(len(paths))
            paths.append(paths[u] + (t,))
            keys.append(-negk)
        level = nxt
    return paths, keys


@pytest.mark.parametrize("seed,topk,max_depth,budget", [(21, 3, 4, 40), (22, 4, 3, 85), (23, 2, 6, 100)])
def test_unlimited_width_grows_level_by_level(seed, topk, max_depth, budget):
    V = 30
    roots = np.array([2], np.int32)
    got = grow_tree(path_rows(seed, V), roots, topk, budget, max_depth, width=10 ** 6)
    paths, keys = level_by_level(lambda p: synth.path_logits(seed, p, V), roots[0], topk, budget, max_depth)
    n = len(paths)
    assert got["num_nodes"][0] == n
    got_paths = []
    for i in range(n):
        path, j = [], i
        while j >= 0:
            path.append(int(got["token"][0, j]))
            j = int(got["parent"][0, j])
        got_paths.append(tuple(reversed(path)))
    assert got_paths == paths
    np.testing.assert_allclose(got["key"][0, :n], keys, rtol=0, atol=1e-12)


@pytest.mark.parametrize("width", [3, 7, 16, 32])
def test_invariants(width):
    V, topk, budget, max_depth = 500, 4, 120, 7
    roots = np.array([9, 10], np.int32)
    seed = 31 + width
    got = grow_tree(path_rows(seed, V), roots, topk, budget, max_depth, width)
    for b in range(2):
        n = int(got["num_nodes"][b])
        assert n == budget
        par, tok, dep, key = got["parent"][b], got["token"][b], got["depth"][b], got["key"][b]
        rounds = got["rounds"][b]
        assert sum(rounds) == n - 1
        assert all(1 <= r <= width for r in rounds)
        assert rounds[0] == min(width, topk)  # the first round can only take the root's children
        # the round each node was added in; a node's parent was added in an earlier round
        rnd = np.zeros(n, np.int64)
        pos = 1
        for t, r in enumerate(rounds, start=1):
            rnd[pos:pos + r] = t
            # keys within one round are non-increasing (appended best-first)
            assert np.all(np.diff(key[pos:pos + r]) <= 0)
            pos += r
        states = {}
        for i in range(1, n):
            p = int(par[i])
            assert 0 <= p < i and rnd[p] < rnd[i]
            assert dep[i] == dep[p] + 1 <= max_depth
            path, j = [], p
            while j >= 0:
                path.append(int(tok[j]))
                j = int(par[j])
            row = synth.path_logits(seed + 1000 * b, tuple(reversed(path)), V).astype(np.float64)
            assert key[i] - key[p] == pytest.approx(row[tok[i]] - logsumexp(row), abs=1e-9)
            states.setdefault(p, []).append(int(tok[i]))
        for p, toks in states.items():
            assert len(set(toks)) == len(toks) <= topk


def test_round_by_round_state_and_exhaustion():
    """A tree that runs out of candidates before the budget: max depth 2, topk 2 gives 1 + 2 + 4 nodes."""
    st = FrontierState(budget=50)
    V = 20
    rounds = []
    from oracle.frontier import start_tree
    start_tree(st, 1)
    while True:
        rows = [synth.path_logits(5, st.path_tokens(i), V) for i in st.frontier()]
        added = expand_frontier(st, rows, 1, 2, 2, width=3)
        rounds.append(added)
        if added == 0:
            break
    assert st.num_nodes == 7 and rounds == [2, 3, 1, 0]
    assert list(st.frontier()) == []


def test_budget_counts_the_root():
    x, roots = synth.draft_logits(3, 1, 4, 50)
    got = grow_tree(per_depth_rows(x), roots, 4, 1, 4, width=8)
    assert got["num_nodes"][0] == 1 and got["rounds"][0] == []
    got = grow_tree(per_depth_rows(x), roots, 4, 2, 4, width=8)
    assert got["num_nodes"][0] == 2 and got["rounds"][0] == [1]
    assert list(itertools.chain(got["parent"][0])) == [-1, 0]
