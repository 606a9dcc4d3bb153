"""Pins for oracle.build_tree: scipy logsumexp and a stable argsort for the row statistics, brute-force
enumeration of small full trees, closed-form special cases, a hand-worked example, invariants."""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle.build_tree import build_tree, row_stats, topk_tokens
from tree_verify_attention_jf_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_row_stats_against_scipy():
    rng = np.random.default_rng(0)
    for scale in (0.1, 2.0, 30.0):
        x = (rng.standard_normal(5000) * scale).astype(np.float32)
        m, lse = row_stats(x)
        assert m == float(x.max())
        assert lse == pytest.approx(float(logsumexp(x.astype(np.float64))), abs=1e-12)


def test_topk_order_against_stable_argsort():
    rng = np.random.default_rng(1)
    x = rng.integers(0, 6, size=300).astype(np.float32)  # many ties: id ascending breaks them
    want = np.argsort(-x, kind="stable")[:8]
    np.testing.assert_array_equal(topk_tokens(x, 8), want)


def rank_tuple(par, tok, lists, i):
    """Node i -> tuple of ranks along its root path (rank = position of its token in its depth's top-k)."""
    ranks = []
    while i > 0:
        d = len(ranks)
        ranks.append(i)
        i = int(par[i])
    out = []
    nodes = ranks[::-1]
    for depth, n in enumerate(nodes, start=1):
        out.append(int(np.nonzero(lists[depth] == tok[n])[0][0]))
    return tuple(out)


@pytest.mark.parametrize("seed,topk,max_depth,budget", [(2, 3, 4, 40), (3, 2, 4, 31), (4, 3, 3, 39), (5, 1, 4, 5)])
def test_brute_force_full_tree(seed, topk, max_depth, budget):
    rng = np.random.default_rng(seed)
    V = 12
    x = (rng.standard_normal((1, max_depth, V)) * 2).astype(np.float32)
    res = build_tree(x, np.array([7]), topk, budget, max_depth)
    # Independent enumeration: every node of the full topk-ary tree, key = sum of per-depth log-probs.
    lists, lps = {}, {}
    for k in range(1, max_depth + 1):
        row = x[0, k - 1].astype(np.float64)
        lists[k] = np.argsort(-row, kind="stable")[:topk]
        lps[k] = row[lists[k]] - logsumexp(row)
    nodes = []
    for d in range(1, max_depth + 1):
        for ranks in itertools.product(range(topk), repeat=d):
            nodes.append((sum(lps[k + 1][r] for k, r in enumerate(ranks)), d, ranks))
    nodes.sort(key=lambda t: (-t[0], t[1]))
    expect = nodes[:budget - 1]
    got = [rank_tuple(res["parent"][0], res["token"][0], lists, i) for i in range(1, budget)]
    assert got == [e[2] for e in expect]
    np.testing.assert_allclose(res["key"][0, 1:], [e[0] for e in expect], rtol=0, atol=1e-12)


def test_topk1_is_chain_of_argmaxes():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, 6, 50)).astype(np.float32)
    res = build_tree(x, np.array([1, 2]), 1, 7, 6)
    for b in range(2):
        np.testing.assert_array_equal(res["parent"][b], np.arange(-1, 6))
        np.testing.assert_array_equal(res["token"][b, 1:], x[b].argmax(axis=1))
        np.testing.assert_array_equal(res["depth"][b], np.arange(7))


def test_flat_first_row_gives_star():
    rng = np.random.default_rng(7)
    V, topk = 20, 5
    x = rng.standard_normal((1, 3, V)).astype(np.float32)
    x[0, 0] = 0.25  # flat: every depth-1 token has lp = -ln V; any child is strictly worse
    res = build_tree(x, np.array([0]), topk, 1 + topk, 3)
    np.testing.assert_array_equal(res["parent"][0], [-1] + [0] * topk)
    np.testing.assert_array_equal(res["token"][0, 1:], np.arange(topk))  # ties -> lowest ids
    np.testing.assert_allclose(res["score"][0, 1:], -np.log(V), rtol=1e-6)


def test_handworked_golden():
    g = json.load(open(os.path.join(GOLDEN, "build_handworked.json")))
    x = np.log(np.array(g["probs"], dtype=np.float64)).astype(np.float32)[None]
    res = build_tree(x, np.array([g["root_token"]]), g["topk"], g["budget"], g["max_depth"])
    np.testing.assert_array_equal(res["parent"][0], g["parent"])
    np.testing.assert_array_equal(res["token"][0], g["token"])
    np.testing.assert_array_equal(res["depth"][0], g["depth"])
    np.testing.assert_allclose(res["score"][0], g["score"], atol=1e-6)


def test_invariants_on_planted_logits():
    x, roots = synth.draft_logits(8, 3, 16, 3000)
    res, margin = build_tree(x, roots, 4, 256, 16, return_margin=True)
    for b in range(3):
        par, tok, sc, dep, key = (res[k][b] for k in ("parent", "token", "score", "depth", "key"))
        assert par[0] == -1 and dep[0] == 0 and tok[0] == roots[b] and sc[0] == 0
        assert all(0 <= par[i] < i for i in range(1, 256))
        assert np.all(np.diff(key) <= 0)
        assert dep.max() <= 16
        for i in range(1, 256):
            assert dep[i] == dep[par[i]] + 1
            row = x[b, dep[i] - 1].astype(np.float64)
            assert key[i] - key[par[i]] == pytest.approx(row[tok[i]] - logsumexp(row), abs=1e-9)
        for p in range(256):
            kids = tok[par == p]
            assert len(kids) <= 4 and len(set(kids.tolist())) == len(kids)
    assert margin.min() > 0


def test_budget_too_large_rejected():
    x = np.zeros((1, 2, 5), dtype=np.float32)
    with pytest.raises(ValueError):
        build_tree(x, np.array([0]), 2, 1 + 2 + 4 + 1, 2)
