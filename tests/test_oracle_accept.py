"""Pins for oracle.accept: planted paths (closed form), special cases, brute force over root paths,
and a hand-worked example."""
import json
import os

import numpy as np
import pytest

from oracle.accept import accept
from oracle.build_tree import build_tree
from tree_verify_attention_jf_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_handworked_golden():
    g = json.load(open(os.path.join(GOLDEN, "accept_handworked.json")))
    V, N = g["vocab"], len(g["parent"])
    x = np.zeros((1, N, V), dtype=np.float32)
    for i, a in enumerate(g["row_argmax"]):
        x[0, i, a] = 1.0
    for case in g["cases"]:
        acc, path, bonus = accept(np.array([g["token"]]), np.array([g["parent"]]), x, case["max_depth"])
        assert acc[0] == case["accepted_len"]
        assert path[0].tolist() == case["path"]
        assert bonus[0] == case["bonus"]


def test_planted_paths_on_built_trees():
    x, roots = synth.draft_logits(11, 4, 16, 2000)
    tree = build_tree(x, roots, 4, 64, 16)
    tgt, paths = synth.target_logits_with_path(12, tree["parent"], tree["token"], 2000)
    acc, path, bonus = accept(tree["token"], tree["parent"], tgt, 16)
    for b in range(4):
        assert acc[b] == len(paths[b]) - 1
        assert path[b, :acc[b] + 1].tolist() == paths[b]
        assert (path[b, acc[b] + 1:] == -1).all()
        assert bonus[b] == int(np.argmax(tgt[b, paths[b][-1]]))


def test_root_mismatch_and_full_chain():
    N, V = 6, 10
    par = synth.chain_tree(N)
    par[0] = -1
    tok = np.array([[9, 1, 2, 3, 4, 5]])
    x = np.zeros((1, N, V), dtype=np.float32)
    x[0, 0, 7] = 1.0  # root's argmax is 7, its only child carries 1
    acc, path, bonus = accept(tok, par[None], x, 5)
    assert acc[0] == 0 and bonus[0] == 7 and path[0].tolist() == [0, -1, -1, -1, -1, -1]
    for i in range(N - 1):
        x[0, i] = 0
        x[0, i, tok[0, i + 1]] = 1.0
    x[0, N - 1] = 0
    x[0, N - 1, 0] = 3.0
    acc, path, bonus = accept(tok, par[None], x, 5)
    assert acc[0] == 5 and path[0].tolist() == [0, 1, 2, 3, 4, 5] and bonus[0] == 0


def test_argmax_ties_take_lowest_id():
    x = np.zeros((1, 2, 6), dtype=np.float32)
    x[0, 0, [2, 4]] = 5.0
    acc, path, bonus = accept(np.array([[0, 4]]), np.array([[-1, 0]]), x, 3)
    assert acc[0] == 0 and bonus[0] == 2
    acc, path, bonus = accept(np.array([[0, 2]]), np.array([[-1, 0]]), x, 3)
    assert acc[0] == 1 and path[0, 1] == 1


@pytest.mark.parametrize("seed", range(5))
def test_brute_force_root_paths(seed):
    rng = np.random.default_rng(seed)
    N, V = 30, 5
    par = synth.bushy_tree(rng, N, 3, 8)
    tok = np.zeros(N, dtype=np.int64)
    for p in range(N):  # distinct sibling tokens
        kids = np.nonzero(par == p)[0]
        tok[kids] = rng.choice(V, size=len(kids), replace=False)
    x = rng.standard_normal((1, N, V)).astype(np.float32)
    am = x[0].argmax(axis=1)
    # A node is accepted iff every edge (u -> w) on its root path has token[w] == argmax(row u).
    best, best_len = 0, 0
    for v in range(1, N):
        path, w = [], v
        while w > 0:
            path.append(w)
            w = int(par[w])
        if all(tok[w] == am[par[w]] for w in path) and len(path) > best_len:
            best, best_len = v, len(path)
    acc, pth, bonus = accept(tok[None], par[None], x, 8)
    assert acc[0] == best_len
    assert pth[0, best_len] == best
    assert bonus[0] == am[best]
