"""GPU parity of jf_expand_frontier (through the C ABI) against oracle.frontier, round by round: every round's
tree (parent, token, depth bit-exact; score within 1e-5), node count and frontier start."""
import numpy as np
import pytest
import torch

from oracle.build_tree import build_tree as oracle_build
from oracle.frontier import FrontierState, expand_frontier, start_tree
from tree_verify_attention_jf_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu

SCORE_ABS = 1e-5


def run_rounds(row_for, roots, V, topk, budget, max_depth, width, pad_rows=0, max_rounds=10_000):
    """Grows the oracle trees and the GPU trees side by side from the same per-round logits and compares them
    after every round.  row_for(b, state, i) -> fp32 [V].  Rows past a sequence's frontier are NaN."""
    B = len(roots)
    states = [FrontierState(budget) for _ in range(B)]
    for b in range(B):
        start_tree(states[b], roots[b])
    dev = torch.device("cuda")
    tree = api.FrontierTree(B, budget, topk, dev)
    roots_d = torch.from_numpy(np.asarray(roots, np.int32)).to(dev)
    rounds = 0
    for _ in range(max_rounds):
        fr = [list(st.frontier()) if st.num_nodes < budget else [] for st in states]
        if all(len(f) == 0 for f in fr):
            break
        F = max(len(f) for f in fr) + pad_rows
        logits = np.full((B, F, V), np.nan, np.float32)
        for b in range(B):
            for j, i in enumerate(fr[b]):
                logits[b, j] = row_for(b, states[b], i)
            if fr[b]:
                expand_frontier(states[b], [logits[b, j] for j in range(len(fr[b]))], roots[b], topk, max_depth, width)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        api.expand_frontier(torch.from_numpy(logits).to(dev), roots_d, tree, max_depth, width, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        rounds += 1
        n_g = tree.num_nodes.cpu().numpy()
        fb_g = tree.frontier_begin.cpu().numpy()
        par, tok = tree.parent.cpu().numpy(), tree.token.cpu().numpy()
        dep, sc = tree.depth.cpu().numpy(), tree.score.cpu().numpy()
        for b, st in enumerate(states):
            if not fr[b]:
                continue
            n = st.num_nodes
            assert n_g[b] == n and fb_g[b] == st.frontier_begin, (rounds, b)
            np.testing.assert_array_equal(par[b, :n], st.parent)
            np.testing.assert_array_equal(tok[b, :n], st.token)
            np.testing.assert_array_equal(dep[b, :n], st.depth)
            np.testing.assert_allclose(sc[b, :n], np.asarray(st.key, np.float32), rtol=0, atol=SCORE_ABS)
    return states, tree, rounds


def test_full_vocab_path_conditioned_rounds():
    """Batch 4 over the full 151936-token vocabulary, top-4, budget 256, max depth 16, 32 nodes per round."""
    V, B = synth.VOCAB, 4
    roots = [11, 22, 33, 44]
    states, tree, rounds = run_rounds(lambda b, st, i: synth.path_logits(700 + b, st.path_tokens(i), V), roots, V,
                                      4, 256, 16, 32)
    assert all(st.num_nodes == 256 for st in states)
    # rounds add 4 (the root's children), 16 (theirs), then 32 seven times, then the last 11: 1 + 255 nodes
    assert rounds == 10


def test_width_one_reproduces_the_per_depth_build():
    V, B, topk, budget, max_depth = 3000, 3, 3, 40, 6
    x, roots = synth.draft_logits(17, B, max_depth, V)
    row = lambda b, st, i: x[b, min(st.depth[i], max_depth - 1)]
    states, tree, rounds = run_rounds(row, list(roots), V, topk, budget, max_depth, 1)
    assert rounds == budget - 1
    ref = oracle_build(x, roots, topk, budget, max_depth)
    np.testing.assert_array_equal(tree.parent.cpu().numpy(), ref["parent"])
    np.testing.assert_array_equal(tree.token.cpu().numpy(), ref["token"])
    np.testing.assert_array_equal(tree.depth.cpu().numpy(), ref["depth"])


@pytest.mark.parametrize("width", [1, 5, 64])
def test_tied_rows(width):
    """Integer logits: ties between tokens (id ascending) and between candidate keys (depth, parent, rank)."""
    V = 40
    rng = np.random.default_rng(width)
    table = rng.integers(0, 4, size=(64, V)).astype(np.float32)
    row = lambda b, st, i: table[(sum(st.path_tokens(i)) * 7 + b) % 64]
    run_rounds(row, [1, 2], V, 4, 120, 6, width)


def test_exhaustion_small_trees_and_padding_rows():
    V = 700
    # topk 2, max depth 2: 1 + 2 + 4 nodes, then no candidate is left; extra NaN rows are never read
    states, tree, _ = run_rounds(lambda b, st, i: synth.path_logits(5, st.path_tokens(i), V), [3], V, 2, 50, 2, 3,
                                 pad_rows=5)
    assert states[0].num_nodes == 7 and int(tree.num_nodes.item()) == 7
    # budget 1: the root alone
    _, tree, _ = run_rounds(lambda b, st, i: synth.path_logits(6, st.path_tokens(i), V), [4], V, 4, 1, 3, 8)
    assert int(tree.num_nodes.item()) == 0  # no round ran: the tree's root is created by its first round
    # topk 8, max depth 1: a star of 8
    states, tree, _ = run_rounds(lambda b, st, i: synth.path_logits(7, st.path_tokens(i), V), [5, 6], V, 8, 100, 1,
                                 16)
    assert all(st.num_nodes == 9 for st in states)


def test_device_checks_leave_the_tree_unchanged():
    dev = torch.device("cuda")
    V, B, budget = 500, 2, 30
    tree = api.FrontierTree(B, budget, 4, dev)
    roots = torch.tensor([1, 2], dtype=torch.int32, device=dev)
    logits = torch.from_numpy(np.stack([synth.path_logits(9, (1,), V), synth.path_logits(9, (2,), V)])[:, None]).to(dev)
    api.expand_frontier(logits.contiguous(), roots, tree, 5, 8)  # first round: 4 nodes + the root
    torch.cuda.synchronize()
    before = (tree.parent.clone(), tree.token.clone(), tree.num_nodes.clone(), tree.frontier_begin.clone())
    # the frontier (4 nodes) is longer than the rows given (1): flagged, nothing written
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    api.expand_frontier(logits.contiguous(), roots, tree, 5, 8, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.JF_ERR_DEVICE_CHECK
    for a, b in zip(before, (tree.parent, tree.token, tree.num_nodes, tree.frontier_begin)):
        assert torch.equal(a, b)
    # a node count past the budget: flagged
    tree.num_nodes[0] = budget + 1
    status.zero_()
    big = torch.zeros(B, 4, V, dtype=torch.float32, device=dev)
    api.expand_frontier(big, roots, tree, 5, 8, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.JF_ERR_DEVICE_CHECK
    assert int(tree.num_nodes[0].item()) == budget + 1
